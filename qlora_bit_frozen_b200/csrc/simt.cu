// simt.cu -- CUDA-core kernels of the QLoRA linear layer.
//
//  * qlinear_simt: the base GEMM with the weight decoded per element from its
//    nibble and block scale inside the K loop ("QLoRA Fine-Tuning", "Forward
//    and backward": decode each nibble inside the sums), fp32 accumulation,
//    plus the adapter term s * Aux * L^T in the epilogue.  Serves the fp32
//    compute mode (true fp32 FFMA; TF32 tensor cores cannot meet a 1e-5
//    relative error) and shapes the tensor-core path does not take.
//  * gemm_simt: a strided fp32-accumulating GEMM with optional split-K,
//    used for the adapter side products U = X A^T, V = dY B,
//    dA = s V^T X and dB = s dY^T U ("QLoRA on Mac", "Design / Q-LoRA
//    layer"; the LoRA chain rule).
//  * staging kernels that build the zero-padded bf16 adapter operands the
//    tensor-core kernels consume, and the split-K reduction.
#include "common.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

template <typename T>
__device__ __forceinline__ float ld_f32(const T* p, int64_t i) {
  return to_f32<T>(p[i]);
}

// Register-tiled 64x64 block, 4x4 outputs per thread.
struct Acc {
  float v[4][4];
};

__device__ __forceinline__ void mma_tile(const float (*Ps)[BM + 4], const float (*Qs)[BN + 4],
                                         int ty, int tx, Acc& acc) {
#pragma unroll
  for (int kk = 0; kk < BK; ++kk) {
    float4 a = *reinterpret_cast<const float4*>(&Ps[kk][ty * 4]);
    float4 b = *reinterpret_cast<const float4*>(&Qs[kk][tx * 4]);
    float av[4] = {a.x, a.y, a.z, a.w};
    float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc.v[i][j] = fmaf(av[i], bv[j], acc.v[i][j]);
  }
}

// C = alpha * sum_k P(m,k) Q(k,n) over the K range of split blockIdx.z.
template <typename TP, typename TQ>
__global__ void __launch_bounds__(NT) gemm_simt_kernel(int64_t M, int64_t N, int64_t K,
                                                       const TP* __restrict__ P, int64_t psm,
                                                       int64_t psk, const TQ* __restrict__ Q,
                                                       int64_t qsk, int64_t qsn, float alpha,
                                                       float* __restrict__ out, int64_t osm,
                                                       int64_t osn, int64_t kchunk,
                                                       int64_t split_stride) {
  __shared__ __align__(16) float Ps[BK][BM + 4];
  __shared__ __align__(16) float Qs[BK][BN + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int64_t m0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
  const int64_t k_lo = (int64_t)blockIdx.z * kchunk;
  const int64_t k_hi = k_lo + kchunk < K ? k_lo + kchunk : K;
  out += (int64_t)blockIdx.z * split_stride;
  Acc acc = {};
  for (int64_t k0 = k_lo; k0 < k_hi; k0 += BK) {
#pragma unroll
    for (int q = 0; q < (BM * BK) / NT; ++q) {
      const int e = tid + NT * q;
      int mm, kk;
      if (psk == 1) { mm = e / BK; kk = e % BK; } else { mm = e % BM; kk = e / BM; }
      const int64_t m = m0 + mm, k = k0 + kk;
      Ps[kk][mm] = (m < M && k < k_hi) ? ld_f32(P, m * psm + k * psk) : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < (BN * BK) / NT; ++q) {
      const int e = tid + NT * q;
      int nn, kk;
      if (qsk == 1) { nn = e / BK; kk = e % BK; } else { nn = e % BN; kk = e / BN; }
      const int64_t n = n0 + nn, k = k0 + kk;
      Qs[kk][nn] = (n < N && k < k_hi) ? ld_f32(Q, k * qsk + n * qsn) : 0.0f;
    }
    __syncthreads();
    mma_tile(Ps, Qs, ty, tx, acc);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) out[m * osm + n * osn] = alpha * acc.v[i][j];
    }
}

// out[m,n] = sum over k of act[m,k] * w_hat(k,n) + s * sum_j aux[m,j] * L(n,j)
//   DX == false (forward):  K = I, N = O, w_hat(k,n) = W[n, k], L(n,j) = B[n, j]
//   DX == true  (input grad): K = O, N = I, w_hat(k,n) = W[k, n], L(n,j) = A[j, n]
template <typename T, bool DX>
__global__ void __launch_bounds__(NT) qlinear_simt_kernel(WView w, int64_t M, const T* __restrict__ act,
                                                          const float* __restrict__ aux,
                                                          const float* __restrict__ lora, int32_t r,
                                                          float s, T* __restrict__ out) {
  __shared__ __align__(16) float Ps[BK][BM + 4];
  __shared__ __align__(16) float Qs[BK][BN + 4];
  const int64_t K = DX ? w.O : w.I;
  const int64_t N = DX ? w.I : w.O;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int64_t m0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
  Acc acc = {};
  for (int64_t k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int q = 0; q < (BM * BK) / NT; ++q) {
      const int e = tid + NT * q;
      const int mm = e / BK, kk = e % BK;
      const int64_t m = m0 + mm, k = k0 + kk;
      Ps[kk][mm] = (m < M && k < K) ? to_f32<T>(act[m * K + k]) : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < (BN * BK) / NT; ++q) {
      const int e = tid + NT * q;
      int nn, kk;
      if (DX) { nn = e % BN; kk = e / BN; } else { nn = e / BK; kk = e % BK; }
      const int64_t n = n0 + nn, k = k0 + kk;
      float v = 0.0f;
      if (n < N && k < K) v = decode_weight(w, DX ? (k * w.I + n) : (n * w.I + k));
      Qs[kk][nn] = v;
    }
    __syncthreads();
    mma_tile(Ps, Qs, ty, tx, acc);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float ad = 0.0f;
      for (int q = 0; q < r; ++q) {
        const float l = DX ? lora[(int64_t)q * w.I + n] : lora[n * r + q];
        ad = fmaf(aux[m * r + q], l, ad);
      }
      out[m * N + n] = from_f32<T>(acc.v[i][j] + s * ad);
    }
  }
}

// dst[m, j] = bf16(mul * src[m, j]) for j < r, 0 for r <= j < 64.
__global__ void pad_rows_bf16_kernel(const float* __restrict__ src, int64_t rows, int32_t r,
                                     float mul, uint16_t* __restrict__ dst) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= rows * 64) return;
  const int64_t m = e >> 6;
  const int j = (int)(e & 63);
  const float v = j < r ? __fmul_rn(mul, src[m * r + j]) : 0.0f;
  dst[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// dst[j, n] = bf16(mul * src[j, n]) for j < r, 0 for r <= j < 64.
__global__ void pad_cols_bf16_kernel(const float* __restrict__ src, int32_t r, int64_t cols,
                                     float mul, uint16_t* __restrict__ dst) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 64 * cols) return;
  const int64_t j = e / cols;
  const float v = j < r ? __fmul_rn(mul, src[e]) : 0.0f;
  dst[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// out[m, n] = sum over splits (in order) of part[s][m][n].
template <typename TO>
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int32_t splits, int64_t MN,
                                     float scale, TO* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= MN) return;
  float acc = 0.0f;
  for (int sidx = 0; sidx < splits; ++sidx) acc += part[(int64_t)sidx * MN + e];
  out[e] = from_f32<TO>(scale * acc);
}

inline unsigned cdiv(int64_t a, int64_t b) { return (unsigned)((a + b - 1) / b); }

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

cudaError_t launch_simt_fwd(const WView& w, const void* X, int64_t R, const float* A,
                            const float* B, int32_t r, float s, bool bf16, void* Y, float* U,
                            cudaStream_t st) {
  if (R == 0) return cudaSuccess;
  cudaError_t e = launch_rowdot(X, bf16, R, w.I, A, false, r, U, st);
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(w.O, BN), cdiv(R, BM));
  if (bf16)
    qlinear_simt_kernel<__nv_bfloat16, false><<<grid, NT, 0, st>>>(
        w, R, (const __nv_bfloat16*)X, U, B, r, s, (__nv_bfloat16*)Y);
  else
    qlinear_simt_kernel<float, false><<<grid, NT, 0, st>>>(w, R, (const float*)X, U, B, r, s,
                                                           (float*)Y);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_simt_dx(const WView& w, const void* dY, int64_t R, const float* A,
                           const float* V, int32_t r, float s, bool bf16, void* dX,
                           cudaStream_t st) {
  if (R == 0) return cudaSuccess;
  dim3 grid(cdiv(w.I, BN), cdiv(R, BM));
  if (bf16)
    qlinear_simt_kernel<__nv_bfloat16, true><<<grid, NT, 0, st>>>(
        w, R, (const __nv_bfloat16*)dY, V, A, r, s, (__nv_bfloat16*)dX);
  else
    qlinear_simt_kernel<float, true><<<grid, NT, 0, st>>>(w, R, (const float*)dY, V, A, r, s,
                                                          (float*)dX);
  count_launch();
  return cudaGetLastError();
}

// out[m, j] = sum_k P[m, k] * L(k, j); L(k, j) = L[k*r + j] if l_is_kr else L[j*K + k].
cudaError_t launch_rowdot(const void* P, bool bf16, int64_t R, int64_t K, const float* L,
                          bool l_is_kr, int32_t r, float* out, cudaStream_t st) {
  if (R == 0) return cudaSuccess;
  dim3 grid(cdiv(r, BN), cdiv(R, BM), 1);
  const int64_t qsk = l_is_kr ? r : 1, qsn = l_is_kr ? 1 : K;
  if (bf16)
    gemm_simt_kernel<__nv_bfloat16, float><<<grid, NT, 0, st>>>(
        R, r, K, (const __nv_bfloat16*)P, K, 1, L, qsk, qsn, 1.0f, out, r, 1, K, 0);
  else
    gemm_simt_kernel<float, float><<<grid, NT, 0, st>>>(R, r, K, (const float*)P, K, 1, L, qsk,
                                                        qsn, 1.0f, out, r, 1, K, 0);
  count_launch();
  return cudaGetLastError();
}

// Split count for the reductions over R: enough blocks for ~2 waves.
static int coldot_splits(int64_t R, int64_t N, int32_t r) {
  const int64_t tiles = (int64_t)cdiv(N, BN) * (int64_t)cdiv(r, BM);
  int64_t splits = (2 * (int64_t)num_sms() + tiles - 1) / tiles;
  const int64_t max_splits = (R + 255) / 256;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  return (int)splits;
}

size_t coldot_ws(int64_t R, int64_t N, int32_t r) {
  const int splits = coldot_splits(R, N, r);
  return splits > 1 ? align_up((size_t)splits * (size_t)N * (size_t)r * 4, 256) : 0;
}

// Reduction over R:  out = s * aux^T P, i.e. out(j, n) = s * sum_m aux[m, j] * P[m, n].
// out_nr == false: out is [r x N] (dA);  true: out is [N x r] (dB).
cudaError_t launch_coldot(const void* P, bool bf16, int64_t R, int64_t N, const float* aux,
                          int32_t r, float s, bool out_nr, float* out, void* ws,
                          cudaStream_t st) {
  const int splits = coldot_splits(R, N, r);
  const int64_t kchunk = splits > 1 ? ((R + splits - 1) / splits + BK - 1) / BK * BK : R;
  const int nsplit = splits > 1 ? (int)((R + kchunk - 1) / kchunk) : 1;
  float* dst = nsplit > 1 ? (float*)ws : out;
  const int64_t osm = out_nr ? 1 : N, osn = out_nr ? r : 1;
  dim3 grid(cdiv(N, BN), cdiv(r, BM), nsplit);
  const float alpha = nsplit > 1 ? 1.0f : s;
  const int64_t stride = (int64_t)N * r;
  // P(m = j, k = row) = aux[row * r + j];  Q(k = row, n) = P[row * N + n]
  if (bf16)
    gemm_simt_kernel<float, __nv_bfloat16><<<grid, NT, 0, st>>>(
        r, N, R, aux, 1, r, (const __nv_bfloat16*)P, N, 1, alpha, dst, osm, osn,
        R == 0 ? 1 : kchunk, stride);
  else
    gemm_simt_kernel<float, float><<<grid, NT, 0, st>>>(r, N, R, aux, 1, r, (const float*)P, N,
                                                        1, alpha, dst, osm, osn,
                                                        R == 0 ? 1 : kchunk, stride);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || nsplit == 1) return e;
  // sequential sum over the splits, then the scale s
  return launch_splitk_reduce(dst, nsplit, 1, stride, false, out, st, s);
}

cudaError_t launch_pad_rows_bf16(const float* src, int64_t rows, int32_t r, float mul,
                                 uint16_t* dst, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  pad_rows_bf16_kernel<<<cdiv(rows * 64, 256), 256, 0, st>>>(src, rows, r, mul, dst);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_pad_cols_bf16(const float* src, int32_t r, int64_t cols, float mul,
                                 uint16_t* dst, cudaStream_t st) {
  if (cols == 0) return cudaSuccess;
  pad_cols_bf16_kernel<<<cdiv(64 * cols, 256), 256, 0, st>>>(src, r, cols, mul, dst);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_splitk_reduce(const float* part, int32_t splits, int64_t R, int64_t N,
                                 bool bf16_out, void* out, cudaStream_t st, float scale) {
  const int64_t MN = R * N;
  if (MN == 0) return cudaSuccess;
  if (bf16_out)
    splitk_reduce_kernel<__nv_bfloat16><<<cdiv(MN, 256), 256, 0, st>>>(part, splits, MN, scale,
                                                                        (__nv_bfloat16*)out);
  else
    splitk_reduce_kernel<float><<<cdiv(MN, 256), 256, 0, st>>>(part, splits, MN, scale, (float*)out);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
