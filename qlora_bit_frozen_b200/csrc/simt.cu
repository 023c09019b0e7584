// simt.cu -- CUDA-core kernels of the QLoRA linear layer.
//
//  * qlinear_simt: the base GEMM with the weight decoded per element from its
//    nibble and block scale inside the K loop ("QLoRA Fine-Tuning", "Forward
//    and backward": decode each nibble inside the sums), fp32 accumulation,
//    plus the adapter term s * Aux * L^T in the epilogue.  Serves the fp32
//    compute mode (true fp32 FFMA; TF32 tensor cores cannot meet a 1e-5
//    relative error) and shapes the tensor-core path does not take.
//  * staging kernels that build the zero-padded bf16 adapter operands the
//    tensor-core kernels consume, and the split-K reduction.
#include "common.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

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

template <typename TO>
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int32_t splits, int64_t MN,
                                     float scale, TO* __restrict__ out) {
  griddep_wait();  // the partials come from the launch just before
  const int64_t e4 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e4 >= MN) return;
  if ((MN & 3) == 0) {
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int sidx = 0; sidx < splits; ++sidx) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(part + (int64_t)sidx * MN + e4));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    out[e4] = from_f32<TO>(scale * acc.x);
    out[e4 + 1] = from_f32<TO>(scale * acc.y);
    out[e4 + 2] = from_f32<TO>(scale * acc.z);
    out[e4 + 3] = from_f32<TO>(scale * acc.w);
    return;
  }
  for (int64_t e = e4; e < e4 + 4 && e < MN; ++e) {
    float acc = 0.0f;
    for (int sidx = 0; sidx < splits; ++sidx) acc += part[(int64_t)sidx * MN + e];
    out[e] = from_f32<TO>(scale * acc);
  }
}

inline unsigned cdiv(int64_t a, int64_t b) { return (unsigned)((a + b - 1) / b); }

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

cudaError_t launch_splitk_reduce(const float* part, int32_t splits, int64_t R, int64_t N,
                                 bool bf16_out, void* out, cudaStream_t st, float scale, bool pdl) {
  const int64_t MN = R * N;
  if (MN == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cdiv(MN, 1024));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e;
  if (bf16_out)
    e = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<__nv_bfloat16>, part, splits, MN, scale,
                           (__nv_bfloat16*)out);
  else
    e = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<float>, part, splits, MN, scale, (float*)out);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace qlora
