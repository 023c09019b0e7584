// simt.cu -- CUDA-core kernels of the QLoRA linear layer.
//
//  * qlinear_simt: the base GEMM with the weight decoded per element from its
//    nibble and block scale inside the K loop ("QLoRA Fine-Tuning", "Forward
//    and backward": decode each nibble inside the sums), fp32 accumulation,
//    plus the adapter term s * Aux * L^T in the epilogue.  Serves the fp32
//    compute mode (true fp32 FFMA; TF32 tensor cores cannot meet a 1e-5
//    relative error) and shapes the tensor-core path does not take.
//  * gemv: affine weights at up to 16 tokens ("LoRA vs QLoRA on Apple
//    Silicon", "Method": the bandwidth-bound sweep), where the GEMM is a few
//    dot products per weight row: stream the codes once, decode in
//    registers, accumulate on the CUDA cores.
//  * the split-K reduction of the tensor-core path.
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

namespace {

// ------------------------------------------------------------------ gemv

constexpr int kGemvKC = 256;            // K columns staged per chunk (8 per lane)
constexpr int kGemvWR = 4;              // weight rows per warp
constexpr int kGemvRows = 8 * kGemvWR;  // weight rows per block
// dX: each thread owns kDxCP(RM) adjacent columns (8 up to 4 tokens, 4
// above, to bound the RM x CP accumulators)
constexpr int dx_cp(int rm) { return rm <= 4 ? 8 : 4; }
constexpr int kDxChunk = 256;           // W rows of dY staged per chunk

// Affine weights are scale_g * q + bias_g, one rounding each (the same
// arithmetic as decode_weight).
// 4 consecutive affine weights from flat index n (n % 4 == 0; the group size
// is a multiple of 8, so they share one scale and bias): one code load.
__device__ __forceinline__ void affine_decode4(const WView& w, int64_t n, float (&v)[4]) {
  const int64_t g = n / w.block;
  const float sc = __ldg(w.scale + g), bi = __ldg(w.bias + g);
  uint32_t q[4];
  if (w.bits == 8) {
    const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(w.codes + n));
#pragma unroll
    for (int e = 0; e < 4; ++e) q[e] = (b >> (8 * e)) & 255u;
  } else {
    const uint32_t b = __ldg(reinterpret_cast<const unsigned short*>(w.codes + (n >> 1)));
#pragma unroll
    for (int e = 0; e < 4; ++e) q[e] = (b >> (4 * e)) & 15u;  // low nibble first
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] = __fadd_rn(__fmul_rn(sc, (float)q[e]), bi);
}

// 8 consecutive affine weights from flat index n (n % 8 == 0; the group size
// is a multiple of 8, so they share one scale and bias): one code load.
__device__ __forceinline__ void affine_decode8(const WView& w, int64_t n, float (&v)[8]) {
  const int64_t g = n / w.block;
  const float sc = __ldg(w.scale + g), bi = __ldg(w.bias + g);
  uint32_t q[8];
  if (w.bits == 8) {
    const uint2 b = __ldg(reinterpret_cast<const uint2*>(w.codes + n));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      q[e] = (b.x >> (8 * e)) & 255u;
      q[e + 4] = (b.y >> (8 * e)) & 255u;
    }
  } else {
    const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(w.codes + (n >> 1)));
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = (b >> (4 * e)) & 15u;  // low nibble first
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __fadd_rn(__fmul_rn(sc, (float)q[e]), bi);
}

// Y[m, o] = sum_i X[m, i] W_hat[o, i] + s sum_j U[m, j] B[o, j], m < R <= RM.
// A warp owns kGemvWR weight rows and streams them in 256-column chunks,
// each lane decoding 8 consecutive weights per row; X is staged per chunk
// in shared memory; lane partials are combined with a butterfly.
template <typename T, int RM>
__global__ void __launch_bounds__(256) gemv_fwd_kernel(WView w, int R, const T* __restrict__ X,
                                                       const float* __restrict__ U,
                                                       const float* __restrict__ Bf, int r,
                                                       float s, T* __restrict__ Y) {
  __shared__ __align__(16) float xs[RM][kGemvKC];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t I = w.I, O = w.O;
  const int64_t o0 = (int64_t)blockIdx.x * kGemvRows + warp * kGemvWR;
  float acc[kGemvWR][RM];
#pragma unroll
  for (int q = 0; q < kGemvWR; ++q)
#pragma unroll
    for (int m = 0; m < RM; ++m) acc[q][m] = 0.0f;
  for (int64_t k0 = 0; k0 < I; k0 += kGemvKC) {
    __syncthreads();
    for (int e = threadIdx.x; e < RM * kGemvKC; e += 256) {
      const int m = e / kGemvKC, c = e % kGemvKC;
      const int64_t k = k0 + c;
      xs[m][c] = (m < R && k < I) ? to_f32<T>(X[(int64_t)m * I + k]) : 0.0f;
    }
    __syncthreads();
    const int64_t k = k0 + lane * 8;
    if (k >= I) continue;
#pragma unroll
    for (int q = 0; q < kGemvWR; ++q) {
      const int64_t o = o0 + q;
      if (o >= O) break;
      float v[8];
      affine_decode8(w, o * I + k, v);
#pragma unroll
      for (int m = 0; m < RM; ++m) {
        const float4 x0 = *reinterpret_cast<const float4*>(&xs[m][lane * 8]);
        const float4 x1 = *reinterpret_cast<const float4*>(&xs[m][lane * 8 + 4]);
        float a = acc[q][m];
        a = fmaf(v[0], x0.x, a); a = fmaf(v[1], x0.y, a); a = fmaf(v[2], x0.z, a);
        a = fmaf(v[3], x0.w, a); a = fmaf(v[4], x1.x, a); a = fmaf(v[5], x1.y, a);
        a = fmaf(v[6], x1.z, a); a = fmaf(v[7], x1.w, a);
        acc[q][m] = a;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kGemvWR; ++q)
#pragma unroll
    for (int m = 0; m < RM; ++m)
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) acc[q][m] += __shfl_xor_sync(0xffffffffu, acc[q][m], d);
#pragma unroll
  for (int q = 0; q < kGemvWR; ++q) {
    const int64_t o = o0 + q;
    if (o >= O) break;
    float tot = 0.0f;  // lane m keeps row m's sum (no dynamic register index)
#pragma unroll
    for (int m = 0; m < RM; ++m)
      if (m == lane) tot = acc[q][m];
    if (lane < R) {
      float ad = 0.0f;
      for (int j = 0; j < r; ++j) ad = fmaf(U[(int64_t)lane * r + j], Bf[o * r + j], ad);
      Y[(int64_t)lane * O + o] = from_f32<T>(tot + s * ad);
    }
  }
}

// dX partial over W rows [oa, oa + orange): part[split][m][i] =
// sum_o dY[m, o] W_hat[o, i].  Each thread owns CP adjacent columns: per W
// row one vector load of their codes and one scale / bias pair (the CP
// columns lie in one affine group), CP x RM multiply-adds; a warp reads a
// contiguous run of the row.  dY is staged per chunk in shared memory.
template <typename T, int RM>
__global__ void __launch_bounds__(256) gemv_dx_kernel(WView w, int R, const T* __restrict__ dY,
                                                      int64_t orange, float* __restrict__ part) {
  constexpr int CP = dx_cp(RM);
  __shared__ float ys[RM][kDxChunk];
  const int64_t I = w.I, O = w.O;
  const int64_t i0 = ((int64_t)blockIdx.x * 256 + threadIdx.x) * CP;
  const int64_t oa = (int64_t)blockIdx.y * orange, ob = min(O, oa + orange);
  float acc[RM][CP];
#pragma unroll
  for (int m = 0; m < RM; ++m)
#pragma unroll
    for (int e = 0; e < CP; ++e) acc[m][e] = 0.0f;
  for (int64_t c0 = oa; c0 < ob; c0 += kDxChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < RM * kDxChunk; e += 256) {
      const int m = e / kDxChunk, c = e % kDxChunk;
      const int64_t o = c0 + c;
      ys[m][c] = (m < R && o < ob) ? to_f32<T>(dY[(int64_t)m * O + o]) : 0.0f;
    }
    __syncthreads();
    if (i0 >= I) continue;
    const int nc = (int)min((int64_t)kDxChunk, ob - c0);
#pragma unroll 4
    for (int c = 0; c < nc; ++c) {
      float v[CP];
      if constexpr (CP == 8)
        affine_decode8(w, (c0 + c) * I + i0, v);
      else
        affine_decode4(w, (c0 + c) * I + i0, v);
#pragma unroll
      for (int m = 0; m < RM; ++m) {
        const float y = ys[m][c];
#pragma unroll
        for (int e = 0; e < CP; ++e) acc[m][e] = fmaf(v[e], y, acc[m][e]);
      }
    }
  }
  if (i0 >= I) return;
#pragma unroll
  for (int m = 0; m < RM; ++m)
    if (m < R) {
      float* dst = part + ((int64_t)blockIdx.y * R + m) * I + i0;
#pragma unroll
      for (int e = 0; e < CP; ++e) dst[e] = acc[m][e];
    }
}

// dX[m, i] = sum over splits (in order) + s sum_j V[m, j] A[j, i].
template <typename T>
__global__ void gemv_dx_reduce_kernel(const float* __restrict__ part, int splits, int R,
                                      int64_t I, const float* __restrict__ V,
                                      const float* __restrict__ A, int r, float s,
                                      T* __restrict__ dX) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)R * I) return;
  const int64_t m = e / I, i = e - m * I;
  float v = 0.0f;
  for (int q = 0; q < splits; ++q) v += part[((int64_t)q * R + m) * I + i];
  float ad = 0.0f;
  for (int j = 0; j < r; ++j) ad = fmaf(V[m * r + j], A[(int64_t)j * I + i], ad);
  dX[e] = from_f32<T>(v + s * ad);
}

struct DxPlan {
  int col_blocks, splits;
  int64_t orange;
};

// Columns per block: 256 threads x the columns each owns at this token count.
int dx_cols(int64_t R) { return 256 * (R <= 4 ? 8 : 4); }

// Row splits: about two CTAs per SM in all, each at least 64 W rows (a
// multiple of 64; the last chunk of a range may be partial).
DxPlan dx_plan(const WView& w, int64_t R) {
  DxPlan p;
  p.col_blocks = (int)cdiv(w.I, dx_cols(R));
  int64_t splits = (2 * 148 + p.col_blocks - 1) / p.col_blocks;
  const int64_t max_splits = cdiv(w.O, 64);
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  p.orange = (cdiv(w.O, splits) + 63) / 64 * 64;
  p.splits = (int)cdiv(w.O, p.orange);
  return p;
}

template <typename T, int RM>
void gemv_fwd_go(const WView& w, int R, const void* X, const float* U, const float* B, int r,
                 float s, void* Y, cudaStream_t st) {
  gemv_fwd_kernel<T, RM><<<cdiv(w.O, kGemvRows), 256, 0, st>>>(w, R, (const T*)X, U, B, r, s,
                                                               (T*)Y);
}

template <typename T, int RM>
void gemv_dx_go(const WView& w, int R, const void* dY, const DxPlan& p, float* part,
                cudaStream_t st) {
  dim3 grid((unsigned)p.col_blocks, (unsigned)p.splits);
  gemv_dx_kernel<T, RM><<<grid, 256, 0, st>>>(w, R, (const T*)dY, p.orange, part);
}

template <typename T>
void gemv_fwd_r(const WView& w, int R, const void* X, const float* U, const float* B, int r,
                float s, void* Y, cudaStream_t st) {
  if (R <= 1) gemv_fwd_go<T, 1>(w, R, X, U, B, r, s, Y, st);
  else if (R <= 2) gemv_fwd_go<T, 2>(w, R, X, U, B, r, s, Y, st);
  else if (R <= 4) gemv_fwd_go<T, 4>(w, R, X, U, B, r, s, Y, st);
  else if (R <= 8) gemv_fwd_go<T, 8>(w, R, X, U, B, r, s, Y, st);
  else gemv_fwd_go<T, 16>(w, R, X, U, B, r, s, Y, st);
}

template <typename T>
void gemv_dx_r(const WView& w, int R, const void* dY, const DxPlan& p, float* part,
               cudaStream_t st) {
  if (R <= 1) gemv_dx_go<T, 1>(w, R, dY, p, part, st);
  else if (R <= 2) gemv_dx_go<T, 2>(w, R, dY, p, part, st);
  else if (R <= 4) gemv_dx_go<T, 4>(w, R, dY, p, part, st);
  else if (R <= 8) gemv_dx_go<T, 8>(w, R, dY, p, part, st);
  else gemv_dx_go<T, 16>(w, R, dY, p, part, st);
}

// Affine weights at up to 16 tokens, rows of 8-aligned codes.
bool gemv_ok(const WView& w, int64_t R) {
  return w.fmt == QLORA_FMT_AFFINE && R >= 1 && R <= 16 && (w.I % 8) == 0 && (w.block % 8) == 0 &&
         ((uintptr_t)w.codes % 8) == 0;
}

}  // namespace

size_t gemv_dx_ws(const WView& w, int64_t R) {
  if (!gemv_ok(w, R)) return 0;
  return align_up((size_t)dx_plan(w, R).splits * (size_t)R * (size_t)w.I * 4, 256);
}

cudaError_t launch_simt_fwd(const WView& w, const void* X, int64_t R, const float* A,
                            const float* B, int32_t r, float s, bool bf16, void* Y, float* U,
                            cudaStream_t st) {
  if (R == 0) return cudaSuccess;
  cudaError_t e = launch_rowdot(X, bf16, R, w.I, A, false, r, U, st);
  if (e != cudaSuccess) return e;
  if (gemv_ok(w, R)) {
    if (bf16)
      gemv_fwd_r<__nv_bfloat16>(w, (int)R, X, U, B, r, s, Y, st);
    else
      gemv_fwd_r<float>(w, (int)R, X, U, B, r, s, Y, st);
    count_launch();
    return cudaGetLastError();
  }
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
                           cudaStream_t st, float* gemv_ws) {
  if (R == 0) return cudaSuccess;
  if (gemv_ws && gemv_ok(w, R)) {
    const DxPlan p = dx_plan(w, R);
    if (bf16)
      gemv_dx_r<__nv_bfloat16>(w, (int)R, dY, p, gemv_ws, st);
    else
      gemv_dx_r<float>(w, (int)R, dY, p, gemv_ws, st);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = R * w.I;
    if (bf16)
      gemv_dx_reduce_kernel<__nv_bfloat16><<<cdiv(n, 256), 256, 0, st>>>(
          gemv_ws, p.splits, (int)R, w.I, V, A, r, s, (__nv_bfloat16*)dX);
    else
      gemv_dx_reduce_kernel<float><<<cdiv(n, 256), 256, 0, st>>>(gemv_ws, p.splits, (int)R, w.I,
                                                                 V, A, r, s, (float*)dX);
    count_launch();
    return cudaGetLastError();
  }
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
