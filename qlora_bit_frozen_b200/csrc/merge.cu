// merge.cu -- export of a trained layer as an ordinary fp32 matrix:
//   W_merged[o, i] = W_hat[o, i] + s * sum_k B[o, k] A[k, i],   s = alpha / r
// ("QLoRA Fine-Tuning", "Training lifecycle": at export every packed weight
// is dequantized and its trained LoRA delta added, restoring the fp32
// parameter schema).  Never part of a training step.
//
// One CTA per 64 x 64 tile of the output.  The rank-r delta is a rank-r
// outer product: the CTA stages A[k0.., tile columns] and B[tile rows, k0..]
// in shared memory, 32 ranks at a time, and each thread accumulates a 4 x 4
// block of the tile with fp32 FMAs in rank order.  The epilogue decodes the
// weight of each element exactly as qlora_dequantize does (levels read from
// a shared-memory copy of the NF4 table) and adds the
// scaled delta with one rounding each (__fmul_rn, __fadd_rn), so with B = 0
// or alpha = 0 the result equals the dequantized weight.  Written with
// float4 stores when every row starts on a 16-byte boundary; the bound is
// the 4 bytes per element written (plus 0.5-1 byte of codes read).
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kRows = 64;      // output rows per CTA
constexpr int kCols = 64;      // output columns per CTA
constexpr int kRank = 32;      // ranks staged per pass
constexpr int kThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each

struct MergeArgs {
  WView w;
  const float* A;  // [r x I]
  const float* B;  // [O x r]
  int32_t r;
  float s;
  float* out;  // [O x I]
  int64_t col_tiles;
};

// Index arithmetic in 32 bits when every flat index fits (NARROW).
template <bool NARROW>
__device__ __forceinline__ uint64_t idiv(uint64_t a, uint32_t d) {
  if (NARROW) return (uint64_t)((uint32_t)a / d);
  return a / d;
}

// Weight at flat index n (same arithmetic as the diagnostic dequantization).
// lut: the 16 NF4 levels in shared memory (lanes that look up different
// levels read different banks; the constant cache would serialize them).
template <bool NARROW>
__device__ __forceinline__ float weight1(const WView& w, uint64_t n, const float* lut) {
  if (w.fmt != QLORA_FMT_AFFINE) {
    const uint32_t byte = __ldg(w.codes + (n >> 1));
    const uint32_t code = (n & 1) ? (byte >> 4) : (byte & 15u);
    const uint64_t b = idiv<NARROW>(n, (uint32_t)w.block);
    float sb;
    if (w.fmt == QLORA_FMT_NF4_FP32SCALE) {
      sb = __ldg(w.scale + b);
    } else {
      const uint64_t g = idiv<NARROW>(b, (uint32_t)w.group);
      sb = decode_block_scale(__ldg(w.qcodes + b), __ldg(w.t + g), __ldg(w.mu));
    }
    return __fmul_rn(lut[code], sb);
  }
  uint32_t q;
  if (w.bits == 8) {
    q = __ldg(w.codes + n);
  } else {
    const uint32_t byte = __ldg(w.codes + (n >> 1));
    q = (n & 1) ? (byte >> 4) : (byte & 15u);
  }
  const uint64_t g = idiv<NARROW>(n, (uint32_t)w.block);
  return __fadd_rn(__fmul_rn(__ldg(w.scale + g), (float)q), __ldg(w.bias + g));
}

// Four consecutive weights n0..n0+3 with n0 % 4 == 0 and block % 4 == 0:
// one block (group), one scale decode.
template <bool NARROW>
__device__ __forceinline__ void weight4(const WView& w, uint64_t n0, const float* lut, float v[4]) {
  if (w.fmt != QLORA_FMT_AFFINE) {
    const uint64_t b = idiv<NARROW>(n0, (uint32_t)w.block);
    float sb;
    if (w.fmt == QLORA_FMT_NF4_FP32SCALE) {
      sb = __ldg(w.scale + b);
    } else {
      const uint64_t g = idiv<NARROW>(b, (uint32_t)w.group);
      sb = decode_block_scale(__ldg(w.qcodes + b), __ldg(w.t + g), __ldg(w.mu));
    }
    const uint32_t lo = __ldg(w.codes + (n0 >> 1));
    const uint32_t hi = __ldg(w.codes + (n0 >> 1) + 1);
    v[0] = __fmul_rn(lut[lo & 15u], sb);
    v[1] = __fmul_rn(lut[lo >> 4], sb);
    v[2] = __fmul_rn(lut[hi & 15u], sb);
    v[3] = __fmul_rn(lut[hi >> 4], sb);
    return;
  }
  const uint64_t g = idiv<NARROW>(n0, (uint32_t)w.block);
  const float sc = __ldg(w.scale + g), bi = __ldg(w.bias + g);
  uint32_t q[4];
  if (w.bits == 8) {
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = __ldg(w.codes + n0 + j);
  } else {
    const uint32_t lo = __ldg(w.codes + (n0 >> 1));
    const uint32_t hi = __ldg(w.codes + (n0 >> 1) + 1);
    q[0] = lo & 15u;
    q[1] = lo >> 4;
    q[2] = hi & 15u;
    q[3] = hi >> 4;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = __fadd_rn(__fmul_rn(sc, (float)q[j]), bi);
}

// VEC: I % 4 == 0, block % 4 == 0 and out 16-byte aligned.
template <bool NARROW, bool VEC>
__global__ void __launch_bounds__(kThreads) merge_kernel(MergeArgs a) {
  __shared__ __align__(16) float As[kRank][kCols];  // A[k0 + k, i0 + c]
  __shared__ float Bs[kRank][kRows + 1];            // B[o0 + row, k0 + k]
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = kNF4[threadIdx.x];  // visible after the first barrier (r >= 1)
  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int64_t O = a.w.O, I = a.w.I;
  const int64_t o0 = ((int64_t)blockIdx.x / a.col_tiles) * kRows;
  const int64_t i0 = ((int64_t)blockIdx.x % a.col_tiles) * kCols;

  float acc[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[q][j] = 0.0f;

  for (int k0 = 0; k0 < a.r; k0 += kRank) {
    const int kc = min(kRank, a.r - k0);
    for (int e = threadIdx.x; e < kRank * kCols; e += kThreads) {
      const int k = e / kCols, c = e % kCols;
      const int64_t i = i0 + c;
      As[k][c] = (k < kc && i < I) ? __ldg(a.A + (int64_t)(k0 + k) * I + i) : 0.0f;
    }
    for (int e = threadIdx.x; e < kRank * kRows; e += kThreads) {
      const int row = e / kRank, k = e % kRank;
      const int64_t o = o0 + row;
      Bs[k][row] = (k < kc && o < O) ? __ldg(a.B + o * a.r + k0 + k) : 0.0f;
    }
    __syncthreads();
    for (int k = 0; k < kc; ++k) {
      const float4 av = *reinterpret_cast<const float4*>(&As[k][4 * tx]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float bv = Bs[k][ty + 16 * q];
        acc[q][0] = fmaf(bv, av.x, acc[q][0]);
        acc[q][1] = fmaf(bv, av.y, acc[q][1]);
        acc[q][2] = fmaf(bv, av.z, acc[q][2]);
        acc[q][3] = fmaf(bv, av.w, acc[q][3]);
      }
    }
    __syncthreads();
  }

  const int64_t ib = i0 + 4 * tx;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t o = o0 + ty + 16 * q;
    if (o >= O || ib >= I) continue;
    const uint64_t n0 = (uint64_t)o * (uint64_t)I + (uint64_t)ib;
    if (VEC) {  // I % 4 == 0: ib < I implies ib + 3 < I
      float v[4];
      weight4<NARROW>(a.w, n0, lut, v);
      float4 res;
      res.x = __fadd_rn(v[0], __fmul_rn(a.s, acc[q][0]));
      res.y = __fadd_rn(v[1], __fmul_rn(a.s, acc[q][1]));
      res.z = __fadd_rn(v[2], __fmul_rn(a.s, acc[q][2]));
      res.w = __fadd_rn(v[3], __fmul_rn(a.s, acc[q][3]));
      *reinterpret_cast<float4*>(a.out + n0) = res;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (ib + j < I)
          a.out[n0 + j] = __fadd_rn(weight1<NARROW>(a.w, n0 + j, lut), __fmul_rn(a.s, acc[q][j]));
      }
    }
  }
}

}  // namespace

cudaError_t launch_merge(const WView& w, const float* A, const float* B, int32_t r, float s,
                         float* out, cudaStream_t st) {
  const int64_t N = w.O * w.I;
  if (N == 0) return cudaSuccess;
  MergeArgs a;
  a.w = w;
  a.A = A;
  a.B = B;
  a.r = r;
  a.s = s;
  a.out = out;
  a.col_tiles = (w.I + kCols - 1) / kCols;
  const int64_t tiles = ((w.O + kRows - 1) / kRows) * a.col_tiles;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const bool narrow = N <= 0xffffffffLL;
  const bool vec = (w.I % 4 == 0) && (w.block % 4 == 0) && ((uintptr_t)out % 16 == 0);
  const dim3 grid((unsigned)tiles);
  if (narrow && vec) merge_kernel<true, true><<<grid, kThreads, 0, st>>>(a);
  else if (narrow) merge_kernel<true, false><<<grid, kThreads, 0, st>>>(a);
  else if (vec) merge_kernel<false, true><<<grid, kThreads, 0, st>>>(a);
  else merge_kernel<false, false><<<grid, kThreads, 0, st>>>(a);
  count_launch(1);
  return cudaGetLastError();
}

}  // namespace qlora
