// quantize.cu -- NF4 quantizers (double-quantized and legacy fp32 scales),
// the affine quantizer, diagnostic dequantize.
//
// "QLoRA Fine-Tuning" (Riftco Transformer how-to), section "NF4
// representation": blockwise absmax s_b, nearest of the 16 NF4 levels to
// w / s_b, low nibble first, all-zero block -> scale 0 and the zero level,
// mean mu of the block scales, per-group absmax t_g of s_b - mu, centred
// byte codes q_b.  "LoRA vs QLoRA on Apple Silicon", "Method": affine
// group-wise codes with fp32 scale and bias (plain min/max scheme).
//
// Every fp32 step is one IEEE round-to-nearest operation (__fdiv_rn,
// __fsub_rn, __fmul_rn; the translation unit is built without fast math and
// without FMA contraction), so codes, scale codes, t_g, mu and the
// dequantized values are bit-exact and deterministic.
#include "common.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int kThreads = 256;

// s_b = max |w| over block b.  One warp per block; any NaN/Inf raises the
// non-finite flag (header word 2).
__global__ void nf4_absmax_kernel(const float* __restrict__ W, int64_t N, int32_t B, int64_t M,
                                  float* __restrict__ s, uint32_t* __restrict__ hdr) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= M) return;
  const int64_t lo = warp * B;
  const int64_t hi = lo + B < N ? lo + B : N;
  float m = 0.0f;
  bool bad = false;
  for (int64_t i = lo + lane; i < hi; i += 32) {
    float v = W[i];
    bad |= !isfinite(v);
    m = fmaxf(m, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(hdr + 2, 1u);
  if (lane == 0) s[warp] = m;
}

__device__ __forceinline__ uint32_t nf4_encode(float w, float sb) {
  if (sb == 0.0f) return 7u;  // the exact-zero level
  const double x = (double)__fdiv_rn(w, sb);
  uint32_t code = 0;
#pragma unroll
  for (int k = 0; k < 15; ++k) code += (x > nf4_mid(k)) ? 1u : 0u;  // ties -> lower level
  return code;
}

// One thread per packed byte: weights 2j (low nibble) and 2j+1 (high).
__global__ void nf4_encode_kernel(const float* __restrict__ W, int64_t N, int32_t B,
                                  const float* __restrict__ s, uint8_t* __restrict__ codes) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nbytes = (N + 1) >> 1;
  if (j >= nbytes) return;
  const int64_t n0 = 2 * j, n1 = 2 * j + 1;
  uint32_t c0 = nf4_encode(W[n0], s[n0 / B]);
  uint32_t c1 = 0;
  if (n1 < N) c1 = nf4_encode(W[n1], s[n1 / B]);
  codes[j] = (uint8_t)(c0 | (c1 << 4));
}

// Group partial sums of s_b in fp64, sequential inside the group.
__global__ void nf4_group_sum_kernel(const float* __restrict__ s, int64_t M, int32_t C, int64_t S,
                                     double* __restrict__ part) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= S) return;
  const int64_t lo = g * C, hi = lo + C < M ? lo + C : M;
  double acc = 0.0;
  for (int64_t b = lo; b < hi; ++b) acc += (double)s[b];
  part[g] = acc;
}

// mu = (sum of the group partials, sequential in group order) / M.  One
// block stages the partials through shared memory; thread 0 adds them in
// order.
__global__ void nf4_mean_kernel(const double* __restrict__ part, int64_t S, int64_t M,
                                float* __restrict__ mu) {
  __shared__ double buf[1024];
  double total = 0.0;
  for (int64_t base = 0; base < S; base += 1024) {
    const int64_t n = S - base < 1024 ? S - base : 1024;
    __syncthreads();
    if (threadIdx.x < n) buf[threadIdx.x] = part[base + threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0)
      for (int64_t k = 0; k < n; ++k) total += buf[k];
  }
  if (threadIdx.x == 0) *mu = (M > 0) ? (float)(total / (double)M) : 0.0f;
}

// t_g = max |fp32(s_b - mu)| over the group, then the centred byte codes.
// One warp per group.
__global__ void nf4_dq_kernel(const float* __restrict__ s, int64_t M, int32_t C, int64_t S,
                              const float* __restrict__ mu_p, float* __restrict__ t,
                              uint8_t* __restrict__ q) {
  const int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (g >= S) return;
  const float mu = *mu_p;
  const int64_t lo = g * C, hi = lo + C < M ? lo + C : M;
  float tg = 0.0f;
  for (int64_t b = lo + lane; b < hi; b += 32) tg = fmaxf(tg, fabsf(__fsub_rn(s[b], mu)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tg = fmaxf(tg, __shfl_xor_sync(0xffffffffu, tg, o));
  if (lane == 0) t[g] = tg;
  for (int64_t b = lo + lane; b < hi; b += 32) {
    uint32_t code = 128u;  // zero range
    if (tg != 0.0f) {
      const float d = __fsub_rn(s[b], mu);
      const float v = __fdiv_rn(__fmul_rn(127.0f, d), tg);
      float rv = roundf(v);  // half away from zero
      rv = fminf(fmaxf(rv, -127.0f), 127.0f);
      code = (uint32_t)(128 + (int)rv);
    }
    q[b] = (uint8_t)code;
  }
}

// Affine: per group min, max, scale, bias.  One warp per group.
__global__ void affine_range_kernel(const float* __restrict__ W, int64_t N, int32_t G, int64_t ng,
                                    float levels, float* __restrict__ scale,
                                    float* __restrict__ bias, uint32_t* __restrict__ hdr) {
  const int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (g >= ng) return;
  const int64_t lo = g * G, hi = lo + G < N ? lo + G : N;
  float mn = W[lo], mx = W[lo];
  bool bad = false;
  for (int64_t i = lo + lane; i < hi; i += 32) {
    float v = W[i];
    bad |= !isfinite(v);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float sc = __fdiv_rn(__fsub_rn(mx, mn), levels);
  bad |= !isfinite(sc);
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(hdr + 2, 1u);
  if (lane == 0) {
    scale[g] = sc;
    bias[g] = mn;
  }
}

__device__ __forceinline__ uint32_t affine_encode(float w, float sc, float b, float levels) {
  if (sc == 0.0f) return 0u;
  float v = __fdiv_rn(__fsub_rn(w, b), sc);
  float rv = roundf(v);
  rv = fminf(fmaxf(rv, 0.0f), levels);
  return (uint32_t)rv;
}

// One thread per output byte (4-bit: two weights; 8-bit: one weight).
__global__ void affine_encode_kernel(const float* __restrict__ W, int64_t N, int32_t bits,
                                     int32_t G, float levels, const float* __restrict__ scale,
                                     const float* __restrict__ bias, uint8_t* __restrict__ codes) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (bits == 8) {
    if (j >= N) return;
    const int64_t g = j / G;
    codes[j] = (uint8_t)affine_encode(W[j], scale[g], bias[g], levels);
  } else {
    const int64_t nbytes = (N + 1) >> 1;
    if (j >= nbytes) return;
    const int64_t n0 = 2 * j, n1 = 2 * j + 1;
    uint32_t c0 = affine_encode(W[n0], scale[n0 / G], bias[n0 / G], levels);
    uint32_t c1 = 0;
    if (n1 < N) c1 = affine_encode(W[n1], scale[n1 / G], bias[n1 / G], levels);
    codes[j] = (uint8_t)(c0 | (c1 << 4));
  }
}

// Diagnostic dequantization, one element per thread.
__global__ void dequantize_kernel(WView w, float* __restrict__ out, int64_t N) {
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n < N) out[n] = decode_weight(w, n);
}

inline unsigned grid_for(int64_t items, int per_block) {
  return (unsigned)((items + per_block - 1) / per_block);
}

}  // namespace

size_t nf4_quantize_ws(int64_t N, int32_t B, int32_t C) {
  const int64_t M = (N + B - 1) / B;
  const int64_t S = (M + C - 1) / C;
  return kWsHeader + align_up((size_t)M * 4, 256) + align_up((size_t)S * 8, 256);
}

cudaError_t launch_nf4_quantize(const float* W, int64_t N, int32_t B, int32_t C, uint8_t* codes,
                                uint8_t* qcodes, float* t, float* mu, void* ws, cudaStream_t st) {
  const int64_t M = (N + B - 1) / B;
  const int64_t S = (M + C - 1) / C;
  uint32_t* hdr = (uint32_t*)ws;
  float* s = (float*)((char*)ws + kWsHeader);
  double* part = (double*)((char*)ws + kWsHeader + align_up((size_t)M * 4, 256));
  cudaError_t e = cudaMemsetAsync(ws, 0, kWsHeader, st);
  if (e != cudaSuccess) return e;
  if (M > 0) {
    nf4_absmax_kernel<<<grid_for(M * 32, kThreads), kThreads, 0, st>>>(W, N, B, M, s, hdr);
    nf4_encode_kernel<<<grid_for((N + 1) / 2, kThreads), kThreads, 0, st>>>(W, N, B, s, codes);
    nf4_group_sum_kernel<<<grid_for(S, kThreads), kThreads, 0, st>>>(s, M, C, S, part);
    count_launch(3);
  }
  nf4_mean_kernel<<<1, 1024, 0, st>>>(part, S, M, mu);
  count_launch(1);
  if (S > 0) {
    nf4_dq_kernel<<<grid_for(S * 32, kThreads), kThreads, 0, st>>>(s, M, C, S, mu, t, qcodes);
    count_launch(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_nf4_fp32scale_quantize(const float* W, int64_t N, int32_t B, uint8_t* codes,
                                          float* scale, void* ws, cudaStream_t st) {
  const int64_t M = (N + B - 1) / B;
  uint32_t* hdr = (uint32_t*)ws;
  cudaError_t e = cudaMemsetAsync(ws, 0, kWsHeader, st);
  if (e != cudaSuccess) return e;
  if (M > 0) {
    // the absmax is the stored scale itself; codes as in the double-quantized format
    nf4_absmax_kernel<<<grid_for(M * 32, kThreads), kThreads, 0, st>>>(W, N, B, M, scale, hdr);
    nf4_encode_kernel<<<grid_for((N + 1) / 2, kThreads), kThreads, 0, st>>>(W, N, B, scale, codes);
    count_launch(2);
  }
  return cudaGetLastError();
}

cudaError_t launch_affine_quantize(const float* W, int64_t N, int32_t bits, int32_t G,
                                   uint8_t* codes, float* scale, float* bias, void* ws,
                                   cudaStream_t st) {
  const int64_t ng = (N + G - 1) / G;
  const float levels = (float)((1 << bits) - 1);
  uint32_t* hdr = (uint32_t*)ws;
  cudaError_t e = cudaMemsetAsync(ws, 0, kWsHeader, st);
  if (e != cudaSuccess) return e;
  if (ng > 0) {
    affine_range_kernel<<<grid_for(ng * 32, kThreads), kThreads, 0, st>>>(W, N, G, ng, levels,
                                                                           scale, bias, hdr);
    const int64_t items = bits == 8 ? N : (N + 1) / 2;
    affine_encode_kernel<<<grid_for(items, kThreads), kThreads, 0, st>>>(W, N, bits, G, levels,
                                                                         scale, bias, codes);
    count_launch(2);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const WView& w, float* out, cudaStream_t st) {
  const int64_t N = w.O * w.I;
  if (N == 0) return cudaSuccess;
  dequantize_kernel<<<grid_for(N, kThreads), kThreads, 0, st>>>(w, out, N);
  count_launch(1);
  return cudaGetLastError();
}

}  // namespace qlora
