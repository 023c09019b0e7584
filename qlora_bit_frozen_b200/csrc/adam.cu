// adam.cu -- the adapter optimizer step ("QLoRA Fine-Tuning", "Training
// lifecycle": only the fp32 LoRA factors are trained, with Adam; "Current
// scope": paged Adam state, split into pages of at most page_size elements
// that are updated one page at a time).  The pages name Adam without a rule;
// this is Adam with bias correction:
//   m' = b1 m + (1 - b1) g
//   v' = b2 v + (1 - b2) g^2
//   p' = p - lr (m' / bc1) / (sqrt(v' / bc2) + eps),   bc = 1 - b^t
// over one flat fp32 arena (the caller keeps every adapter factor of the
// model in it, so one launch updates them all).  Each fp32 step is one
// rounding (__fmul_rn / __fadd_rn / __fdiv_rn / __fsqrt_rn), so the result
// does not depend on the launch split: a paged call gives the same bits as
// a single launch.  Streaming, 28 bytes per parameter (4 read, 3 written).
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;

struct AdamCoef {
  float lr, b1, b2, omb1, omb2, bc1, bc2, eps;
};

__global__ void __launch_bounds__(kThreads)
    adam_kernel(float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m,
                float* __restrict__ v, int64_t begin, int64_t end, AdamCoef c) {
  const int64_t j = begin + (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (j >= end) return;
  const float gj = g[j];
  const float mj = __fadd_rn(__fmul_rn(c.b1, m[j]), __fmul_rn(c.omb1, gj));
  const float vj = __fadd_rn(__fmul_rn(c.b2, v[j]), __fmul_rn(c.omb2, __fmul_rn(gj, gj)));
  const float mhat = __fdiv_rn(mj, c.bc1);
  const float vhat = __fdiv_rn(vj, c.bc2);
  const float den = __fadd_rn(__fsqrt_rn(vhat), c.eps);
  const float step = __fdiv_rn(__fmul_rn(c.lr, mhat), den);
  p[j] = __fsub_rn(p[j], step);
  m[j] = mj;
  v[j] = vj;
}

}  // namespace

cudaError_t launch_adam(float* p, const float* g, float* m, float* v, int64_t n, int64_t t,
                        float lr, float beta1, float beta2, float eps, int64_t page,
                        cudaStream_t st) {
  AdamCoef c;
  c.lr = lr;
  c.b1 = beta1;
  c.b2 = beta2;
  c.omb1 = (float)(1.0 - (double)beta1);
  c.omb2 = (float)(1.0 - (double)beta2);
  c.bc1 = (float)(1.0 - pow((double)beta1, (double)t));
  c.bc2 = (float)(1.0 - pow((double)beta2, (double)t));
  c.eps = eps;
  const int64_t span = page > 0 ? page : n;
  for (int64_t b = 0; b < n; b += span) {
    const int64_t e = b + span < n ? b + span : n;
    const int64_t blocks = (e - b + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    adam_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(p, g, m, v, b, e, c);
    count_launch(1);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace qlora
