// common.cuh -- device helpers shared by the libqlora kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qlora.h"

namespace qlora {

// ---------------------------------------------------------------------------
// NF4 levels, fp32: the canonical table of the NF4 data type ("QLoRA
// Fine-Tuning", "NF4 representation": the fixed 16-value codebook matches
// the canonical bitsandbytes mapping; "QLoRA: Fine-Tuning Under Memory
// Constraints", "Understand what NF4 chooses": the levels follow a normal
// distribution).  These are the values printed for the NormalFloat 4-bit
// type in the QLoRA paper's appendix, written as exact hex floats: normal
// quantiles at single-precision probabilities spaced evenly from 0.9677083
// down to 1/2 (8 positive, 7 negative, 1/2 excluded), plus 0, divided by
// the largest.
// ---------------------------------------------------------------------------
#define QLORA_NF4_LEVELS                                                                   \
  {-0x1.000000p+0f, -0x1.647362p-1f, -0x1.0cd660p-1f, -0x1.946540p-2f, -0x1.23449ap-2f,    \
   -0x1.7a6a7ep-3f, -0x1.74f0e2p-4f, 0.0f,           0x1.45f5fep-4f,  0x1.4995c6p-3f,     \
   0x1.f809bap-3f,  0x1.5a0674p-2f,  0x1.c34970p-2f, 0x1.200f56p-1f,  0x1.722766p-1f,     \
   0x1.000000p+0f}

static __device__ __constant__ float kNF4[16] = QLORA_NF4_LEVELS;
static const float kNF4Host[16] = QLORA_NF4_LEVELS;

// Midpoints between neighbouring levels, exact in fp64.
__device__ __forceinline__ double nf4_mid(int k) {
  return 0.5 * ((double)kNF4[k] + (double)kNF4[k + 1]);
}

// ---------------------------------------------------------------------------
// Workspace header: the first 256 bytes of every workspace.
//   word 0: first error status recorded by a kernel (0 = none)
//   word 1: where (kernel-specific code)
//   word 2: non-finite flag (quantizers)
// ---------------------------------------------------------------------------
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ void report_error(uint32_t* ws_header, uint32_t status, uint32_t where) {
  if (ws_header == nullptr) return;
  if (atomicCAS(ws_header, 0u, status) == 0u) ws_header[1] = where;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// bf16 helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// Weight view passed to kernels by value.
// ---------------------------------------------------------------------------
struct WView {
  int32_t fmt;
  int64_t O, I;
  int32_t block, group, bits;
  const uint8_t* codes;
  const uint8_t* qcodes;
  const float* t;
  const float* mu;
  const float* scale;
  const float* bias;
};

// "QLoRA Fine-Tuning", "NF4 representation": decoded block scale
// clamp(mu + t_g (q_b - 128)/127, 0, FLT_MAX), one fp32 rounding per step.
__device__ __forceinline__ float decode_block_scale(uint32_t q, float t, float mu) {
  float k = (float)((int)q - 128);
  float a = __fmul_rn(t, k);
  float b = __fdiv_rn(a, 127.0f);
  float s = __fadd_rn(mu, b);
  if (s < 0.0f) s = 0.0f;
  if (s > 3.402823466e38f) s = 3.402823466e38f;
  return s;
}

// Scale of NF4 block b: the double-quantized s_hat_b, or the stored fp32
// absmax of the legacy format ("NF4 representation": legacy scale storage).
__device__ __forceinline__ float nf4_block_scale(const WView& w, int64_t b) {
  if (w.fmt == QLORA_FMT_NF4_FP32SCALE) return __ldg(w.scale + b);
  const int64_t g = b / w.group;
  return decode_block_scale(__ldg(w.qcodes + b), __ldg(w.t + g), __ldg(w.mu));
}

// w_hat at flat index n (per-element decode; used by the SIMT and
// diagnostic kernels).
__device__ __forceinline__ float decode_weight(const WView& w, int64_t n) {
  if (w.fmt != QLORA_FMT_AFFINE) {
    uint32_t byte = __ldg(w.codes + (n >> 1));
    uint32_t code = (n & 1) ? (byte >> 4) : (byte & 15u);
    return __fmul_rn(kNF4[code], nf4_block_scale(w, n / w.block));
  } else {
    uint32_t q;
    if (w.bits == 8) {
      q = __ldg(w.codes + n);
    } else {
      uint32_t byte = __ldg(w.codes + (n >> 1));
      q = (n & 1) ? (byte >> 4) : (byte & 15u);
    }
    int64_t g = n / w.block;
    return __fadd_rn(__fmul_rn(__ldg(w.scale + g), (float)q), __ldg(w.bias + g));
  }
}

// ---------------------------------------------------------------------------
// mbarrier / TMA / tcgen05 wrappers (inline PTX, sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity`.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier.  Gives up after
// `limit_ns` nanoseconds of %globaltimer, records QLORA_ERR_TIMEOUT in the
// workspace header and returns false.  Never spins without a bound.
// A phase that has already completed is seen by the cheap non-blocking
// test; try_wait (which may suspend the thread and costs a few hundred
// cycles even on a completed phase) is left for phases still pending.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          uint32_t* err, uint32_t where) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  // Two bounds: elapsed %globaltimer time, and (should the timer not
  // advance) a hard iteration cap.
  for (uint32_t it = 0; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 15u && globaltimer_ns() - t0 > limit_ns) break;
  }
  report_error(err, QLORA_ERR_TIMEOUT, where);
  return false;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2D tiled TMA load (no multicast) completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// 3D tiled TMA load (no multicast) completing on an mbarrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int32_t x,
                                            int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// Bring a tensor map (kernel parameter) into the TMA descriptor cache.
__device__ __forceinline__ void prefetch_tensormap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16: the A tile sits in TMEM
// (row m in lane m, two bf16 per 32-bit column, K-major).
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once all prior tcgen05.mma of this thread complete.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM data: thread i of the warp gets lane
// (warp's lane quarter base + i), columns col .. col+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Thread i of the warp writes r[0..31] to lane (warp's lane quarter base +
// i), columns col .. col+31.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// Thread i of the warp writes r[0..15] to lane (warp's lane quarter base +
// i), columns col .. col+15.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start
// (launch_dependents), and wait until the kernels this one depends on have
// finished and their writes are visible (wait; returns at once when the
// launch had no programmatic dependency).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace qlora
