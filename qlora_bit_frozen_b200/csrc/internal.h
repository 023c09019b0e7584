// internal.h -- host-side declarations shared by the libqlora translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "qlora.h"

namespace qlora {

struct WView;

extern std::atomic<uint64_t> g_launches;
inline void count_launch(uint64_t n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Largest weight count any entry point accepts (2^40, far beyond one GPU's
// memory).  Checked before any size arithmetic, so that O * I and the byte
// counts derived from it cannot overflow.
constexpr int64_t kMaxWeights = (int64_t)1 << 40;
inline bool weight_count_ok(int64_t O, int64_t I) {
  if (O < 0 || I < 0) return false;
  if (O == 0 || I == 0) return true;
  return O <= kMaxWeights / I;
}

// Zeroed ticket counters after the workspace status header (1024 x u32):
// zeroed with the header at the start of every linear call; kernels that
// take one leave it zero again.
constexpr size_t kWsTickets = 4096;

// Bounded-wait limit for device spin loops, nanoseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// quantize.cu
cudaError_t launch_nf4_quantize(const float* W, int64_t N, int32_t B, int32_t C, uint8_t* codes,
                                uint8_t* qcodes, float* t, float* mu, void* ws, cudaStream_t st);
size_t nf4_quantize_ws(int64_t N, int32_t B, int32_t C);
// legacy scale storage: codes and the fp32 block absmax (ws: the status header)
cudaError_t launch_nf4_fp32scale_quantize(const float* W, int64_t N, int32_t B, uint8_t* codes,
                                          float* scale, void* ws, cudaStream_t st);
cudaError_t launch_affine_quantize(const float* W, int64_t N, int32_t bits, int32_t G,
                                   uint8_t* codes, float* scale, float* bias, void* ws,
                                   cudaStream_t st);
cudaError_t launch_dequantize(const WView& w, float* out, cudaStream_t st);

// merge.cu -- out [O x I] = W_hat + s B A (B [O x r], A [r x I], fp32)
cudaError_t launch_merge(const WView& w, const float* A, const float* B, int32_t r, float s,
                         float* out, cudaStream_t st);

// adam.cu -- one Adam step over n fp32 parameters; page > 0: one launch per
// page of at most `page` elements, in order
cudaError_t launch_adam(float* p, const float* g, float* m, float* v, int64_t n, int64_t t,
                        float lr, float beta1, float beta2, float eps, int64_t page,
                        cudaStream_t st);

// simt.cu -- generic (SIMT) linear kernels, both compute modes
cudaError_t launch_simt_fwd(const WView& w, const void* X, int64_t R, const float* A,
                            const float* B, int32_t r, float s, bool bf16, void* Y, float* U,
                            cudaStream_t st);
// gemv_ws (gemv_dx_ws bytes, nullable): split partials of the small-R
// affine path.
cudaError_t launch_simt_dx(const WView& w, const void* dY, int64_t R, const float* A,
                           const float* V, int32_t r, float s, bool bf16, void* dX,
                           cudaStream_t st, float* gemv_ws = nullptr);
size_t gemv_dx_ws(const WView& w, int64_t R);
// adapter side products
// adapter.cu
//   out[m, j] = sum_k P[m, k] L(k, j); pad (nullable): its bf16 copy [R x 64].
//   Optional side job in the same launch (side_dst != nullptr): the
//   zero-padded bf16(side_mul * src) operand, mode 0: [extent x 64] from
//   src [extent x r]; mode 1: [64 x extent] from src [r x extent].
//   lt_ws (nullable, r*K floats): scratch for L^T when l_is_kr, which lets
//   the pipelined kernel read the factor row-wise.
cudaError_t launch_rowdot(const void* P, bool bf16, int64_t R, int64_t K, const float* L,
                          bool l_is_kr, int32_t r, float* out, cudaStream_t st,
                          uint16_t* pad = nullptr, const float* side_src = nullptr,
                          int64_t side_extent = 0, int side_mode = 0, float side_mul = 1.0f,
                          uint16_t* side_dst = nullptr, float* lt_ws = nullptr,
                          float* part_ws = nullptr, unsigned* tickets = nullptr,
                          uint16_t* split_ws = nullptr);
// part_ws (rowdot_ws bytes) and tickets (kWsTickets bytes, zero on entry
// and left zero) let the bf16 tensor-core path split K across blocks.
size_t rowdot_ws(int64_t R, int64_t K, int32_t r);
// split_ws (adapter_split_ws(extent, r) bytes, nullable): scratch for the
// bf16 hi / lo copy of the r-wide operand (factor over K, or U / V over R)
// that the tensor-core side products read above rank 8.
size_t adapter_split_ws(int64_t extent, int32_t r);
size_t coldot_ws(int64_t R, int64_t N, int32_t r);
// tickets: as for launch_rowdot (nullptr: no row splits on the tensor-core path)
cudaError_t launch_coldot(const void* P, bool bf16, int64_t R, int64_t N, const float* aux,
                          int32_t r, float s, bool out_nr, float* out, void* ws,
                          cudaStream_t st, unsigned* tickets = nullptr,
                          uint16_t* split_ws = nullptr);
// Two coldot products over the same R rows in one launch (the backward's
// dA = s V^T X and dB = s dY^T U), each with its own partial buffer
// (coldot_ws) and split scratch; *done = false (nothing launched) when the
// tensor-core path does not apply to both, and the caller launches them one
// by one.
cudaError_t launch_coldot_pair(const void* PA, int64_t NA, const float* auxA, bool out_nrA,
                               float* outA, void* wsA, uint16_t* splitA, const void* PB,
                               int64_t NB, const float* auxB, bool out_nrB, float* outB, void* wsB,
                               uint16_t* splitB, int64_t R, int32_t r, float s, cudaStream_t st,
                               unsigned* tickets, bool* done);
// out = scale * sum of the split partials.  pdl: launched with a
// programmatic dependency on the kernel before it (which must have
// triggered its dependents); the kernel waits for that grid first.
cudaError_t launch_splitk_reduce(const float* part, int32_t splits, int64_t R, int64_t N,
                                 bool bf16_out, void* out, cudaStream_t st, float scale = 1.0f,
                                 bool pdl = false);

// selftest
cudaError_t launch_wait_selftest(uint32_t* ws_header, uint64_t limit_ns, cudaStream_t st);

// kernel timing instrumentation (api.cu): returns a slot to record into, or -1
int timing_begin(cudaStream_t st, int kind, double flops);
void timing_end(int slot, cudaStream_t st);
// true while kernel timing is switched on (launches then keep plain stream order)
bool timing_enabled();

}  // namespace qlora
