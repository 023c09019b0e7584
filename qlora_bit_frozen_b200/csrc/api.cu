// api.cu -- the extern "C" entry points of libqlora (declared in qlora.h):
// host-side argument checks, workspace layout and kernel dispatch.
#include <math.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "smallr.h"
#include "tc_gemm.h"

namespace qlora {

std::atomic<uint64_t> g_launches{0};

// ------------------------------------------------- kernel timing records
namespace {
struct TimingRec {
  cudaEvent_t a, b;
  int kind;
  double flops;
};
std::mutex g_tmu;
std::vector<TimingRec> g_trecs;
int g_tmax = 0;
}  // namespace

// Under stream capture an event record must be an external event node to
// record at every replay of the graph.
static void record_event(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
}

int timing_begin(cudaStream_t st, int kind, double flops) {
  std::lock_guard<std::mutex> lk(g_tmu);
  if ((int)g_trecs.size() >= g_tmax) return -1;
  TimingRec r;
  if (cudaEventCreate(&r.a) != cudaSuccess) return -1;
  if (cudaEventCreate(&r.b) != cudaSuccess) {
    cudaEventDestroy(r.a);
    return -1;
  }
  r.kind = kind;
  r.flops = flops;
  record_event(r.a, st);
  g_trecs.push_back(r);
  return (int)g_trecs.size() - 1;
}

bool timing_enabled() {
  std::lock_guard<std::mutex> lk(g_tmu);
  return g_tmax > 0;
}

void timing_end(int slot, cudaStream_t st) {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_tmu);
  if (slot < (int)g_trecs.size()) record_event(g_trecs[slot].b, st);
}

static void timing_clear_locked() {
  for (auto& r : g_trecs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_trecs.clear();
}

namespace {

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
// Element alignment of fp32 arrays (null counts as aligned).
bool al4(const void* p) { return aligned(p, 4); }

qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

qlora_status device_ready() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

// Reads header words 0..2 of a workspace after synchronizing the stream.
qlora_status read_header(const void* ws, cudaStream_t st, uint32_t out[3]) {
  uint32_t h[4] = {0, 0, 0, 0};
  cudaError_t e = cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  out[0] = h[0];
  out[1] = h[1];
  out[2] = h[2];
  return QLORA_OK;
}

int64_t nf4_blocks(int64_t N, int32_t B) { return (N + B - 1) / B; }

qlora_status check_weight(const qlora_weight* w, bool for_linear) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  if (w->O < 0 || w->I < 0 || w->block < 1) return QLORA_ERR_SHAPE;
  if (!weight_count_ok(w->O, w->I)) return QLORA_ERR_SHAPE;
  const int64_t N = w->O * w->I;
  if (w->fmt == QLORA_FMT_NF4_DQ) {
    if (w->bits != 4 || w->group < 1) return QLORA_ERR_SHAPE;
    if (N > 0 && (!w->codes || !w->scale_codes || !w->group_absmax || !w->mean))
      return QLORA_ERR_INVALID_ARG;
    if (!al4(w->group_absmax) || !al4(w->mean)) return QLORA_ERR_ALIGNMENT;
  } else if (w->fmt == QLORA_FMT_NF4_FP32SCALE) {
    if (w->bits != 4) return QLORA_ERR_SHAPE;
    if (N > 0 && (!w->codes || !w->scale)) return QLORA_ERR_INVALID_ARG;
    if (!al4(w->scale)) return QLORA_ERR_ALIGNMENT;
  } else if (w->fmt == QLORA_FMT_AFFINE) {
    if (w->bits != 4 && w->bits != 8) return QLORA_ERR_SHAPE;
    if (N > 0 && (!w->codes || !w->scale || !w->bias)) return QLORA_ERR_INVALID_ARG;
    if (!al4(w->scale) || !al4(w->bias)) return QLORA_ERR_ALIGNMENT;
  } else {
    return QLORA_ERR_INVALID_ARG;
  }
  if (for_linear && w->I % w->block != 0) return QLORA_ERR_SHAPE;
  return QLORA_OK;
}

WView view_of(const qlora_weight* w) {
  WView v;
  v.fmt = w->fmt;
  v.O = w->O;
  v.I = w->I;
  v.block = w->block;
  v.group = w->group < 1 ? 1 : w->group;
  v.bits = w->bits;
  v.codes = w->codes;
  v.qcodes = w->scale_codes;
  v.t = w->group_absmax;
  v.mu = w->mean;
  v.scale = w->scale;
  v.bias = w->bias;
  return v;
}

// ---------------------------------------------------------------- layouts

// Every layout starts with the status header and the ticket counters, both
// zeroed by one memset at the start of the call.
constexpr size_t kWsZeroed = kWsHeader + kWsTickets;

struct FwdLayout {
  size_t u = 0, red = 0, split = 0, sr = 0, tc = 0, total = 0;
};
struct BwdLayout {
  size_t u = 0, v = 0, bt = 0, red = 0, red2 = 0, split = 0, split2 = 0, gemv = 0, sr = 0, tc = 0,
         total = 0;
};

FwdLayout fwd_layout(const qlora_weight* w, int64_t R, int32_t r, int32_t compute) {
  FwdLayout L;
  size_t off = kWsZeroed;
  L.u = off;
  off += align_up((size_t)R * r * 4, 256);
  L.red = off;  // split partials of U = X A^T
  off += rowdot_ws(R, w->I, r);
  L.split = off;  // bf16 hi / lo copy of A (above rank 8)
  off += adapter_split_ws(w->I, r);
  L.sr = off;  // split-K partials of the few-token path
  if (compute == QLORA_COMPUTE_BF16) off += smallr_ws(false, view_of(w), R);
  L.tc = off;
  if (compute == QLORA_COMPUTE_BF16) off += tc_fwd_ws(view_of(w), R);
  L.total = off;
  return L;
}

BwdLayout bwd_layout(const qlora_weight* w, int64_t R, int32_t r, int32_t compute) {
  BwdLayout L;
  size_t off = kWsZeroed;
  L.u = off;
  off += align_up((size_t)R * r * 4, 256);
  L.v = off;
  off += align_up((size_t)R * r * 4, 256);
  L.bt = off;  // B^T [r x O] for the pipelined V = dY B
  off += align_up((size_t)r * w->O * 4, 256);
  L.red = off;
  // partials of the four side products, used one after another
  size_t red = coldot_ws(R, w->I, r);
  const size_t more[3] = {coldot_ws(R, w->O, r), rowdot_ws(R, w->O, r), rowdot_ws(R, w->I, r)};
  for (size_t m : more)
    if (m > red) red = m;
  off += red;
  L.split = off;  // bf16 hi / lo copy of B, V, A or U (one at a time)
  size_t sp = adapter_split_ws(w->O, r);
  const size_t sps[2] = {adapter_split_ws(w->I, r), adapter_split_ws(R, r)};
  for (size_t m : sps)
    if (m > sp) sp = m;
  off += sp;
  L.red2 = off;  // dB partials when dA and dB share a launch
  off += coldot_ws(R, w->O, r);
  L.split2 = off;  // bf16 hi / lo copy of U for that launch
  off += adapter_split_ws(R, r);
  L.gemv = off;  // dX partials of the small-R affine path
  off += gemv_dx_ws(view_of(w), R);
  L.sr = off;  // split-K partials of the few-token path
  if (compute == QLORA_COMPUTE_BF16) off += smallr_ws(true, view_of(w), R);
  L.tc = off;
  if (compute == QLORA_COMPUTE_BF16) off += tc_dx_ws(view_of(w), R);
  L.total = off;
  return L;
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" {

const char* qlora_status_string(qlora_status st) {
  switch (st) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_SHAPE: return "inconsistent shape";
    case QLORA_ERR_ALIGNMENT: return "misaligned pointer or workspace";
    case QLORA_ERR_NONFINITE: return "non-finite weight";
    case QLORA_ERR_UNSUPPORTED: return "unsupported configuration";
    case QLORA_ERR_CUDA: return "CUDA runtime error";
    case QLORA_ERR_TIMEOUT: return "bounded device wait ran out";
    case QLORA_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

qlora_status qlora_nf4_codebook(float out[16]) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  memcpy(out, kNF4Host, sizeof(kNF4Host));
  return QLORA_OK;
}

size_t qlora_nf4_payload_bytes(int64_t N, int32_t B, int32_t C) {
  if (N < 0 || B < 1 || C < 1) return 0;
  const int64_t M = nf4_blocks(N, B);
  const int64_t S = (M + C - 1) / C;
  return (size_t)((N + 1) / 2 + M + 4 * S + 4);
}

size_t qlora_quantize_nf4_workspace_bytes(int64_t N, int32_t B, int32_t C) {
  if (N < 0 || N > kMaxWeights || B < 1 || C < 1) return 0;
  return nf4_quantize_ws(N, B, C);
}

qlora_status qlora_quantize_nf4(const float* W, int64_t O, int64_t I, int32_t B, int32_t C,
                                uint8_t* codes, uint8_t* scale_codes, float* t, float* mu,
                                void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (O < 0 || I < 0 || B < 1 || C < 1) return QLORA_ERR_SHAPE;
  if (!weight_count_ok(O, I)) return QLORA_ERR_SHAPE;
  const int64_t N = O * I;
  if (!mu || !ws) return QLORA_ERR_INVALID_ARG;
  if (N > 0 && (!W || !codes || !scale_codes || !t)) return QLORA_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || !al4(W) || !al4(t) || !al4(mu)) return QLORA_ERR_ALIGNMENT;
  if (ws_bytes < nf4_quantize_ws(N, B, C)) return QLORA_ERR_WORKSPACE;
  qlora_status st = device_ready();
  if (st != QLORA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  st = cuda_status(launch_nf4_quantize(W, N, B, C, codes, scale_codes, t, mu, ws, s));
  if (st != QLORA_OK) return st;
  uint32_t h[3];
  st = read_header(ws, s, h);
  if (st != QLORA_OK) return st;
  if (h[2]) return QLORA_ERR_NONFINITE;
  return h[0] ? (qlora_status)h[0] : QLORA_OK;
}

size_t qlora_nf4_fp32scale_payload_bytes(int64_t N, int32_t B) {
  if (N < 0 || N > kMaxWeights || B < 1) return 0;
  return (size_t)((N + 1) / 2) + 4 * (size_t)((N + B - 1) / B);
}

size_t qlora_quantize_nf4_fp32scale_workspace_bytes(int64_t N, int32_t B) {
  if (N < 0 || N > kMaxWeights || B < 1) return 0;
  return kWsHeader;
}

qlora_status qlora_quantize_nf4_fp32scale(const float* W, int64_t O, int64_t I, int32_t B,
                                          uint8_t* codes, float* scale, void* ws, size_t ws_bytes,
                                          qlora_stream_t stream) {
  if (O < 0 || I < 0 || B < 1) return QLORA_ERR_SHAPE;
  if (!weight_count_ok(O, I)) return QLORA_ERR_SHAPE;
  const int64_t N = O * I;
  if (!ws) return QLORA_ERR_INVALID_ARG;
  if (N > 0 && (!W || !codes || !scale)) return QLORA_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || !al4(W) || !al4(scale)) return QLORA_ERR_ALIGNMENT;
  if (ws_bytes < kWsHeader) return QLORA_ERR_WORKSPACE;
  qlora_status st = device_ready();
  if (st != QLORA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  st = cuda_status(launch_nf4_fp32scale_quantize(W, N, B, codes, scale, ws, s));
  if (st != QLORA_OK) return st;
  uint32_t h[3];
  st = read_header(ws, s, h);
  if (st != QLORA_OK) return st;
  if (h[2]) return QLORA_ERR_NONFINITE;
  return h[0] ? (qlora_status)h[0] : QLORA_OK;
}

size_t qlora_quantize_affine_workspace_bytes(int64_t N, int32_t bits, int32_t G) {
  (void)N;
  (void)bits;
  (void)G;
  return kWsHeader;
}

qlora_status qlora_quantize_affine(const float* W, int64_t O, int64_t I, int32_t bits, int32_t G,
                                   uint8_t* codes, float* scale, float* bias, void* ws,
                                   size_t ws_bytes, qlora_stream_t stream) {
  if (O < 0 || I < 0 || G < 1) return QLORA_ERR_SHAPE;
  if (bits != 4 && bits != 8) return QLORA_ERR_SHAPE;
  if (!weight_count_ok(O, I)) return QLORA_ERR_SHAPE;
  const int64_t N = O * I;
  if (!ws) return QLORA_ERR_INVALID_ARG;
  if (N > 0 && (!W || !codes || !scale || !bias)) return QLORA_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || !al4(W) || !al4(scale) || !al4(bias)) return QLORA_ERR_ALIGNMENT;
  if (ws_bytes < kWsHeader) return QLORA_ERR_WORKSPACE;
  qlora_status st = device_ready();
  if (st != QLORA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  st = cuda_status(launch_affine_quantize(W, N, bits, G, codes, scale, bias, ws, s));
  if (st != QLORA_OK) return st;
  uint32_t h[3];
  st = read_header(ws, s, h);
  if (st != QLORA_OK) return st;
  if (h[2]) return QLORA_ERR_NONFINITE;
  return h[0] ? (qlora_status)h[0] : QLORA_OK;
}

qlora_status qlora_dequantize(const qlora_weight* w, float* W_hat, qlora_stream_t stream) {
  qlora_status st = check_weight(w, false);
  if (st != QLORA_OK) return st;
  if (w->O * w->I > 0 && !W_hat) return QLORA_ERR_INVALID_ARG;
  if (!al4(W_hat)) return QLORA_ERR_ALIGNMENT;
  st = device_ready();
  if (st != QLORA_OK) return st;
  return cuda_status(launch_dequantize(view_of(w), W_hat, (cudaStream_t)stream));
}

qlora_status qlora_merge(const qlora_weight* w, const float* A, const float* B, int32_t r,
                         float alpha, float* W_out, qlora_stream_t stream) {
  qlora_status st = check_weight(w, false);
  if (st != QLORA_OK) return st;
  if (r < 1) return QLORA_ERR_SHAPE;
  if (w->O * w->I > 0 && (!A || !B || !W_out)) return QLORA_ERR_INVALID_ARG;
  if (!al4(A) || !al4(B) || !al4(W_out)) return QLORA_ERR_ALIGNMENT;
  st = device_ready();
  if (st != QLORA_OK) return st;
  const float s = alpha / (float)r;
  return cuda_status(launch_merge(view_of(w), A, B, r, s, W_out, (cudaStream_t)stream));
}

qlora_status qlora_adam_step(float* params, const float* grads, float* m, float* v, int64_t n,
                             int64_t t, float lr, float beta1, float beta2, float eps,
                             int64_t page_elems, qlora_stream_t stream) {
  if (n < 0 || t < 1 || page_elems < 0) return QLORA_ERR_SHAPE;
  if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f))
    return QLORA_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || !isfinite(eps) || !isfinite(lr)) return QLORA_ERR_INVALID_ARG;
  if (n == 0) return QLORA_OK;
  if (!params || !grads || !m || !v) return QLORA_ERR_INVALID_ARG;
  if (!al4(params) || !al4(grads) || !al4(m) || !al4(v)) return QLORA_ERR_ALIGNMENT;
  qlora_status st = device_ready();
  if (st != QLORA_OK) return st;
  return cuda_status(launch_adam(params, grads, m, v, n, t, lr, beta1, beta2, eps, page_elems,
                                 (cudaStream_t)stream));
}

size_t qlora_linear_workspace_bytes(const qlora_weight* w, int64_t R, int32_t r, int32_t op,
                                    int32_t compute) {
  if (!w || R < 0 || r < 1 || r > 64) return 0;
  if (compute != QLORA_COMPUTE_FP32 && compute != QLORA_COMPUTE_BF16) return 0;
  if (op == QLORA_OP_FWD) return fwd_layout(w, R, r, compute).total;
  if (op == QLORA_OP_BWD) return bwd_layout(w, R, r, compute).total;
  return 0;
}

static qlora_status check_linear_common(const qlora_weight* w, int64_t R, const float* A,
                                        const float* B, int32_t r, int32_t compute, void* ws) {
  qlora_status st = check_weight(w, true);
  if (st != QLORA_OK) return st;
  if (R < 0) return QLORA_ERR_SHAPE;
  if (r < 1) return QLORA_ERR_SHAPE;
  if (r > 64) return QLORA_ERR_UNSUPPORTED;
  if (compute != QLORA_COMPUTE_FP32 && compute != QLORA_COMPUTE_BF16) return QLORA_ERR_INVALID_ARG;
  if (!A || !B || !ws) return QLORA_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || !al4(A) || !al4(B)) return QLORA_ERR_ALIGNMENT;
  return QLORA_OK;
}

qlora_status qlora_linear_fwd(const qlora_weight* w, const void* X, int64_t R, const float* A,
                              const float* B, int32_t r, float alpha, int32_t compute, void* Y,
                              float* U_out, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  qlora_status st = check_linear_common(w, R, A, B, r, compute, ws);
  if (st != QLORA_OK) return st;
  if (R > 0 && (!X || !Y)) return QLORA_ERR_INVALID_ARG;
  const size_t esz = compute == QLORA_COMPUTE_BF16 ? 2 : 4;
  if (!aligned(X, esz) || !aligned(Y, esz) || !al4(U_out)) return QLORA_ERR_ALIGNMENT;
  const FwdLayout L = fwd_layout(w, R, r, compute);
  if (ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  st = device_ready();
  if (st != QLORA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, kWsZeroed, s);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  if (R == 0) return QLORA_OK;
  unsigned* tickets = (unsigned*)((char*)ws + kWsHeader);
  float* red = (float*)((char*)ws + L.red);
  const float sc = alpha / (float)r;
  float* U = U_out ? U_out : (float*)((char*)ws + L.u);
  const WView v = view_of(w);
  const bool bf16 = compute == QLORA_COMPUTE_BF16;
  // bf16: the few-token kernels where they are measured faster (or the only
  // fast path), else the tensor-core kernel, else the SIMT tiles
  const bool fwd_tc = bf16 && tc_fwd_supported(v, X, Y, R);
  const bool fwd_sr = bf16 && smallr_supported(v, R, X, Y) && (!fwd_tc || smallr_preferred(false, v, R));
  if (fwd_sr) {
    // 1..16 tokens: U = X A^T, then the bandwidth-bound GEMV, which starts
    // its weight stream at once and waits for U only in its epilogue
    e = launch_rowdot(X, true, R, w->I, A, false, r, U, s, nullptr, nullptr, 0, 0, 1.0f, nullptr,
                      nullptr, red, tickets, (uint16_t*)((char*)ws + L.split));
    if (e == cudaSuccess)
      e = launch_smallr_fwd(v, X, R, U, B, r, sc, Y, (char*)ws + L.sr, (uint32_t*)ws, tickets, s);
  } else if (fwd_tc) {
    void* tcws = (char*)ws + L.tc;
    e = tc_prepare(false, v, R, tcws, s);
    if (e == cudaSuccess)
      e = launch_rowdot(X, true, R, w->I, A, false, r, U, s, tc_act_pad(tcws), B, w->O, 0, sc,
                      tc_w_pad(tcws, R), nullptr, red, tickets, (uint16_t*)((char*)ws + L.split));
    if (e == cudaSuccess) e = launch_tc_fwd(v, X, R, U, B, r, sc, Y, tcws, (uint32_t*)ws, s);
  } else {
    e = launch_simt_fwd(v, X, R, A, B, r, sc, bf16, Y, U, s);
  }
  return cuda_status(e);
}

qlora_status qlora_linear_bwd(const qlora_weight* w, const void* X, const void* dY, int64_t R,
                              const float* A, const float* B, int32_t r, float alpha,
                              const float* U_in, int32_t compute, void* dX, float* dA, float* dB,
                              void* ws, size_t ws_bytes, qlora_stream_t stream) {
  qlora_status st = check_linear_common(w, R, A, B, r, compute, ws);
  if (st != QLORA_OK) return st;
  if (R > 0 && !dY) return QLORA_ERR_INVALID_ARG;
  if (R > 0 && (dA || (dB && !U_in)) && !X) return QLORA_ERR_INVALID_ARG;
  const size_t esz = compute == QLORA_COMPUTE_BF16 ? 2 : 4;
  if (!aligned(X, esz) || !aligned(dY, esz) || !aligned(dX, esz) || !al4(U_in) || !al4(dA) ||
      !al4(dB))
    return QLORA_ERR_ALIGNMENT;
  const BwdLayout L = bwd_layout(w, R, r, compute);
  if (ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  st = device_ready();
  if (st != QLORA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, kWsZeroed, s);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  unsigned* tickets = (unsigned*)((char*)ws + kWsHeader);
  const bool bf16 = compute == QLORA_COMPUTE_BF16;
  const float sc = alpha / (float)r;
  const WView v = view_of(w);
  float* V = (float*)((char*)ws + L.v);
  void* red = (char*)ws + L.red;
  // V = dY B  (B is [O x r]: L(k = o, j) = B[o*r + j]); its padded bf16 copy
  // feeds the tensor-core kernel's adapter step
  const bool dx_tc = dX && bf16 && tc_dx_supported(v, dY, dX, R);
  const bool sr = dX && bf16 && smallr_supported(v, R, dY, dX) && (!dx_tc || smallr_preferred(true, v, R));
  const bool tc = !sr && dx_tc;
  void* tcws = (char*)ws + L.tc;
  if (tc) e = tc_prepare(true, v, R, tcws, s);
  if (e == cudaSuccess && (dX || dA)) {
    float* bt = (float*)((char*)ws + L.bt);
    float* part = (float*)red;
    uint16_t* split = (uint16_t*)((char*)ws + L.split);
    if (tc)
      e = launch_rowdot(dY, bf16, R, w->O, B, true, r, V, s, tc_act_pad(tcws), A, w->I, 1, sc,
                        tc_w_pad(tcws, R), bt, part, tickets, split);
    else
      e = launch_rowdot(dY, bf16, R, w->O, B, true, r, V, s, nullptr, nullptr, 0, 0, 1.0f,
                        nullptr, bt, part, tickets, split);
  }
  // dA = s V^T X [r x I] and dB = s dY^T U [O x r]: one launch when both
  // are wanted (two independent side products), else one each.
  uint16_t* split = (uint16_t*)((char*)ws + L.split);
  const float* U = U_in;
  if (e == cudaSuccess && dB && !U) {
    float* Uw = (float*)((char*)ws + L.u);
    e = launch_rowdot(X, bf16, R, w->I, A, false, r, Uw, s, nullptr, nullptr, 0, 0, 1.0f,
                      nullptr, nullptr, (float*)red, tickets, split);
    U = Uw;
  }
  bool paired = false;
  if (e == cudaSuccess && dA && dB && bf16)
    e = launch_coldot_pair(X, w->I, V, false, dA, red, split, dY, w->O, U, true, dB,
                           (char*)ws + L.red2, (uint16_t*)((char*)ws + L.split2), R, r, sc, s,
                           tickets, &paired);
  if (e == cudaSuccess && dA && !paired)
    e = launch_coldot(X, bf16, R, w->I, V, r, sc, false, dA, red, s, tickets, split);
  if (e == cudaSuccess && dB && !paired)
    e = launch_coldot(dY, bf16, R, w->O, U, r, sc, true, dB, red, s, tickets, split);
  // dX last: the tensor-core kernel starts behind the side products
  // (programmatic dependent launch) and waits for them only before its
  // adapter step, which reads the padded V written above.
  if (e == cudaSuccess && dX) {
    if (sr)
      e = launch_smallr_dx(v, dY, R, V, A, r, sc, dX, (char*)ws + L.sr, (uint32_t*)ws, tickets, s);
    else if (tc)
      e = launch_tc_dx(v, dY, R, V, A, r, sc, dX, tcws, (uint32_t*)ws, s);
    else
      e = launch_simt_dx(v, dY, R, A, V, r, sc, bf16, dX, s, (float*)((char*)ws + L.gemv));
  }
  return cuda_status(e);
}

qlora_status qlora_workspace_status(const void* ws, qlora_stream_t stream) {
  if (!ws) return QLORA_ERR_INVALID_ARG;
  qlora_status st = device_ready();
  if (st != QLORA_OK) return st;
  uint32_t h[3];
  st = read_header(ws, (cudaStream_t)stream, h);
  if (st != QLORA_OK) return st;
  return h[0] ? (qlora_status)h[0] : QLORA_OK;
}

qlora_status qlora_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us,
                                         qlora_stream_t stream) {
  if (!ws) return QLORA_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return QLORA_ERR_ALIGNMENT;
  if (ws_bytes < kWsHeader) return QLORA_ERR_WORKSPACE;
  if (limit_us < 1 || limit_us > 1000000) return QLORA_ERR_INVALID_ARG;
  qlora_status st = device_ready();
  if (st != QLORA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, kWsHeader, s) != cudaSuccess) return QLORA_ERR_CUDA;
  st = cuda_status(launch_wait_selftest((uint32_t*)ws, (uint64_t)limit_us * 1000ull, s));
  if (st != QLORA_OK) return st;
  return qlora_workspace_status(ws, stream);
}

uint64_t qlora_kernel_launch_count(void) { return g_launches.load(); }

qlora_status qlora_kernel_timing_enable(int32_t max_records) {
  if (max_records < 0) return QLORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_tmu);
  timing_clear_locked();
  g_tmax = max_records;
  return QLORA_OK;
}

int32_t qlora_kernel_timing_collect(float* ms, int32_t* kind, double* flops, int32_t max) {
  std::lock_guard<std::mutex> lk(g_tmu);
  int32_t n = 0;
  for (auto& r : g_trecs) {
    if (n >= max) break;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float t = 0.0f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return -1;
    if (ms) ms[n] = t;
    if (kind) kind[n] = r.kind;
    if (flops) flops[n] = r.flops;
    ++n;
  }
  return n;
}

}  // extern "C"
