// noalloc.cu -- NF4 quantization without any caller workspace.
//
// Some callers cannot allocate device memory themselves: a plugin running
// inside a framework whose caching allocator owns the device memory (a raw
// cudaMalloc there would fight the pool or be forbidden by policy), or a
// plain C caller with no allocator to hand, cannot supply the workspace
// qlora_quantize_nf4 asks for.  qlora_quantize_nf4_noalloc serves them: its
// scratch (the per-block absmax values, the fp64 group sums and the status
// header) lives in one file-scope device array of fixed size, reserved when
// the library is loaded, so the call itself allocates nothing.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

// Shared scratch of qlora_quantize_nf4_noalloc.  Every GPU that loads the
// library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// The array's name is only a host-side stand-in; its device address is
// looked up once per device, with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" qlora_status qlora_quantize_nf4_noalloc(const float* W, int64_t O, int64_t I, int32_t B,
                                                   int32_t C, uint8_t* codes,
                                                   uint8_t* scale_codes, float* t, float* mu,
                                                   qlora_stream_t stream) {
  if (O < 0 || I < 0 || B < 1 || C < 1) return QLORA_ERR_SHAPE;
  // O * I (and the scratch size derived from it) is computed only once it
  // is known not to overflow; the size check then bounds every write.
  if (!weight_count_ok(O, I)) return QLORA_ERR_SHAPE;
  const int64_t N = O * I;
  if (!mu) return QLORA_ERR_INVALID_ARG;
  if (N > 0 && (!W || !codes || !scale_codes || !t)) return QLORA_ERR_INVALID_ARG;
  if ((uintptr_t)W % 4 || (uintptr_t)t % 4 || (uintptr_t)mu % 4) return QLORA_ERR_ALIGNMENT;
  if (nf4_quantize_ws(N, B, C) > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  cudaStream_t s = (cudaStream_t)stream;
  // launch_nf4_quantize clears the status header itself; the rest of the
  // scratch is fully overwritten before it is read.
  if (launch_nf4_quantize(W, N, B, C, codes, scale_codes, t, mu, scratch, s) != cudaSuccess)
    return QLORA_ERR_CUDA;
  uint32_t h[4] = {0, 0, 0, 0};
  if (cudaMemcpyAsync(h, scratch, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (h[2]) return QLORA_ERR_NONFINITE;
  return h[0] ? (qlora_status)h[0] : QLORA_OK;
}
