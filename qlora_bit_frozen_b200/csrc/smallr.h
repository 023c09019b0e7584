// smallr.h -- host interface of the small-token-count kernels (1..16 tokens).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

struct WView;

// NF4 (B = 64) or affine (4/8-bit, G = 32/64/128) weight, 1 <= R <= 16 tokens,
// O % 128 == 0, I % 64 == 0, codes and activations 16-byte aligned.
bool smallr_supported(const WView& w, int64_t R, const void* act, const void* out);
// Whether the few-token kernels are the faster choice for this op, format and
// token count where the tensor-core kernel also applies (measured).
bool smallr_preferred(bool dx, const WView& w, int64_t R);
// Workspace bytes of the split-K partial sums (0 when the plan has one split).
size_t smallr_ws(bool dx, const WView& w, int64_t R);

// Y = X W_hat^T + s U B^T.  U [R x r] is written by the launch just before
// (the kernel waits for it only before its epilogue).  tickets: the
// workspace's zeroed counters (this path uses [512, 1024)).
cudaError_t launch_smallr_fwd(const WView& w, const void* X, int64_t R, const float* U,
                              const float* B, int32_t r, float s, void* Y, void* ws,
                              uint32_t* hdr, unsigned* tickets, cudaStream_t st);
// dX = dY W_hat + s V A.
cudaError_t launch_smallr_dx(const WView& w, const void* dY, int64_t R, const float* V,
                             const float* A, int32_t r, float s, void* dX, void* ws,
                             uint32_t* hdr, unsigned* tickets, cudaStream_t st);

}  // namespace qlora
