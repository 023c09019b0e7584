// tc_gemm.h -- host interface of the tcgen05 (tensor-core) QLoRA kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

struct WView;

// Tile plan shared by the workspace-size query and the launch.
struct TcPlan {
  int bn;          // token tile (MMA N): 16, 32, 64, 128 or 256
  int stages;      // pipeline depth
  int splits;      // split-K factor over the reduction dimension
  int kb_per_split;
};
TcPlan tc_plan(int64_t Mw, int64_t KB, int64_t R);

bool tc_fwd_supported(const WView& w, const void* X, const void* Y, int64_t R);
bool tc_dx_supported(const WView& w, const void* dY, const void* dX, int64_t R);
size_t tc_fwd_ws(const WView& w, int64_t R);
size_t tc_dx_ws(const WView& w, int64_t R);

// The first R*128 bytes of the tensor-core workspace hold the bf16 copy of
// U (forward) or V (input gradient), zero-padded to 64 columns; the caller
// fills it (launch_rowdot's pad output) before the launch.
inline uint16_t* tc_act_pad(void* tcws) { return (uint16_t*)tcws; }
// Next region: the adapter-step weight operand, bf16(s B) [O x 64] in the
// forward or bf16(s A) [64 x I] in the input gradient, also filled by the
// caller (launch_rowdot's side job).
inline uint16_t* tc_w_pad(void* tcws, int64_t R) {
  return (uint16_t*)((char*)tcws + (((size_t)R * 128 + 255) / 256) * 256);
}

// From 2048 tokens (256-token tiles, no K split) the input gradient decodes
// the weight to a bf16 copy in the workspace once per call and the GEMM
// reads that copy: this launches the decode (nothing otherwise).  Call it
// before the rowdot launch that precedes launch_tc_fwd / launch_tc_dx.
cudaError_t tc_prepare(bool dx, const WView& w, int64_t R, void* tcws, cudaStream_t st);

// Y = X W_hat^T + s U B^T  (bf16 in/out, fp32 accumulation in TMEM).
cudaError_t launch_tc_fwd(const WView& w, const void* X, int64_t R, const float* U,
                          const float* B, int32_t r, float s, void* Y, void* tcws,
                          uint32_t* hdr, cudaStream_t st);
// dX = dY W_hat + s V A.
cudaError_t launch_tc_dx(const WView& w, const void* dY, int64_t R, const float* V,
                         const float* A, int32_t r, float s, void* dX, void* tcws, uint32_t* hdr,
                         cudaStream_t st);

}  // namespace qlora
