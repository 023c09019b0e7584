/*
 * qlora.h -- C ABI of libqlora: the QLoRA linear layer on one NVIDIA B200
 * (sm_100a).  A frozen base weight stored as blockwise NF4 with
 * double-quantized scales (or as affine 4/8-bit groups), plus a trainable
 * fp32 rank-r LoRA adapter:
 *
 *   forward   Y  = X W_hat^T + s (X A^T) B^T             s = alpha / r
 *   backward  dX = dY W_hat  + s (dY B) A
 *             dA = s (dY B)^T X          dB = s dY^T (X A^T)
 *   (no weight gradient: the base is frozen)
 *
 * Sources (page title, section):
 *   "QLoRA Fine-Tuning" (Riftco Transformer how-to): "NF4 representation"
 *     (format, double quantization, payload sizes) and "Forward and
 *     backward" (the two sums, one autograd parent, decode inside the sums).
 *   "QLoRA on Mac -- fine-tuning larger open models on 48 GB", "Design /
 *     Q-LoRA layer" (base + (alpha/r)(x A^T) B^T with fp32 A/B).
 *   "LoRA vs QLoRA on Apple Silicon ... in MLX", "Method" (affine
 *     group-wise 4/8-bit quantization with fp32 scale and bias).
 *   "QLoRA Fine-Tuning", "Training lifecycle" and "Current scope" (the
 *     adapter-only Adam step with paged state, and the fp32 export).
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers owned by the caller, unless a
 *     comment says "host".  Matrices are row-major and dense.
 *   - The library never allocates device memory.  Scratch space is a caller
 *     workspace (`ws`, `ws_bytes`); its required size comes from the
 *     matching *_workspace_bytes() function.  `ws` must be 256-byte aligned.
 *   - fp32 arrays must be 4-byte aligned and bf16 arrays 2-byte aligned
 *     (QLORA_ERR_ALIGNMENT otherwise); faster paths that need 16-byte
 *     alignment are chosen only when the pointers have it.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Only qlora_quantize_nf4, qlora_quantize_affine and
 *     qlora_workspace_status synchronize `stream` (to read a device flag).
 *   - Arguments are validated on the host before anything is launched; a
 *     rejected call returns a status and enqueues nothing.  Nothing aborts
 *     and no exception crosses the ABI.
 *   - Weights are read-only in fwd/bwd.  dA and dB are overwritten, not
 *     accumulated.
 *   - Calls on distinct streams with distinct workspaces are thread-safe.
 *   - If no CUDA device is usable, every compute entry point returns
 *     QLORA_ERR_CUDA; there is no CPU fallback.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qlora_stream_t; /* same handle as cudaStream_t */

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, negative size      */
  QLORA_ERR_SHAPE = 2,        /* sizes inconsistent with the format         */
  QLORA_ERR_ALIGNMENT = 3,    /* pointer or workspace misaligned            */
  QLORA_ERR_NONFINITE = 4,    /* NaN/Inf weight given to a quantizer        */
  QLORA_ERR_UNSUPPORTED = 5,  /* valid but not implemented (e.g. r > 64)    */
  QLORA_ERR_CUDA = 6,         /* a CUDA runtime call failed                 */
  QLORA_ERR_TIMEOUT = 7,      /* a bounded device wait ran out              */
  QLORA_ERR_WORKSPACE = 8     /* ws_bytes smaller than required             */
} qlora_status;

typedef enum {
  QLORA_FMT_NF4_DQ = 0,        /* NF4 codes + u8 scale codes + fp32 t_g + fp32 mu */
  QLORA_FMT_NF4_FP32SCALE = 1, /* NF4 codes + one fp32 absmax per block (legacy) */
  QLORA_FMT_AFFINE = 2         /* 4/8-bit codes + fp32 scale and bias per group   */
} qlora_format;

typedef enum {
  QLORA_COMPUTE_FP32 = 0, /* X, dY, Y, dX are fp32; fp32 SIMT arithmetic     */
  QLORA_COMPUTE_BF16 = 1  /* X, dY, Y, dX are bf16; bf16 tensor-core operands,
                             fp32 accumulation                               */
} qlora_compute;

/*
 * Non-owning view of a quantized weight W_hat [O x I] (logical row-major,
 * flat index n = o*I + i).  All pointers are device memory.
 *   NF4_DQ:  block = B (weights per absmax block), group = C (blocks per
 *            second-level group), bits = 4.
 *            codes        ceil(N/2) bytes, weight 2j in the low nibble of
 *                         byte j, 2j+1 in the high nibble
 *            scale_codes  M = ceil(N/B) bytes q_b
 *            group_absmax S = ceil(M/C) floats t_g
 *            mean         1 float mu
 *   NF4_FP32SCALE (legacy scale storage):  block = B, group ignored,
 *            bits = 4.
 *            codes        ceil(N/2) bytes, as for NF4_DQ
 *            scale        M = ceil(N/B) floats: the block absmax s_b itself
 *            (ceil(N/2) + 4M payload bytes, about 4.5 bits per weight at
 *            B = 64; w_hat = c[code] * s_b)
 *   AFFINE:  block = G (weights per group), group ignored, bits = 4 or 8.
 *            codes        ceil(N*bits/8) bytes (4-bit: low nibble first)
 *            scale, bias  ceil(N/G) floats each
 *            w_hat = scale_g * code + bias_g
 * The fwd/bwd entry points require I % block == 0 (blocks never straddle
 * rows); the quantizers and qlora_dequantize accept any N.
 */
typedef struct {
  int32_t fmt; /* qlora_format */
  int64_t O, I;
  int32_t block, group, bits;
  const uint8_t* codes;
  const uint8_t* scale_codes;
  const float* group_absmax;
  const float* mean;
  const float* scale;
  const float* bias;
} qlora_weight;

/* Human-readable name of a status (static string, never NULL). */
const char* qlora_status_string(qlora_status st);

/*
 * HOST.  Writes the library's 16 fp32 NF4 levels (ascending, c[7] = 0) to
 * the host array `out`.  Source: "QLoRA Fine-Tuning", "NF4 representation"
 * (a fixed 16-value codebook whose constants match the canonical
 * bitsandbytes mapping) and "QLoRA: Fine-Tuning Under Memory Constraints",
 * "Understand what NF4 chooses" (levels follow a normal distribution).  The
 * values are that canonical table bit for bit: normal quantiles at
 * single-precision probabilities spaced evenly from 0.9677083 down to 1/2
 * (8 positive, 7 negative, plus zero), divided by the largest.
 */
qlora_status qlora_nf4_codebook(float out[16]);

/*
 * HOST.  Payload bytes of the double-quantized format: ceil(N/2) + M + 4S
 * + 4 ("QLoRA Fine-Tuning", "NF4 representation").  0 on bad arguments.
 */
size_t qlora_nf4_payload_bytes(int64_t N, int32_t B, int32_t C);

/* HOST.  Workspace bytes qlora_quantize_nf4 needs for N weights. */
size_t qlora_quantize_nf4_workspace_bytes(int64_t N, int32_t B, int32_t C);

/*
 * Quantize W [O x I] fp32 to NF4 with double-quantized scales
 * ("QLoRA Fine-Tuning", "NF4 representation"):
 *   s_b = max |w| over block b (B consecutive weights of the flat order);
 *   code = nearest of the 16 levels to fp32(w / s_b), ties to the lower
 *   level; an all-zero block gets s_b = 0 and the zero level (code 7);
 *   mu = mean of s_b (fp64 sums: sequential within each group of C blocks,
 *   then over groups; rounded to fp32);
 *   t_g = max |fp32(s_b - mu)| over group g;
 *   q_b = 128 + clamp(round(fp32(fp32(127 (s_b - mu)) / t_g)), -127, 127),
 *   round half away from zero; q_b = 128 when t_g = 0.
 * Outputs (device): codes [ceil(N/2)], scale_codes [M], t [S], mu [1].
 * Bit-exact and deterministic.  Synchronizes `stream` at the end to read
 * the non-finite flag: returns QLORA_ERR_NONFINITE (outputs undefined) if
 * W holds a NaN or Inf.  N = 0 is valid (mu = 0).
 */
qlora_status qlora_quantize_nf4(const float* W, int64_t O, int64_t I, int32_t B, int32_t C,
                                uint8_t* codes, uint8_t* scale_codes, float* t, float* mu,
                                void* ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * qlora_quantize_nf4 for callers that cannot allocate device memory (the
 * pages have no counterpart; this is an interface convenience).  A plugin
 * inside a framework whose caching allocator owns the device memory, or a
 * plain C caller with no allocator, may be unable to provide the workspace
 * qlora_quantize_nf4 needs; this entry point takes none and calls no
 * allocation routine.  Its scratch is one file-scope device array of
 * 8 MiB that every GPU loading the library holds until the process exits;
 * that covers qlora_quantize_nf4_workspace_bytes(N, B, C) <= 8 MiB (at B = 64,
 * C = 256 about 133 million weights).  Larger inputs return
 * QLORA_ERR_WORKSPACE (use qlora_quantize_nf4 with a workspace instead).
 * Same arguments (minus the workspace), outputs, bit-exact results and
 * synchronization as qlora_quantize_nf4.
 * The first call on a device looks up the array's device address there
 * (with that device current); make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents: calls that overlap on the GPU (another stream, another host
 * thread on the same device) race and must be serialized by the caller.
 */
qlora_status qlora_quantize_nf4_noalloc(const float* W, int64_t O, int64_t I, int32_t B, int32_t C,
                                        uint8_t* codes, uint8_t* scale_codes, float* t, float* mu,
                                        qlora_stream_t stream);

/*
 * HOST.  Payload bytes of the legacy format: ceil(N/2) + 4 ceil(N/B)
 * ("QLoRA Fine-Tuning", "NF4 representation": one fp32 scale per block,
 * about 4.5 bits per weight at B = 64).  0 on bad arguments.
 */
size_t qlora_nf4_fp32scale_payload_bytes(int64_t N, int32_t B);

/* HOST.  Workspace bytes qlora_quantize_nf4_fp32scale needs (the status header). */
size_t qlora_quantize_nf4_fp32scale_workspace_bytes(int64_t N, int32_t B);

/*
 * Quantize W [O x I] fp32 to NF4 with the legacy scale storage ("QLoRA
 * Fine-Tuning", "NF4 representation": each block's absmax kept as an fp32
 * number).  Codes exactly as qlora_quantize_nf4 (nearest level to
 * fp32(w / s_b), ties to the lower level, low nibble first, an all-zero
 * block gets s_b = 0 and code 7); scale[b] = s_b.
 * Outputs (device): codes [ceil(N/2)], scale [M].  Bit-exact and
 * deterministic.  Synchronizes `stream` to read the non-finite flag
 * (QLORA_ERR_NONFINITE on NaN/Inf).  N = 0 is valid.
 */
qlora_status qlora_quantize_nf4_fp32scale(const float* W, int64_t O, int64_t I, int32_t B,
                                          uint8_t* codes, float* scale, void* ws, size_t ws_bytes,
                                          qlora_stream_t stream);

/* HOST.  Workspace bytes qlora_quantize_affine needs. */
size_t qlora_quantize_affine_workspace_bytes(int64_t N, int32_t bits, int32_t G);

/*
 * Affine group-wise quantization ("LoRA vs QLoRA on Apple Silicon",
 * "Method"; the pages print no formula -- the plain min/max scheme):
 *   per group of G weights: bias = min, scale = fp32(fp32(max - min) /
 *   (2^bits - 1)), code = clamp(round(fp32(fp32(w - bias) / scale)), 0,
 *   2^bits - 1) (0 when scale = 0).  4-bit codes pack low nibble first.
 * Outputs: codes [ceil(N*bits/8)], scale [ceil(N/G)], bias [ceil(N/G)].
 * Synchronizes `stream`; QLORA_ERR_NONFINITE for NaN/Inf or an infinite
 * range.
 */
qlora_status qlora_quantize_affine(const float* W, int64_t O, int64_t I, int32_t bits, int32_t G,
                                   uint8_t* codes, float* scale, float* bias, void* ws,
                                   size_t ws_bytes, qlora_stream_t stream);

/*
 * Diagnostic dequantization ("QLoRA Fine-Tuning", "NF4 representation":
 * dequantize() is an explicit diagnostic/export operation that the training
 * kernels never call).  W_hat [O x I] fp32:
 *   NF4_DQ: c[code] * s_hat_b,  s_hat_b = clamp(mu + fp32(fp32(t_g (q_b -
 *           128)) / 127), 0, FLT_MAX);
 *   NF4_FP32SCALE: c[code] * s_b;
 *   AFFINE: fp32(scale_g * code) + bias_g.
 * Bit-exact.  Never used by qlora_linear_fwd / qlora_linear_bwd.
 */
qlora_status qlora_dequantize(const qlora_weight* w, float* W_hat, qlora_stream_t stream);

/*
 * Export of a trained layer ("QLoRA Fine-Tuning", "Training lifecycle":
 * at export the packed weights are dequantized and the trained LoRA deltas
 * added, restoring ordinary fp32 weights).  W_out [O x I] fp32:
 *   W_out[o,i] = fp32(W_hat[o,i] + fp32(s * delta)),  s = alpha / r (fp32),
 *   delta = sum_k B[o,k] A[k,i]  (fp32 FMAs in k order),
 * W_hat decoded exactly as qlora_dequantize does, so B = 0 or alpha = 0
 * gives the dequantized weight.  A [r x I], B [O x r] fp32, device memory;
 * W_out must not overlap the inputs.  Any r >= 1 and any O, I.  The result
 * is a plain fp32 matrix; requantizing it (qlora_quantize_nf4) is a second,
 * separate approximation.  Never used by the training entry points.
 */
qlora_status qlora_merge(const qlora_weight* w, const float* A, const float* B, int32_t r,
                         float alpha, float* W_out, qlora_stream_t stream);

/*
 * One Adam step over n fp32 parameters ("QLoRA Fine-Tuning", "Training
 * lifecycle": only the LoRA factors are optimizer inputs; "Current scope":
 * paged Adam state).  params, grads, m, v: n floats each, device (or
 * managed) memory, distinct buffers; params, m and v are updated in place.
 * With step count t >= 1, bc1 = fp32(1 - beta1^t), bc2 = fp32(1 - beta2^t):
 *   m = b1 m + fp32(1 - b1) g
 *   v = b2 v + fp32(1 - b2) g^2
 *   params -= lr (m / bc1) / (sqrt(v / bc2) + eps)
 * every fp32 operation rounded once (no contraction).  No weight decay.
 * page_elems > 0 updates the state in pages of at most page_elems elements,
 * one launch per page in order (for state kept in managed memory); 0 is one
 * launch.  The result is the same bits either way.  Requires 0 <= beta < 1,
 * eps > 0, finite lr.  To update every adapter factor in one call, keep them
 * in one flat arena (A and B of each layer as views into it).
 */
qlora_status qlora_adam_step(float* params, const float* grads, float* m, float* v, int64_t n,
                             int64_t t, float lr, float beta1, float beta2, float eps,
                             int64_t page_elems, qlora_stream_t stream);

/* op codes for qlora_linear_workspace_bytes */
#define QLORA_OP_FWD 0
#define QLORA_OP_BWD 1

/*
 * HOST.  Workspace bytes of qlora_linear_fwd (op 0) or qlora_linear_bwd
 * (op 1) for this weight, token count R, rank r and compute mode.  Besides
 * small per-call scratch (status header, tickets, U / V, split partials),
 * the bf16 backward from 2048 tokens on includes a bf16 copy of the decoded
 * weight (2 O I bytes): the input gradient decodes the weight into it once
 * per call and its GEMM reads it there.  The workspace is scratch for one
 * call at a time; the weight itself stays packed.
 */
size_t qlora_linear_workspace_bytes(const qlora_weight* w, int64_t R, int32_t r, int32_t op,
                                    int32_t compute);

/*
 * QLoRA linear forward ("QLoRA Fine-Tuning", "Forward and backward";
 * "QLoRA on Mac", "Design / Q-LoRA layer"):
 *   U = X A^T                      [R x r] fp32
 *   Y = X W_hat^T + s U B^T        [R x O]
 * X [R x I] and Y [R x O] are fp32 (QLORA_COMPUTE_FP32) or bf16
 * (QLORA_COMPUTE_BF16); A [r x I] and B [O x r] are fp32; s = alpha / r in
 * fp32.  U_out (nullable) receives U for reuse by the backward pass.
 * Every weight is decoded from its nibble and block scale inside the
 * kernels; no full-size floating-point weight is formed.  R = 0 is valid.
 * bf16 mode: W_hat and the adapter operands enter the tensor cores as bf16,
 * accumulation is fp32, Y is rounded to bf16 once.  U (and, in the
 * backward, V, dA and dB) use the bf16 activations exactly and the fp32
 * factors to 16 significant bits (each split into two bf16 halves).
 * Deterministic: the same inputs give the same bits (every reduction
 * across blocks is summed in a fixed order).
 * Requires 1 <= r <= 64 and I % block == 0.
 */
qlora_status qlora_linear_fwd(const qlora_weight* w, const void* X, int64_t R, const float* A,
                              const float* B, int32_t r, float alpha, int32_t compute, void* Y,
                              float* U_out, void* ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * QLoRA linear backward (vector-Jacobian product; "QLoRA Fine-Tuning",
 * "Forward and backward": the node's only parent is the input, so there is
 * no weight gradient; the LoRA factors get the ordinary chain rule):
 *   V  = dY B                      [R x r]
 *   dX = dY W_hat + s V A          [R x I]  (nullable: skipped)
 *   dA = s V^T X                   [r x I]  (nullable: skipped)
 *   dB = s dY^T U                  [O x r]  (nullable: skipped)
 * U_in (nullable) is U = X A^T from the forward; when NULL it is
 * recomputed.  Types as in qlora_linear_fwd; dA and dB are fp32 and
 * overwritten.
 */
qlora_status qlora_linear_bwd(const qlora_weight* w, const void* X, const void* dY, int64_t R,
                              const float* A, const float* B, int32_t r, float alpha,
                              const float* U_in, int32_t compute, void* dX, float* dA, float* dB,
                              void* ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * Reads the device error word that the kernels of the last call using
 * workspace `ws` may have set (bounded waits that ran out, device-side
 * argument checks).  Synchronizes `stream`.  Returns QLORA_OK or the first
 * error recorded (e.g. QLORA_ERR_TIMEOUT).
 */
qlora_status qlora_workspace_status(const void* ws, qlora_stream_t stream);

/*
 * Failure-detection self test: launches one tiny kernel that waits on an
 * mbarrier nothing ever arrives on, with a wait limit of `limit_us`
 * microseconds (1..1000000).  The wait gives up, the kernel records
 * QLORA_ERR_TIMEOUT in `ws` (>= 256 bytes) and returns; the context stays
 * usable.  Returns the status read back (QLORA_ERR_TIMEOUT when the
 * mechanism works).  Synchronizes `stream`.
 */
qlora_status qlora_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us,
                                         qlora_stream_t stream);

/*
 * HOST.  Number of CUDA kernels the library launched in this process so far
 * (counted on the host at each launch).
 */
uint64_t qlora_kernel_launch_count(void);

/*
 * HOST.  Kernel timing instrumentation.  With max_records > 0 the library
 * records a CUDA event pair on the launching stream around each launch of
 * its tensor-core GEMM kernels (up to max_records launches; events are
 * created here, no device memory is allocated); 0 disables and drops
 * pending records.  While enabled, those kernels are launched in plain
 * stream order (no programmatic overlap with the launch before them), so
 * the recorded durations are the kernels' own.
 */
qlora_status qlora_kernel_timing_enable(int32_t max_records);

/*
 * HOST.  Waits for the recorded event pairs, writes up to `max` launch
 * durations (milliseconds) to ms[] and each launch's kind to kind[]
 * (0 = forward GEMM, 1 = input-gradient GEMM) and its algorithmic flop count
 * to flops[] (host arrays; any may be NULL) and returns how many were
 * written (negative on a CUDA error).  Records are kept (launches captured
 * in a CUDA graph re-record the same events at every replay, so collect
 * after each replay); qlora_kernel_timing_enable() drops them.
 */
int32_t qlora_kernel_timing_collect(float* ms, int32_t* kind, double* flops, int32_t max);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
