// smallr.cu -- the QLoRA linear layer at a handful of tokens (1..16).
//
// Forward  Y  = X W_hat^T + s U B^T     ("QLoRA Fine-Tuning", "Forward and
// Input    dX = dY W_hat + s V A         backward": every weight decoded from
// gradient                               its code and block scale inside the
//                                        sums; "LoRA vs QLoRA on Apple
//                                        Silicon", "Results": the 4-bit base
//                                        reads 4x fewer weight bytes)
//
// With 1..16 tokens the layer streams the packed weight once and does a few
// multiply-adds per weight: it is bound by HBM bandwidth on the packed
// bytes, and the work per byte is the decode.  The kernels here are a
// split-K GEMV shaped for that:
//
//  * the weight is the M side of mma.sync.m16n8k16 (bf16 in, fp32
//    accumulate); the tokens are N (one or two 8-token tiles), so a single
//    token wastes MMA columns, not decode work;
//  * codes are decoded two weights at a time through a 256-entry byte table
//    in shared memory: entry[byte] = (v[byte & 15], v[byte >> 4]) as a bf16
//    pair, one copy per lane at stride 256 bytes, so a lookup is one byte
//    permute (which builds the address) and one conflict-free 32-bit shared
//    load, and the result is an MMA operand register as it stands;
//  * the tables hold UNSCALED values (the 16 NF4 levels, or the integers
//    0..15 of affine codes), so the block or group scale is applied once per
//    block: in the forward pass to the block's fp32 partial sums
//    (acc += s_b * D_b; the affine bias adds bias_g * sum(x) over the group),
//    in the input gradient to the dY operand (dY[o] * s(o, b) is the same for
//    every column of a 64-column block);
//  * 8-bit affine codes are split into their two nibbles: a code byte looks
//    up (lo, hi) in the same integer table and meets the activation pair
//    (x, 16 x), so x q = x lo + 16 x hi with the K dimension doubled;
//  * affine groups of 32 (two per 64-column block) run two passes with the
//    other group's operand lanes zeroed;
//  * K is split across the CTAs of a one-wave grid; partial sums go to the
//    workspace and the last CTA of each output tile (a ticket counter) adds
//    them in split order, so the result is deterministic, and adds the
//    adapter term s U B^T (or s V A) from U / V computed by the launch just
//    before (programmatic dependent launch: the weight stream starts at
//    once, the wait comes only before U / V are read).
//
// No floating-point copy of the weight exists anywhere: codes go from HBM to
// registers and from registers, through the table, into the MMA.
#include "common.cuh"
#include "internal.h"
#include "smallr.h"

namespace qlora {

namespace {

constexpr int kSrThreads = 256;       // 8 warps
constexpr int kTableBytes = 256 * 256;  // 256 entries x 64 words (32 lane copies used)
constexpr int kTicketBase = 512;      // ticket counters [512, 1024) of the workspace

enum SrFmt { kFmtNF4 = 0, kFmtA4 = 1, kFmtA8 = 2 };

struct SrParams {
  const uint8_t* codes;
  const uint8_t* qcodes;  // NF4: scale codes q_b
  const float* t;         // NF4: t_g
  const float* mu;        // NF4: mu
  const float* scale;     // affine scale, or the legacy format's fp32 s_b
  const float* bias;      // affine
  int32_t legacy;         // NF4 with fp32 block scales
  int32_t G;              // affine group size
  uint32_t C;             // NF4 scale-group size (blocks)
  int32_t c_shift;        // log2(C) or -1
  const __nv_bfloat16* act;  // X [R x I] (forward) or dY [R x O] (input gradient)
  int32_t R;
  int64_t O, I;
  const float* aux;   // U [R x r] (forward) or V [R x r] (input gradient)
  const float* lora;  // B [O x r] (forward) or A [r x I] (input gradient)
  int32_t r;
  float s;
  __nv_bfloat16* out;  // Y [R x O] or dX [R x I]
  float* part;         // split partials [splits][R][extent]
  unsigned* tickets;   // one counter per output tile, zero on entry, left zero
  int32_t splits;
  int32_t per_split;   // K blocks (forward) or 16-row steps (input gradient) per split
  uint32_t* err;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}


// The lane's copy of table entry `byte k of w`: address byte * 256 + lane * 4
// (laneoff holds lane * 4 in its low byte, zeros above), built by one permute.
__device__ __forceinline__ uint32_t tbl(const uint32_t* table, uint32_t w, uint32_t laneoff,
                                        int k) {
  const uint32_t addr = prmt(w, laneoff, 0x5504u | ((uint32_t)k << 4));
  return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(table) + addr);
}

// Fill the byte table: NF4 levels, or the integers 0..15 (affine codes).
template <int FMT>
__device__ __forceinline__ void fill_table(uint32_t* table) {
  for (int e = threadIdx.x; e < 256 * 8; e += kSrThreads) {
    const int entry = e >> 3, q4 = e & 7;  // 8 x uint4 = 32 lane copies
    float lo, hi;
    if (FMT == kFmtNF4) {
      lo = kNF4[entry & 15];
      hi = kNF4[entry >> 4];
    } else {
      lo = (float)(entry & 15);
      hi = (float)(entry >> 4);
    }
    const uint32_t v = pack_bf16x2(lo, hi);
    reinterpret_cast<uint4*>(table)[entry * 16 + q4] = make_uint4(v, v, v, v);
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Raw inputs of a block scale, loaded ahead of their use: NF4 (q_b, t_g),
// or the legacy format's stored s_b (in t, with q = 0xFFFFFFFF).
__device__ __forceinline__ void nf4_scale_load(const SrParams& p, uint32_t b, uint32_t& q, float& t) {
  if (p.legacy) {
    q = 0xFFFFFFFFu;
    t = __ldg(p.scale + b);
    return;
  }
  const uint32_t g = p.c_shift >= 0 ? (b >> p.c_shift) : b / p.C;
  q = __ldg(p.qcodes + b);
  t = __ldg(p.t + g);
}
// The block scale as the GEMM uses it: mu + t_g (q_b - 128) / 127 with the
// division replaced by a multiply (within an ulp of the stored-format
// decode; the GEMM rounds its operands to bf16 anyway).
__device__ __forceinline__ float nf4_scale_decode(uint32_t q, float t, float mu) {
  if (q == 0xFFFFFFFFu) return t;
  const float s = fmaf(t * (float)((int)q - 128), 1.0f / 127.0f, mu);
  return fmaxf(s, 0.0f);
}


// ------------------------------------------------------------------ forward
//
// CTA: 128 weight rows x one K range (split blockIdx.y).  Warp w owns the
// 16 rows 16 w .. 16 w + 15 of the tile (one m16 MMA tile) over the CTA's
// whole K range, so no two warps share an output and nothing is reduced
// inside the CTA.  Per 64-column block the lane holds, for rows g and g + 8
// (t = lane % 4, g = lane / 4), the 16 columns 16 t .. 16 t + 15: 8 code
// bytes (4-bit) or 16 (8-bit).  MMA j of the block pairs K index (2t, 2t+1)
// with columns 16t + 4j + {0,1} and (2t+8, 2t+9) with 16t + 4j + {2,3}
// (4-bit; 8-bit: one column per K pair, 16t + 2j and 16t + 2j + 1), and the
// activation operand is loaded in the same order.
//
// Codes stream through a ring of kStages stages per warp, a stage being
// 128 contiguous bytes of each of the warp's 16 rows (4 blocks of 4-bit
// codes, 2 of 8-bit): whole 128-byte lines, so that DRAM serves long runs of
// each row rather than 32-byte pieces of thousands of rows.  In shared
// memory the 16-byte chunk c of row y sits at c ^ swz(y), which keeps the
// lanes' reads conflict-free.  Per stage lane l loads the scale inputs of
// row l % 16 (blocks l / 16, l / 16 + 2, ...; groups of 32: group half
// l / 16 of every block), and rows g and g + 8 take theirs by shuffles.
template <int FMT>
struct FwdShape {
  static constexpr int kChunkU32 = FMT == kFmtA8 ? 4 : 2;  // code words per row per block
  static constexpr int kMmas = FMT == kFmtA8 ? 8 : 4;      // MMAs per block
  static constexpr int kRowBytes = FMT == kFmtA8 ? 64 : 32;
  static constexpr int kStageBlocks = 128 / kRowBytes;     // blocks per stage
  static constexpr int kStages = 3;
};
// chunk position swizzle of stage row y (see above)
template <int FMT>
__device__ __forceinline__ uint32_t fwd_swz(uint32_t y) {
  return FMT == kFmtA8 ? ((y & 1u) << 2) : ((y & 3u) << 1);
}

__device__ __forceinline__ void mma_bf16_16816_zc(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ void mma_bf16_16816_acc(float (&d)[4], uint32_t a0, uint32_t a1,
                                                   uint32_t a2, uint32_t a3, uint32_t b0,
                                                   uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT, int FMT, bool G32>
__global__ void __launch_bounds__(kSrThreads, 2) smallr_fwd_kernel(const SrParams p) {
  using S = FwdShape<FMT>;
  constexpr int CW = S::kChunkU32;
  constexpr int KM = S::kMmas;
  constexpr int RB = S::kRowBytes;
  constexpr int SB = S::kStageBlocks;
  constexpr int STG = 16 * 128;      // one stage: 16 rows x 128 bytes
  constexpr int NSTG = S::kStages;
  constexpr int NP = G32 ? 2 : 1;    // group passes per block
  constexpr int NE = G32 ? SB : SB / 2;  // scale entries a lane loads per stage
  extern __shared__ __align__(1024) uint8_t sr_smem[];
  uint32_t* table = reinterpret_cast<uint32_t*>(sr_smem);
  fill_table<FMT>(table);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t I = p.I, O = p.O;
  const int64_t row0 = (int64_t)blockIdx.x * 128 + 16 * warp;
  const int KB = (int)(I / 64);
  const int kb_lo = (int)blockIdx.y * p.per_split;
  const int kb_hi = min(KB, kb_lo + p.per_split);
  const int nblk = kb_hi > kb_lo ? kb_hi - kb_lo : 0;
  const int nstage = (nblk + SB - 1) / SB;
  const uint32_t laneoff = (uint32_t)lane * 4u;
  const int64_t row_bytes = FMT == kFmtA8 ? I : I / 2;
  const float mu = (FMT == kFmtNF4 && !p.legacy) ? __ldg(p.mu) : 0.0f;
  const int glog = FMT == kFmtNF4 ? 0 : 31 - __clz(p.G);
  const uint8_t* ring = sr_smem + kTableBytes + warp * NSTG * STG;
  const uint32_t ring_s = smem_u32(ring);

  // This lane's copies of a stage: chunk c = lane % 8 of rows lane / 8 + 4 j
  // (block c * 16 / RB of the stage), stored at chunk c ^ swz(row).
  const int cch = lane & 7;
  const int cblk = cch * 16 / RB;
  const uint8_t* gsrc = p.codes + (row0 + (lane >> 3)) * row_bytes + (int64_t)kb_lo * RB + cch * 16;
  auto issue = [&](int st) {
    if (st < nstage && st * SB + cblk < nblk) {
      const uint32_t dst = ring_s + (uint32_t)((st % NSTG) * STG);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t y = (uint32_t)((lane >> 3) + 4 * j);
        cp_async16(dst + y * 128u + ((((uint32_t)cch) ^ fwd_swz<FMT>(y)) << 4),
                   gsrc + (int64_t)st * 128 + (int64_t)(4 * j) * row_bytes);
      }
    }
    cp_async_commit();  // one group per stage (empty past the end: uniform counting)
  };

  // Raw scale inputs of stage st: NF4 (q_b as float bits, t_g) of row
  // l % 16, blocks l / 16 + 2 e; affine (scale, bias), groups of 32: half
  // l / 16 of block e.
  const int64_t prow = row0 + (lane & 15);
  const int phalf = lane >> 4;
  auto load_params = [&](int st, float (&ra)[NE], float (&rb)[NE]) {
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      const int blk = st * SB + (G32 ? e : phalf + 2 * e);
      const bool ok = blk < nblk;
      if (FMT == kFmtNF4) {
        uint32_t q = 0xFFFFFFFFu;
        float tt = 0.0f;
        if (ok) nf4_scale_load(p, (uint32_t)(prow * KB + kb_lo + blk), q, tt);
        ra[e] = __uint_as_float(q);
        rb[e] = tt;
      } else {
        ra[e] = 0.0f;
        rb[e] = 0.0f;
        if (ok) {
          const int64_t gi = (prow * I + (int64_t)(kb_lo + blk) * 64 + (G32 ? 32 * phalf : 0)) >> glog;
          ra[e] = __ldg(p.scale + gi);
          rb[e] = __ldg(p.bias + gi);
        }
      }
    }
  };
  // activation rows of this lane: tokens g (n = 0) and 8 + g (n = 1)
  const bool tok_ok0 = g < p.R, tok_ok1 = (8 + g) < p.R;
  const __nv_bfloat16* xrow[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n)
    xrow[n] = p.act + (int64_t)(8 * n + g) * I + (int64_t)kb_lo * 64 + 16 * t;

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[n][c] = 0.0f;

  // prologue: NSTG - 1 stages in flight, the first stage's scale inputs
#pragma unroll
  for (int i = 0; i < NSTG - 1; ++i) issue(i);
  float ca[NE], cb[NE], na[NE], nb[NE];
  load_params(0, ca, cb);
  __syncthreads();  // the table is complete

  for (int st = 0; st < nstage; ++st) {
    issue(st + NSTG - 1);
    if (st + 1 < nstage) load_params(st + 1, na, nb);
    // activation lines two stages ahead into L1
#pragma unroll
    for (int jb = 0; jb < SB; ++jb) {
      const int bp = (st + 2) * SB + jb;
      if (bp < nblk) {
#pragma unroll
        for (int n = 0; n < NT; ++n)
          if (n == 0 ? tok_ok0 : tok_ok1)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(xrow[n] + (int64_t)bp * 64));
      }
    }
    cp_async_wait<NSTG - 1>();  // stage st has landed (this lane's copies)
    __syncwarp();               // ... and every lane's
    float sdec[NE];
    if (FMT == kFmtNF4) {
#pragma unroll
      for (int e = 0; e < NE; ++e) sdec[e] = nf4_scale_decode(__float_as_uint(ca[e]), cb[e], mu);
    }
    const uint8_t* stg = ring + (st % NSTG) * STG;
#pragma unroll
    for (int jb = 0; jb < SB; ++jb) {
      const int blkn = st * SB + jb;
      if (blkn >= nblk) break;
      // activation operand: 16 columns of tokens g, 8 + g as pairs
      uint32_t bx[NT][KM][2];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (n == 0 ? tok_ok0 : tok_ok1) {
          const uint4* xp = reinterpret_cast<const uint4*>(xrow[n] + (int64_t)blkn * 64);
          v0 = __ldg(xp);
          v1 = __ldg(xp + 1);
        }
        const uint32_t xw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        if (FMT == kFmtA8) {
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t w0 = xw[2 * m], w1 = xw[2 * m + 1];
            const uint32_t s0 = hmul2_bf16(w0, 0x41804180u), s1 = hmul2_bf16(w1, 0x41804180u);  // 16.0
            bx[n][2 * m][0] = prmt(w0, s0, 0x5410u);
            bx[n][2 * m][1] = prmt(w0, s0, 0x7632u);
            bx[n][2 * m + 1][0] = prmt(w1, s1, 0x5410u);
            bx[n][2 * m + 1][1] = prmt(w1, s1, 0x7632u);
          }
        } else {
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            bx[n][m][0] = xw[2 * m];
            bx[n][m][1] = xw[2 * m + 1];
          }
        }
      }
      // decoded pairs of rows g (pA) and g + 8 (pB): one per code byte
      uint32_t pA[4 * CW], pB[4 * CW];
      {
        uint32_t wa[CW], wb[CW];
        if (CW == 2) {
          // 8 bytes: block jb, columns 16 t .. (chunk 2 jb + t / 2, half t % 2)
          const uint32_t c = (uint32_t)(2 * jb + (t >> 1));
          const uint32_t off = (uint32_t)(t & 1) * 8u;
          const uint2 va = *reinterpret_cast<const uint2*>(stg + g * 128 + ((c ^ fwd_swz<FMT>(g)) << 4) + off);
          const uint2 vb = *reinterpret_cast<const uint2*>(stg + (g + 8) * 128 + ((c ^ fwd_swz<FMT>(g + 8)) << 4) + off);
          wa[0] = va.x; wa[CW - 1] = va.y;
          wb[0] = vb.x; wb[CW - 1] = vb.y;
        } else {
          // 16 bytes: block jb, columns 16 t .. (chunk 4 jb + t)
          const uint32_t c = (uint32_t)(4 * jb + t);
          const uint4 va = *reinterpret_cast<const uint4*>(stg + g * 128 + ((c ^ fwd_swz<FMT>(g)) << 4));
          const uint4 vb = *reinterpret_cast<const uint4*>(stg + (g + 8) * 128 + ((c ^ fwd_swz<FMT>(g + 8)) << 4));
          wa[0] = va.x; wa[1 % CW] = va.y; wa[2 % CW] = va.z; wa[3 % CW] = va.w;
          wb[0] = vb.x; wb[1 % CW] = vb.y; wb[2 % CW] = vb.z; wb[3 % CW] = vb.w;
        }
#pragma unroll
        for (int w = 0; w < CW; ++w)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            pA[4 * w + k] = tbl(table, wa[w], laneoff, k);
            pB[4 * w + k] = tbl(table, wb[w], laneoff, k);
          }
      }
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        // scale (and bias) of rows g and g + 8 for this block / group half:
        // from lane 16 q + row, entry jb (groups of 32), else lane
        // 16 (jb % 2) + row, entry jb / 2
        const int src = G32 ? 16 * q : 16 * (jb & 1);
        const int ent = G32 ? jb : (jb >> 1);
        float sA, sB, bA = 0.0f, bB = 0.0f;
        if (FMT == kFmtNF4) {
          sA = __shfl_sync(0xffffffffu, sdec[ent], src + g);
          sB = __shfl_sync(0xffffffffu, sdec[ent], src + 8 + g);
        } else {
          sA = __shfl_sync(0xffffffffu, ca[ent], src + g);
          sB = __shfl_sync(0xffffffffu, ca[ent], src + 8 + g);
          bA = __shfl_sync(0xffffffffu, cb[ent], src + g);
          bB = __shfl_sync(0xffffffffu, cb[ent], src + 8 + g);
        }
        const bool keep = !G32 || (t >> 1) == q;
        float D[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
          for (int j = 0; j < KM; ++j) {
            const uint32_t a0 = keep ? pA[2 * j] : 0u, a1 = keep ? pB[2 * j] : 0u;
            const uint32_t a2 = keep ? pA[2 * j + 1] : 0u, a3 = keep ? pB[2 * j + 1] : 0u;
            if (j == 0)
              mma_bf16_16816_zc(D[n], a0, a1, a2, a3, bx[n][j][0], bx[n][j][1]);
            else
              mma_bf16_16816_acc(D[n], a0, a1, a2, a3, bx[n][j][0], bx[n][j][1]);
          }
        }
        if (FMT == kFmtNF4) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            acc[n][0] = fmaf(sA, D[n][0], acc[n][0]);
            acc[n][1] = fmaf(sA, D[n][1], acc[n][1]);
            acc[n][2] = fmaf(sB, D[n][2], acc[n][2]);
            acc[n][3] = fmaf(sB, D[n][3], acc[n][3]);
          }
        } else {
          // sum of the activations over the group (ones operand: (1, 1)
          // pairs for 4-bit, (1, 0) for 8-bit, the x half only)
          const uint32_t one = keep ? (FMT == kFmtA8 ? 0x00003F80u : 0x3F803F80u) : 0u;
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            float xs[4];
#pragma unroll
            for (int j = 0; j < KM; ++j) {
              if (j == 0)
                mma_bf16_16816_zc(xs, one, one, one, one, bx[n][j][0], bx[n][j][1]);
              else
                mma_bf16_16816_acc(xs, one, one, one, one, bx[n][j][0], bx[n][j][1]);
            }
            acc[n][0] = fmaf(sA, D[n][0], fmaf(bA, xs[0], acc[n][0]));
            acc[n][1] = fmaf(sA, D[n][1], fmaf(bA, xs[1], acc[n][1]));
            acc[n][2] = fmaf(sB, D[n][2], fmaf(bB, xs[2], acc[n][2]));
            acc[n][3] = fmaf(sB, D[n][3], fmaf(bB, xs[3], acc[n][3]));
          }
        }
      }
    }
    __syncwarp();  // every lane is done with this slot before it is refilled
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      ca[e] = na[e];
      cb[e] = nb[e];
    }
  }
  cp_async_wait<0>();

  // ---- outputs of this warp: rows row0 + g (+ 8 for c2, c3), tokens 8 n + 2 t (+ 1)
  const bool single = p.splits == 1;
  if (single) griddep_wait();  // U comes from the launch before this one
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t row = row0 + g + 8 * (c >> 1);
      const int tok = 8 * n + 2 * t + (c & 1);
      if (tok >= p.R) continue;
      if (single) {
        float ad = 0.0f;
        for (int j = 0; j < p.r; ++j)
          ad = fmaf(__ldg(p.aux + (int64_t)tok * p.r + j), __ldg(p.lora + row * p.r + j), ad);
        p.out[(int64_t)tok * O + row] = __float2bfloat16_rn(fmaf(p.s, ad, acc[n][c]));
      } else {
        p.part[((int64_t)blockIdx.y * p.R + tok) * O + row] = acc[n][c];
      }
    }
  if (single) return;
  // ---- split-K: the last CTA of this 128-row tile sums the partials in order
  __shared__ unsigned s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    s_last = atomicAdd(&p.tickets[blockIdx.x], 1u) == (unsigned)(p.splits - 1) ? 1u : 0u;
  __syncthreads();
  if (!s_last) {
    if (threadIdx.x == 0) griddep_wait();
    return;
  }
  __threadfence();
  griddep_wait();
  const int64_t r0 = (int64_t)blockIdx.x * 128;
  for (int e = threadIdx.x; e < 128 * p.R; e += kSrThreads) {
    const int tok = e >> 7;
    const int64_t row = r0 + (e & 127);
    float v = 0.0f;
    for (int sp = 0; sp < p.splits; ++sp) v += __ldcg(p.part + ((int64_t)sp * p.R + tok) * O + row);
    float ad = 0.0f;
    for (int j = 0; j < p.r; ++j)
      ad = fmaf(__ldg(p.aux + (int64_t)tok * p.r + j), __ldg(p.lora + row * p.r + j), ad);
    p.out[(int64_t)tok * O + row] = __float2bfloat16_rn(fmaf(p.s, ad, v));
  }
  if (threadIdx.x == 0) p.tickets[blockIdx.x] = 0u;  // ready for the next call
}

// ------------------------------------------------------------ input gradient
//
// CTA: one 64-column block cb of W (the M side: 64 outputs of dX) x one
// range of W rows (split blockIdx.y), the rows split evenly over the 8
// warps.  A K step is 16 rows (4-bit) or 8 rows (8-bit).
//   4-bit: lane (g, t) reads bytes 4 g .. 4 g + 3 of the block (columns
//     8 g .. 8 g + 7) of rows o + 2t, o + 2t + 1, o + 2t + 8, o + 2t + 9; the
//     nibbles of two consecutive rows are interleaved into bytes
//     (w[o][c], w[o+1][c]) and looked up, giving the MMA pairs along K.
//   8-bit: bytes 8 g .. 8 g + 7 (columns 8 g .. 8 g + 7) of rows o + t and
//     o + t + 4; a byte's (lo, hi) pair is the K pair, met by (v, 16 v).
// M mapping (both): m-tile mt row g <-> column 8 g + 2 mt, row g + 8 <->
// column 8 g + 2 mt + 1.  The B operand is dY[token][row] times the row's
// scale for this block (NF4 s_hat, affine scale), rounded to bf16; the
// affine bias enters through a ones-operand MMA with dY * bias.
template <int FMT>
struct DxShape {
  static constexpr int kStepRows = FMT == kFmtA8 ? 8 : 16;
  static constexpr int kSteps = 4;  // K steps per loop iteration (loaded one iteration ahead)
};

template <int NT, int FMT, bool G32>
__global__ void __launch_bounds__(kSrThreads, FMT == kFmtNF4 ? 2 : 1) smallr_dx_kernel(const SrParams p) {
  using S = DxShape<FMT>;
  constexpr int SR = S::kStepRows, NS = S::kSteps;
  constexpr int RB = FMT == kFmtA8 ? 64 : 32;  // code bytes per row of the column block
  constexpr int STG = NS * SR * RB;            // one iteration: 2 KB
  constexpr int NSTG = 3;                      // iterations per warp ring
  extern __shared__ __align__(1024) uint8_t sr_smem[];
  uint32_t* table = reinterpret_cast<uint32_t*>(sr_smem);
  fill_table<FMT>(table);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t I = p.I, O = p.O;
  const int cb = blockIdx.x;  // 64-column block
  const int KB = (int)(I / 64);
  const int64_t row_bytes = FMT == kFmtA8 ? I : I / 2;
  const uint32_t laneoff = (uint32_t)lane * 4u;
  const float mu = (FMT == kFmtNF4 && !p.legacy) ? __ldg(p.mu) : 0.0f;
  constexpr int NP = G32 ? 2 : 1;
  uint8_t* ring = sr_smem + kTableBytes + warp * NSTG * STG;
  const uint32_t ring_s = smem_u32(ring);

  // rows of this CTA, then of this warp, in K steps
  const int64_t nsteps_all = O / SR;
  const int64_t st_lo = (int64_t)blockIdx.y * p.per_split;
  const int64_t st_hi = min(nsteps_all, st_lo + (int64_t)p.per_split);
  const int64_t cnt = st_hi > st_lo ? st_hi - st_lo : 0;
  const int64_t w_lo = st_lo + cnt * warp / 8, w_hi = st_lo + cnt * (warp + 1) / 8;
  const int nit = (int)((w_hi - w_lo + NS - 1) / NS);  // iterations of NS steps

  // Copy iteration i (NS steps x SR rows x RB bytes of column block cb)
  // into ring slot i % NSTG; rows past the warp's range are not copied.
  auto issue = [&](int i) {
    if (i < nit) {
      const int64_t r0 = (w_lo + (int64_t)i * NS) * SR;
      const int64_t rend = w_hi * SR;
      const uint32_t dst = ring_s + (uint32_t)((i % NSTG) * STG);
      constexpr int CPR = RB / 16;
#pragma unroll
      for (int j = 0; j < NS * SR * CPR / 32; ++j) {
        const int c = lane + 32 * j;
        const int row = c / CPR, ch = c % CPR;
        if (r0 + row < rend)
          cp_async16(dst + (uint32_t)(row * RB + ch * 16),
                     p.codes + (r0 + row) * row_bytes + (int64_t)cb * RB + ch * 16);
      }
    }
    cp_async_commit();
  };

  float acc[4][NT][4];
  float accb[NP][NT][4];  // affine bias term (same for every M row of a pass)
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][n][c] = 0.0f;
#pragma unroll
  for (int q = 0; q < NP; ++q)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) accb[q][n][c] = 0.0f;

  // rows of lane (g, t) within a step: 4-bit (2t, 2t+1) and (2t+8, 2t+9);
  // 8-bit t and t + 4
  auto step_row = [&](int i) -> int {
    if (FMT == kFmtA8) return t + 4 * i;
    return 2 * t + (i & 1) + 8 * (i >> 1);
  };
  // Per-row scale (and bias) for this column block: lane L holds row
  // st0 * SR + 32 k + L of the iteration's NS * SR rows.
  constexpr int PRL = NS * SR / 32;  // parameter rows per lane
  float ps[PRL][NP], pbv[PRL][NP], ns_[PRL][NP], nbv[PRL][NP];
  auto load_params = [&](float (&sv)[PRL][NP], float (&bv)[PRL][NP], int64_t st0) {
#pragma unroll
    for (int k = 0; k < PRL; ++k) {
      const int64_t row = st0 * SR + 32 * k + lane;
      const bool ok = row < w_hi * SR;
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        if (!ok) {
          sv[k][q] = 0.0f;
          bv[k][q] = 0.0f;
        } else if (FMT == kFmtNF4) {  // raw (q_b bits, t_g), decoded at use
          uint32_t qq;
          float tt;
          nf4_scale_load(p, (uint32_t)(row * KB + cb), qq, tt);
          sv[k][q] = __uint_as_float(qq);
          bv[k][q] = tt;
        } else {
          const int64_t gi = (row * I + (int64_t)cb * 64 + 32 * q) / p.G;
          sv[k][q] = __ldg(p.scale + gi);
          bv[k][q] = __ldg(p.bias + gi);
        }
      }
    }
  };
  // dY of the lane's K rows, tokens g and 8 + g, one iteration ahead:
  // 4-bit: the bf16 pair (row, row + 1); 8-bit: the row's bf16 in the low half
  uint32_t dy[NS][NT][2], dyn[NS][NT][2];
  auto load_dy = [&](uint32_t (&dst)[NS][NT][2], int64_t st0) {
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int tok = 8 * n + g;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int64_t st = st0 + s;
          const int64_t orow = st * SR + (FMT == kFmtA8 ? (t + 4 * hh) : (2 * t + 8 * hh));
          uint32_t v = 0u;
          if (tok < p.R && st < w_hi) {
            if (FMT == kFmtA8)
              v = (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p.act + (int64_t)tok * O + orow));
            else
              v = __ldg(reinterpret_cast<const uint32_t*>(p.act + (int64_t)tok * O + orow));
          }
          dst[s][n][hh] = v;
        }
      }
  };

#pragma unroll
  for (int i = 0; i < NSTG - 1; ++i) issue(i);
  if (nit > 0) {
    load_params(ps, pbv, w_lo);
    load_dy(dy, w_lo);
  }
  __syncthreads();  // the table is complete

  for (int it = 0; it < nit; ++it) {
    const int64_t st0 = w_lo + (int64_t)it * NS;
    const int64_t stn = st0 + NS;
    issue(it + NSTG - 1);
    if (stn < w_hi) {
      load_params(ns_, nbv, stn);
      load_dy(dyn, stn);
    }
    cp_async_wait<NSTG - 1>();
    __syncwarp();
    const uint8_t* stg = ring + (it % NSTG) * STG;
    // NF4: decode the block scales of the rows this lane loaded
    float sdec[PRL];
    if (FMT == kFmtNF4) {
#pragma unroll
      for (int k = 0; k < PRL; ++k) sdec[k] = nf4_scale_decode(__float_as_uint(ps[k][0]), pbv[k][0], mu);
    }
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int64_t st = st0 + s;
      if (st >= w_hi) break;
      // B operand: bf16 (dY * scale) for the lane's K rows, tokens g, 8 + g
      // 4-bit: pairs of rows (2t, 2t+1) -> b0, (2t+8, 2t+9) -> b1
      // 8-bit: (v, 16 v) of row t -> b0, of row t + 4 -> b1
      uint32_t bq[NP][NT][2], bb[NP][NT][2];
#pragma unroll
      for (int q = 0; q < NP; ++q) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // scale / bias of the rows this register covers, from the lanes
          // that loaded them (lane = row within the iteration mod 32)
          float sv0, sv1, bv0 = 0.0f, bv1 = 0.0f;
          const int rr0 = s * SR + (FMT == kFmtA8 ? (t + 4 * hh) : (2 * t + 8 * hh));
          {
            const int k0 = rr0 >> 5;
            const float vs = FMT == kFmtNF4 ? (k0 == 0 ? sdec[0] : sdec[PRL - 1])
                                            : (k0 == 0 ? ps[0][q] : ps[PRL - 1][q]);
            sv0 = __shfl_sync(0xffffffffu, vs, rr0 & 31);
            if (FMT != kFmtNF4) {
              const float vb = k0 == 0 ? pbv[0][q] : pbv[PRL - 1][q];
              bv0 = __shfl_sync(0xffffffffu, vb, rr0 & 31);
            }
          }
          if (FMT != kFmtA8) {
            const int rr1 = rr0 + 1;
            const int k1 = rr1 >> 5;
            const float vs = FMT == kFmtNF4 ? (k1 == 0 ? sdec[0] : sdec[PRL - 1])
                                            : (k1 == 0 ? ps[0][q] : ps[PRL - 1][q]);
            sv1 = __shfl_sync(0xffffffffu, vs, rr1 & 31);
            if (FMT != kFmtNF4) {
              const float vb = k1 == 0 ? pbv[0][q] : pbv[PRL - 1][q];
              bv1 = __shfl_sync(0xffffffffu, vb, rr1 & 31);
            }
          } else {
            sv1 = 0.0f;
          }
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const uint32_t pr = dy[s][n][hh];
            const float d0 = __uint_as_float(pr << 16);
            const float d1 = __uint_as_float(pr & 0xFFFF0000u);
            if (FMT == kFmtA8) {
              const float v = d0 * sv0;
              bq[q][n][hh] = pack_bf16x2(v, 16.0f * __bfloat162float(__float2bfloat16_rn(v)));
              bb[q][n][hh] = pack_bf16x2(d0 * bv0, 0.0f);
            } else {
              bq[q][n][hh] = pack_bf16x2(d0 * sv0, d1 * sv1);
              bb[q][n][hh] = FMT == kFmtNF4 ? 0u : pack_bf16x2(d0 * bv0, d1 * bv1);
            }
          }
        }
      }
      // A operand pairs: [m-tile][a0..a3] from the staged rows
      uint32_t A[4][4];
      const uint8_t* sbase = stg + s * SR * RB;
      if (FMT == kFmtA8) {
        // rows t (a0: M row g, a1: M row g + 8) and t + 4 (a2, a3); column
        // 8 g + 2 mt (+1 for M row g + 8) is byte 2 mt (+1) of the 8 bytes
        uint32_t w[2][2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint2 v = *reinterpret_cast<const uint2*>(sbase + step_row(i) * RB + 8 * g);
          w[i][0] = v.x;
          w[i][1] = v.y;
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int wi = mt >> 1, k = 2 * (mt & 1);
          A[mt][0] = tbl(table, w[0][wi], laneoff, k);
          A[mt][1] = tbl(table, w[0][wi], laneoff, k + 1);
          A[mt][2] = tbl(table, w[1][wi], laneoff, k);
          A[mt][3] = tbl(table, w[1][wi], laneoff, k + 1);
        }
      } else {
        // rows (2t, 2t+1) -> P1, (2t+8, 2t+9) -> P2; zip the nibbles so that
        // byte m of ze is (w[o][8g+2m], w[o+1][8g+2m]) and of zo the odd column
        uint32_t ze[2], zo[2];
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
          const uint32_t wa = *reinterpret_cast<const uint32_t*>(sbase + step_row(2 * pp) * RB + 4 * g);
          const uint32_t wb = *reinterpret_cast<const uint32_t*>(sbase + step_row(2 * pp + 1) * RB + 4 * g);
          ze[pp] = (wa & 0x0F0F0F0Fu) | ((wb << 4) & 0xF0F0F0F0u);
          zo[pp] = ((wa >> 4) & 0x0F0F0F0Fu) | (wb & 0xF0F0F0F0u);
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          A[mt][0] = tbl(table, ze[0], laneoff, mt);
          A[mt][1] = tbl(table, zo[0], laneoff, mt);
          A[mt][2] = tbl(table, ze[1], laneoff, mt);
          A[mt][3] = tbl(table, zo[1], laneoff, mt);
        }
      }
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        const bool keep = !G32 || (g >> 2) == q;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const uint32_t a0 = keep ? A[mt][0] : 0u, a1 = keep ? A[mt][1] : 0u;
          const uint32_t a2 = keep ? A[mt][2] : 0u, a3 = keep ? A[mt][3] : 0u;
#pragma unroll
          for (int n = 0; n < NT; ++n) mma_bf16_16816(acc[mt][n], a0, a1, a2, a3, bq[q][n][0], bq[q][n][1]);
        }
        if (FMT != kFmtNF4) {
          const uint32_t one = keep ? 0x3F803F80u : 0u;
#pragma unroll
          for (int n = 0; n < NT; ++n) mma_bf16_16816(accb[q][n], one, one, one, one, bb[q][n][0], bb[q][n][1]);
        }
      }
    }
    __syncwarp();  // every lane is done with this slot before it is refilled
    if (stn < w_hi) {
#pragma unroll
      for (int k = 0; k < PRL; ++k)
#pragma unroll
        for (int q = 0; q < NP; ++q) {
          ps[k][q] = ns_[k][q];
          pbv[k][q] = nbv[k][q];
        }
#pragma unroll
      for (int s = 0; s < NS; ++s)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          dy[s][n][0] = dyn[s][n][0];
          dy[s][n][1] = dyn[s][n][1];
        }
    }
  }
  cp_async_wait<0>();
  if (FMT != kFmtNF4) {  // the bias term belongs to every M row of its pass
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const bool mine = !G32 || (g >> 2) == q;
      if (!mine) continue;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[mt][n][c] += accb[q][n][c];
    }
  }

  // ---- combine the 8 warps (fixed order)
  __syncthreads();
  float* red = reinterpret_cast<float*>(sr_smem);  // [warp 1..7][mt][n][c][lane]
  constexpr int kSlab = 4 * NT * 4 * 32;
  if (warp > 0) {
    float* dst = red + (size_t)(warp - 1) * kSlab;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[((mt * NT + n) * 4 + c) * 32 + lane] = acc[mt][n][c];
  }
  __syncthreads();
  const bool single = p.splits == 1;
  if (warp == 0) {
    for (int k = 0; k < 7; ++k) {
      const float* src = red + (size_t)k * kSlab;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[mt][n][c] += src[((mt * NT + n) * 4 + c) * 32 + lane];
    }
    if (single) griddep_wait();  // V comes from the launches before this one
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t col = (int64_t)cb * 64 + 8 * g + 2 * mt + (c >> 1);
          const int tok = 8 * n + 2 * t + (c & 1);
          if (tok >= p.R) continue;
          if (single) {
            float ad = 0.0f;
            for (int j = 0; j < p.r; ++j)
              ad = fmaf(__ldg(p.aux + (int64_t)tok * p.r + j), __ldg(p.lora + (int64_t)j * I + col), ad);
            p.out[(int64_t)tok * I + col] = __float2bfloat16_rn(fmaf(p.s, ad, acc[mt][n][c]));
          } else {
            p.part[((int64_t)blockIdx.y * p.R + tok) * I + col] = acc[mt][n][c];
          }
        }
  }
  if (single) {
    if (threadIdx.x == 0) griddep_wait();
    return;
  }
  __shared__ unsigned s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    s_last = atomicAdd(&p.tickets[blockIdx.x], 1u) == (unsigned)(p.splits - 1) ? 1u : 0u;
  __syncthreads();
  if (!s_last) {
    if (threadIdx.x == 0) griddep_wait();
    return;
  }
  __threadfence();
  griddep_wait();
  const int64_t c0 = (int64_t)cb * 64;
  for (int e = threadIdx.x; e < 64 * p.R; e += kSrThreads) {
    const int tok = e >> 6;
    const int64_t col = c0 + (e & 63);
    float v = 0.0f;
    for (int sp = 0; sp < p.splits; ++sp) v += __ldcg(p.part + ((int64_t)sp * p.R + tok) * I + col);
    float ad = 0.0f;
    for (int j = 0; j < p.r; ++j)
      ad = fmaf(__ldg(p.aux + (int64_t)tok * p.r + j), __ldg(p.lora + (int64_t)j * I + col), ad);
    p.out[(int64_t)tok * I + col] = __float2bfloat16_rn(fmaf(p.s, ad, v));
  }
  if (threadIdx.x == 0) p.tickets[blockIdx.x] = 0u;
}

// ------------------------------------------------------------------ host

int sr_fmt(const WView& w) {
  if (w.fmt != QLORA_FMT_AFFINE) return kFmtNF4;
  return w.bits == 8 ? kFmtA8 : kFmtA4;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

struct SrPlan {
  int tiles;      // 128-row tiles (forward) or 64-column blocks (input gradient)
  int splits;
  int per_split;  // K blocks or K steps per split
};

// One wave: tiles x splits <= CTAs per SM x SMs (two CTAs per SM; one for
// the affine input-gradient variants, which take more registers); never a
// second, partial wave.
SrPlan sr_plan(bool dx, const WView& w) {
  SrPlan pl;
  const int per_sm = (!dx || sr_fmt(w) == kFmtNF4) ? 2 : 1;
  const int target = per_sm * num_sms();
  if (!dx) {
    pl.tiles = (int)(w.O / 128);
    const int KB = (int)(w.I / 64);
    int sp = target / pl.tiles;
    if (sp < 1) sp = 1;
    if (sp > KB / 4) sp = KB / 4 > 0 ? KB / 4 : 1;  // at least one block per K warp
    pl.per_split = (KB + sp - 1) / sp;
    pl.splits = (KB + pl.per_split - 1) / pl.per_split;
  } else {
    pl.tiles = (int)(w.I / 64);
    const int step = sr_fmt(w) == kFmtA8 ? 8 : 16;
    const int nst = (int)(w.O / step);
    int sp = target / pl.tiles;
    if (sp < 1) sp = 1;
    if (sp > nst / 8) sp = nst / 8 > 0 ? nst / 8 : 1;  // at least one step per warp
    pl.per_split = (nst + sp - 1) / sp;
    pl.splits = (nst + pl.per_split - 1) / pl.per_split;
  }
  return pl;
}

// Dynamic shared memory: the byte table plus the eight warps' rings of code
// (forward: 3 stages of 16 rows x 128 bytes; input gradient: 3 iterations
// of 64 rows (4-bit) or 32 rows (8-bit)).
constexpr int sr_smem_bytes(bool dx, int fmt) {
  (void)fmt;
  return kTableBytes + 8 * 3 * 2048;
}

template <int NT, int FMT, bool G32>
cudaError_t sr_launch(bool dx, const SrPlan& pl, const SrParams& p, cudaStream_t st) {
  auto kern = dx ? smallr_dx_kernel<NT, FMT, G32> : smallr_fwd_kernel<NT, FMT, G32>;
  const int smem = sr_smem_bytes(dx, FMT);
  static bool attr_fwd = false, attr_dx = false;
  bool& attr = dx ? attr_dx : attr_fwd;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.tiles, (unsigned)pl.splits);
  cfg.blockDim = dim3(kSrThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr1[1];
  attr1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr1[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr1;
  cfg.numAttrs = timing_enabled() ? 0 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int FMT, bool G32>
cudaError_t sr_launch_nt(bool dx, const SrPlan& pl, const SrParams& p, cudaStream_t st) {
  if (p.R <= 8) return sr_launch<1, FMT, G32>(dx, pl, p, st);
  return sr_launch<2, FMT, G32>(dx, pl, p, st);
}

cudaError_t sr_dispatch(bool dx, const WView& w, const SrParams& p, const SrPlan& pl,
                        cudaStream_t st) {
  const int f = sr_fmt(w);
  if (f == kFmtNF4) return sr_launch_nt<kFmtNF4, false>(dx, pl, p, st);
  const bool g32 = w.block == 32;
  if (f == kFmtA4) return g32 ? sr_launch_nt<kFmtA4, true>(dx, pl, p, st) : sr_launch_nt<kFmtA4, false>(dx, pl, p, st);
  return g32 ? sr_launch_nt<kFmtA8, true>(dx, pl, p, st) : sr_launch_nt<kFmtA8, false>(dx, pl, p, st);
}

SrParams sr_params(const WView& w, const void* act, int64_t R, const float* aux,
                   const float* lora, int32_t r, float s, void* out, void* ws, uint32_t* hdr,
                   unsigned* tickets, const SrPlan& pl) {
  SrParams p;
  p.codes = w.codes;
  p.qcodes = w.qcodes;
  p.t = w.t;
  p.mu = w.mu;
  p.scale = w.scale;
  p.bias = w.bias;
  p.legacy = w.fmt == QLORA_FMT_NF4_FP32SCALE ? 1 : 0;
  p.G = w.block;
  p.C = (uint32_t)(w.group < 1 ? 1 : w.group);
  p.c_shift = ((p.C & (p.C - 1)) == 0) ? __builtin_ctz(p.C) : -1;
  p.act = (const __nv_bfloat16*)act;
  p.R = (int32_t)R;
  p.O = w.O;
  p.I = w.I;
  p.aux = aux;
  p.lora = lora;
  p.r = r;
  p.s = s;
  p.out = (__nv_bfloat16*)out;
  p.part = (float*)ws;
  p.tickets = tickets + kTicketBase;
  p.splits = pl.splits;
  p.per_split = pl.per_split;
  p.err = hdr;
  return p;
}

}  // namespace

// Measured on one B200 (W 12288 x 4096 and 4096 x 4096, whole call in a
// CUDA graph, cold L2), against the tensor-core kernel: at one token the
// forward here is faster for NF4 (12288 x 4096: 17.1 vs 28.9 us), 4-bit
// affine codes (G = 64: 23.3 vs 30.0 us) and 8-bit codes in groups of 64
// or 128 (31.1 vs 31.4 us), the input gradient only for NF4 (23.9 vs
// 30.0 us; 4-bit affine G = 64: 36.3 vs 33.9 us); at 16 tokens the
// tensor-core kernel wins every case (NF4 forward 31.4 vs 29.6 us, input
// gradient 38.9 vs 31.4 us).  So this path is taken while one 8-token MMA
// tile covers the tokens, in those cases.
bool smallr_preferred(bool dx, const WView& w, int64_t R) {
  if (R > 8) return false;
  if (w.fmt == QLORA_FMT_AFFINE) return !dx && (w.bits == 4 || w.block >= 64);
  return true;
}

bool smallr_supported(const WView& w, int64_t R, const void* act, const void* out) {
  if (R < 1 || R > 16) return false;
  if (w.O < 128 || w.I < 64 || w.O % 128 != 0 || w.I % 64 != 0) return false;
  if (w.O > 65536 || w.I > 32768) return false;  // ticket ranges (see kTicketBase)
  if (((uintptr_t)w.codes % 16) != 0 || ((uintptr_t)act % 16) != 0 || ((uintptr_t)out % 4) != 0)
    return false;
  if (w.fmt == QLORA_FMT_NF4_DQ) return w.block == 64 && w.group >= 1;
  if (w.fmt == QLORA_FMT_NF4_FP32SCALE) return w.block == 64;
  if (w.fmt == QLORA_FMT_AFFINE)
    return (w.bits == 4 || w.bits == 8) && (w.block == 32 || w.block == 64 || w.block == 128);
  return false;
}

size_t smallr_ws(bool dx, const WView& w, int64_t R) {
  if (!smallr_supported(w, R, (const void*)16, (const void*)16)) return 0;
  const SrPlan pl = sr_plan(dx, w);
  if (pl.splits <= 1) return 0;
  const int64_t extent = dx ? w.I : w.O;
  return align_up((size_t)pl.splits * (size_t)R * (size_t)extent * 4, 256);
}

cudaError_t launch_smallr_fwd(const WView& w, const void* X, int64_t R, const float* U,
                              const float* B, int32_t r, float s, void* Y, void* ws,
                              uint32_t* hdr, unsigned* tickets, cudaStream_t st) {
  const SrPlan pl = sr_plan(false, w);
  const SrParams p = sr_params(w, X, R, U, B, r, s, Y, ws, hdr, tickets, pl);
  return sr_dispatch(false, w, p, pl, st);
}

cudaError_t launch_smallr_dx(const WView& w, const void* dY, int64_t R, const float* V,
                             const float* A, int32_t r, float s, void* dX, void* ws,
                             uint32_t* hdr, unsigned* tickets, cudaStream_t st) {
  const SrPlan pl = sr_plan(true, w);
  const SrParams p = sr_params(w, dY, R, V, A, r, s, dX, ws, hdr, tickets, pl);
  return sr_dispatch(true, w, p, pl, st);
}

}  // namespace qlora
