// tc_gemm.cu -- tcgen05 / TMEM kernels of the QLoRA linear layer (sm_100a).
//
// Forward  Y  = X W_hat^T + s U B^T     ("QLoRA Fine-Tuning", "Forward and
// Input    dX = dY W_hat + s V A         backward"; "QLoRA on Mac",
// gradient                               "Design / Q-LoRA layer")
//
// Packed codes arrive in shared memory by TMA, decoder warps turn each
// 64-weight block into bf16 in registers -- NF4: codebook level times the
// block scale (double-quantized, rebuilt from q_b, t_g and mu, or the
// legacy fp32 absmax); affine 4/8-bit: scale * code + bias of the code's
// group ("LoRA vs QLoRA on Apple Silicon", "Method") -- and write it where
// the tensor core reads it (TMEM rows, or 128-byte-swizzled shared-memory
// rows), and tcgen05.mma accumulates in TMEM.  The one exception: the input
// gradient from 2048 tokens on 256-token tiles decodes the weight once per
// call (expand_bf16_kernel, the same decode) into a bf16 copy in the
// call's workspace and reads that by TMA ("QLoRA: Fine-Tuning Under Memory
// Constraints", "Separate representation from arithmetic": fused or
// temporary dequantized tensors are the implementation's choice); the
// weight itself stays packed.
//
// Orientation: the decoded weight tile is the MMA "A" operand (M = 128
// weight-side rows: output features in the forward, input features in the
// input gradient) and the activation tile is the "B" operand (N = a tile of
// tokens, 16..256).  Small token counts therefore cost no wasted MMA rows,
// and the same kernel serves the bandwidth-bound and the tensor-bound
// regimes (split-K supplies parallelism when there are few tiles).
//   forward : A = W_hat[o, i] tile, K-major, decoded into TMEM
//   dX      : A = W_hat^T[i, o] tile, MN-major, decoded into shared memory
// A 64-weight NF4 block is one row of either tile, so one register decode
// serves both.
//
// The adapter term is the last K step of the same accumulation: its A
// operand is bf16(s B) (forward) or bf16(s A)^T (dX), zero-padded to 64
// along the rank, and its B operand is bf16 U or V, all loaded by TMA once
// the launch that computed them has finished (programmatic dependent
// launch: the K loop before it overlaps that launch).
//
// Tiles are taken in groups of up to 16 weight tiles, every token tile of
// a group before the next, so a wave's operands stay in L2.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer,
// then the decoders in groups of four warps (a whole 64-weight row per
// thread) that take K steps in turn: two groups (320 threads) up to
// 128-token tiles, four (576 threads) at 256-token tiles; the decoder warps
// then run the epilogue (TMEM -> registers -> shared memory -> TMA store).
// Every mbarrier wait is bounded (%globaltimer); on expiry the CTA records
// QLORA_ERR_TIMEOUT in the workspace header, stops issuing work, waits
// (bounded) for its copies in flight, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_gemm.h"

namespace qlora {

namespace {

constexpr int kBM = 128;             // weight-side rows per CTA (MMA M)
constexpr int kBK = 64;              // reduction step (one NF4 block)
// Decoder groups (group g decodes the K steps g, g + groups, ...): four at
// 256-token tiles (one CTA per SM), so that each group has four MMA steps'
// time for its tile decode (the decode is a dependent chain of ~200
// instructions per thread; with two groups it set the pace of the tensor
// pipe), except for the 8-bit input gradient, whose rings leave no room for
// the fourth decoded slot; two at smaller tiles, which keep two CTAs per SM.
#ifndef QLORA_TC_DEC_GROUPS_256
#define QLORA_TC_DEC_GROUPS_256 4
#endif
constexpr int dec_groups(bool dx, int bn, int pb) {
  return (bn >= 256 && !(dx && pb == 8) && pb != 16) ? QLORA_TC_DEC_GROUPS_256 : 2;
}
// Decoder warps per group: four, a whole 64-weight row per thread (a
// compile-time option gives eight at 256-token tiles, each thread decoding
// half a row; it measured no faster on the 8B / 14B / Qwen steps).
#ifndef QLORA_TC_DEC_WARPS_256
#define QLORA_TC_DEC_WARPS_256 4
#endif
constexpr int dec_warps(int bn) { return bn >= 256 ? QLORA_TC_DEC_WARPS_256 : 4; }
// epilogue groups: four warps each, one per TMEM lane quarter (the warps of
// the first two decoder groups)
constexpr int epi_groups(int bn) { return 2 * dec_warps(bn) / 4; }
constexpr int kWTile = kBM * kBK * 2;  // decoded weight tile bytes (16 KB)

struct TcParams {
  int64_t R;         // tokens
  int32_t Mw;        // weight-side extent (O forward, I input gradient)
  int32_t KB;        // reduction steps of 64
  int32_t I;         // W row length
  int32_t kb_per_split;
  int32_t r_slices;  // ceil(r / 16): MMA K=16 slices of the adapter step
  int32_t rank;      // r (for the algorithmic flop count only)
  uint32_t C;        // scale-group size in blocks
  int32_t c_shift;   // log2(C) when C is a power of two, else -1
  const uint8_t* qcodes;
  const float* t;
  const float* mu;
  const float* sb;   // legacy format: the fp32 block absmax s_b (else null)
  const float* asc;  // affine 4-bit: per-group scale (else null)
  const float* abi;  // affine 4-bit: per-group bias
  int32_t g_shift;   // affine: log2(G / 32), G in {32, 64, 128}
  int32_t pbits;     // code bits: 4, or 8 (affine)
  int32_t pre;       // the weight was decoded to bf16 before the launch (256-token tiles)
  void* out;         // bf16 [R x Mw], or fp32 partials [splits][R][Mw]
  int32_t partial;
  uint32_t* err;
  uint64_t wait_ns;
};

// K steps per TMA load of the token and packed tiles (see Cfg::G).
constexpr int tma_group(int bn) { return bn <= 16 ? 4 : bn <= 32 ? 2 : 1; }

constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
}

// Shared-memory and TMEM plan of one instantiation.
//   in ring  : NIN stages of {token tile [BN x 64] bf16, packed tile 4 KB},
//              filled by TMA, released by the MMA that consumed them
//   dec ring : NDEC decoded weight tiles, bf16 [128 x 64]; in TMEM (forward:
//              the MMA reads A from TMEM) or in shared memory (input
//              gradient: A is read MN-major through a descriptor)
//   adw      : the adapter step's A operand (16 KB, loaded once)
// Tiles of up to 128 tokens stay under half the SM's shared memory and TMEM
// so that two CTAs share an SM.
//   G        : K steps per TMA load (small token tiles: one load of the
//              token and packed tiles covers G ring slots, so the single
//              producer thread issues a few large copies, not many small ones)
//   adx      : with G > 1, the adapter step's token tile (U / V), outside
//              the ring
// bits per weight of a format's packed tile (WF 4: bf16, already decoded)
constexpr int wf_bits(int wf) { return wf == 4 ? 16 : wf == 3 ? 8 : 4; }

template <bool DX, int BN, int PB = 4>
struct Cfg {
  static constexpr int kAct = BN * kBK * 2;
  static constexpr int kPk = kBM * kBK * PB / 8;  // packed codes per step: 4 KB (4-bit), 8 KB (8-bit)
  static constexpr int G = tma_group(BN);
  // 8-bit codes double the packed tile: shallower rings keep the same
  // occupancy (two CTAs per SM below 256-token tiles)
  // PB 16: the weight tile is bf16 already (decoded once per call into the
  // workspace), 16 KB per step, no decoded-tile slots; 256-token tiles only
  static constexpr bool kPre = PB == 16;
  static constexpr int NIN = kPre ? 4
      : PB == 4
      ? (DX ? (BN >= 256 ? 4 : BN >= 128 ? 3 : BN >= 64 ? 5 : BN >= 32 ? 6 : 8)
            : (BN >= 256 ? 5 : BN >= 128 ? 4 : BN >= 64 ? 6 : BN >= 32 ? 8 : 12))
      : (DX ? (BN >= 256 ? 4 : BN >= 128 ? 2 : BN >= 64 ? 3 : 4)
            : (BN >= 256 ? 5 : BN >= 128 ? 3 : BN >= 64 ? 5 : BN >= 32 ? 6 : 8));
  static_assert(NIN % G == 0, "a TMA group fills whole ring slots");
  static constexpr int DG = dec_groups(DX, BN, PB);
  static constexpr int kThreads = 32 * (2 + DG * dec_warps(BN));
  static constexpr int NDEC4 = DX ? (BN >= 256 ? (DG > 3 ? DG : 3) : 2) : (BN >= 128 ? 4 : 6);
  static constexpr int NDEC = NDEC4 < NIN ? NDEC4 : NIN;
  static_assert(NDEC <= NIN, "decoded slots are released through the in-ring barriers");
  static_assert(DG <= NDEC && DG <= NIN, "one group's next step is at most one ring cycle on");
  static constexpr int kAccCols = BN < 32 ? 32 : BN;
  static constexpr int kTmemCols = pow2_at_least((DX || kPre) ? kAccCols : kAccCols + NDEC * 32);
  static constexpr int kWdec = (DX && !kPre) ? NDEC * kWTile : 0;
  static constexpr int kRing = NIN * (kAct + kPk) + kWdec;  // also the epilogue staging
  static constexpr int kAdx = G > 1 ? (kAct + 1023) / 1024 * 1024 : 0;
  static constexpr int kBars = 8 * (2 * NIN + NDEC + 2) + 16;
  static constexpr int kSmem = 1024 + kRing + kWTile + kAdx + kBars;
  static constexpr int kMinCtas = BN >= 256 ? 1 : 2;
  static_assert(kMinCtas == 1 || (kSmem <= 113 * 1024 && 2 * kTmemCols <= 512),
                "two CTAs per SM must fit");
  static_assert(kMinCtas == 2 || (kSmem <= 227 * 1024 && kTmemCols <= 512), "one CTA must fit");
  // more than 76 KB keeps a third CTA (and a third TMEM allocation) off the SM
  static_assert(kSmem > 76 * 1024, "at most two CTAs per SM");
};

// UMMA shared-memory descriptor, 128-byte swizzle (sm_100 version field).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// kind::f16 instruction descriptor: bf16 x bf16 -> fp32, B K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Decoding one 64-weight NF4 block with block scale s.
//
// The 16 possible outputs bf16(fp32(c[k] * s)) are formed once per block
// and kept in registers as two byte planes (low and high byte of each bf16,
// 4 entries per register); each group of 4 nibbles then selects its bytes
// with byte permutes: one permute per plane and per half of the table
// (nibble bits 0..2), one to pick the half (nibble bit 3) and two to
// interleave the planes back into bf16 pairs.  No shared-memory lookups.
struct Nf4Planes {
  uint32_t L0, L1, L2, L3, H0, H1, H2, H3;
};

__device__ __forceinline__ Nf4Planes nf4_planes(float s) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    P[j] = pack_bf16x2(__fmul_rn(kNF4[2 * j], s), __fmul_rn(kNF4[2 * j + 1], s));
  Nf4Planes t;
  t.L0 = __byte_perm(P[0], P[1], 0x6420); t.H0 = __byte_perm(P[0], P[1], 0x7531);
  t.L1 = __byte_perm(P[2], P[3], 0x6420); t.H1 = __byte_perm(P[2], P[3], 0x7531);
  t.L2 = __byte_perm(P[4], P[5], 0x6420); t.H2 = __byte_perm(P[4], P[5], 0x7531);
  t.L3 = __byte_perm(P[6], P[7], 0x6420); t.H3 = __byte_perm(P[6], P[7], 0x7531);
  return t;
}

// The same two byte planes for an affine group: the 16 values
// bf16(fp32(fp32(scale * k) + bias)), k = 0..15 ("LoRA vs QLoRA on Apple
// Silicon", "Method": w_hat = scale * code + bias, fp32, one rounding per
// step, as the diagnostic dequantization computes it).
__device__ __forceinline__ Nf4Planes affine_planes(float sc, float bi) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    P[j] = pack_bf16x2(__fadd_rn(__fmul_rn(sc, (float)(2 * j)), bi),
                       __fadd_rn(__fmul_rn(sc, (float)(2 * j + 1)), bi));
  Nf4Planes t;
  t.L0 = __byte_perm(P[0], P[1], 0x6420); t.H0 = __byte_perm(P[0], P[1], 0x7531);
  t.L1 = __byte_perm(P[2], P[3], 0x6420); t.H1 = __byte_perm(P[2], P[3], 0x7531);
  t.L2 = __byte_perm(P[4], P[5], 0x6420); t.H2 = __byte_perm(P[4], P[5], 0x7531);
  t.L3 = __byte_perm(P[6], P[7], 0x6420); t.H3 = __byte_perm(P[6], P[7], 0x7531);
  return t;
}

// 8 nibbles (weights 8j .. 8j+7, low nibble first) -> 4 bf16 pairs
// o[q] = (weight 2q, weight 2q+1) of the 8, low half first.
// A byte permute reads only the low 16 bits of its selector, so the
// selectors of both 4-nibble halves come from one pass over the word.
__device__ __forceinline__ void nf4_word(const Nf4Planes& t, uint32_t w, uint32_t (&o)[4]) {
  const uint32_t s7w = w & 0x77777777u;                            // table index, nibble bits 0..2
  const uint32_t sbw = ((w >> 1) & 0x44444444u) | 0x32103210u;     // bit 3 -> second half
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s7 = h ? (s7w >> 16) : s7w;
    const uint32_t sb = h ? (sbw >> 16) : sbw;
    const uint32_t alo = __byte_perm(t.L0, t.L1, s7), blo = __byte_perm(t.L2, t.L3, s7);
    const uint32_t ahi = __byte_perm(t.H0, t.H1, s7), bhi = __byte_perm(t.H2, t.H3, s7);
    const uint32_t lo = __byte_perm(alo, blo, sb), hi = __byte_perm(ahi, bhi, sb);
    o[2 * h] = __byte_perm(lo, hi, 0x5140);
    o[2 * h + 1] = __byte_perm(lo, hi, 0x7362);
  }
}

// Block (packed bytes 0..15 at pk_lo, 16..31 at pk_hi) -> one 128-byte
// swizzled shared-memory row at row_addr (row index within its 8-row atom
// = sw).  Weights 0..31 decode through table tA, 32..63 through tB (the
// same table unless an affine group of 32 splits the block).
__device__ __forceinline__ void decode_row_smem(const uint8_t* pk_lo, const uint8_t* pk_hi,
                                                const Nf4Planes& tA, const Nf4Planes& tB,
                                                uint32_t row_addr, uint32_t sw) {
  const uint4 p0 = *reinterpret_cast<const uint4*>(pk_lo);
  const uint4 p1 = *reinterpret_cast<const uint4*>(pk_hi);
  const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t o[4];
    nf4_word(j < 4 ? tA : tB, w[j], o);
    st_shared_v4(row_addr + ((j ^ sw) << 4), o[0], o[1], o[2], o[3]);
  }
}

// Half block (weights 32 h .. 32 h + 31 from the 16 packed bytes at pk) ->
// shared-memory chunks 4 h .. 4 h + 3 of the swizzled row at row_addr.
__device__ __forceinline__ void decode_half_smem(const uint8_t* pk, const Nf4Planes& t,
                                                 uint32_t row_addr, uint32_t sw, int h) {
  const uint4 p = *reinterpret_cast<const uint4*>(pk);
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t o[4];
    nf4_word(t, w[j], o);
    st_shared_v4(row_addr + ((((uint32_t)(4 * h + j)) ^ sw) << 4), o[0], o[1], o[2], o[3]);
  }
}

// Half block -> 16 registers, v[c] = (weight 32 h + 2c, 32 h + 2c + 1):
// TMEM columns 16 h .. 16 h + 15 of the row.
__device__ __forceinline__ void decode_half_regs(const uint8_t* pk, const Nf4Planes& t,
                                                 uint32_t (&v)[16]) {
  const uint4 p = *reinterpret_cast<const uint4*>(pk);
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t o[4];
    nf4_word(t, w[j], o);
    v[4 * j] = o[0];
    v[4 * j + 1] = o[1];
    v[4 * j + 2] = o[2];
    v[4 * j + 3] = o[3];
  }
}

// Block -> 32 registers, v[c] = (weight 2c, weight 2c+1): one TMEM row of
// the A operand (32 columns of two bf16 each); tables as decode_row_smem.
__device__ __forceinline__ void decode_row_regs(const uint8_t* pk_lo, const uint8_t* pk_hi,
                                                const Nf4Planes& tA, const Nf4Planes& tB,
                                                uint32_t (&v)[32]) {
  const uint4 p0 = *reinterpret_cast<const uint4*>(pk_lo);
  const uint4 p1 = *reinterpret_cast<const uint4*>(pk_hi);
  const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t o[4];
    nf4_word(j < 4 ? tA : tB, w[j], o);
    v[4 * j] = o[0];
    v[4 * j + 1] = o[1];
    v[4 * j + 2] = o[2];
    v[4 * j + 3] = o[3];
  }
}

// 8-bit affine codes: weight = fp32(fp32(scale * q) + bias) ("LoRA vs QLoRA
// on Apple Silicon", "Method"; the diagnostic dequantization's arithmetic),
// the code byte placed in the mantissa of 2^23 and the 2^23 subtracted
// (exact), two weights packed per bf16 pair.
__device__ __forceinline__ float aff8_weight(uint32_t w, int k, float sc, float bi) {
  uint32_t m;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m) : "r"(w), "r"(0x4B000000u), "r"(0x7540u | (uint32_t)k));
  const float q = __fsub_rn(__uint_as_float(m), 8388608.0f);
  return __fadd_rn(__fmul_rn(sc, q), bi);
}
// 16 code bytes (weights 16 c .. 16 c + 15) -> 8 bf16 pairs
__device__ __forceinline__ void aff8_chunk(uint4 c, float sc, float bi, uint32_t (&o)[8]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    o[2 * j] = pack_bf16x2(aff8_weight(w[j], 0, sc, bi), aff8_weight(w[j], 1, sc, bi));
    o[2 * j + 1] = pack_bf16x2(aff8_weight(w[j], 2, sc, bi), aff8_weight(w[j], 3, sc, bi));
  }
}
// Forward, 8-bit: the row's 64 bytes as TMA wrote them (64-byte swizzle:
// chunk c at c ^ x), chunks c0 .. c0 + nc - 1 -> v[8 (c - c0) ..], weights
// 0..31 with (sc0, bi0), 32..63 with (sc1, bi1).
template <int NC>
__device__ __forceinline__ void aff8_regs(const uint8_t* row, uint32_t x, int c0, float sc0, float bi0,
                                          float sc1, float bi1, uint32_t (&v)[8 * NC]) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int cc = c0 + c;
    const uint4 p = *reinterpret_cast<const uint4*>(row + ((((uint32_t)cc) ^ x) << 4));
    uint32_t o[8];
    aff8_chunk(p, cc < 2 ? sc0 : sc1, cc < 2 ? bi0 : bi1, o);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[8 * c + j] = o[j];
  }
}
// Input gradient, 8-bit: the unit's 64 bytes are chunks 4 h .. 4 h + 3 of a
// 128-byte row (128-byte swizzle: chunk c at c ^ y7); chunks cl .. cl + nc - 1
// of the unit decode into output chunks 2 cl .. of the swizzled decoded row.
template <int NC>
__device__ __forceinline__ void aff8_smem(const uint8_t* row, uint32_t y7, int h, int cl, float sc0,
                                          float bi0, float sc1, float bi1, uint32_t row_addr,
                                          uint32_t sw) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int cc = cl + c;  // 0..3 within the unit
    const uint4 p = *reinterpret_cast<const uint4*>(row + ((((uint32_t)(4 * h + cc)) ^ y7) << 4));
    uint32_t o[8];
    aff8_chunk(p, cc < 2 ? sc0 : sc1, cc < 2 ? bi0 : bi1, o);
    st_shared_v4(row_addr + ((((uint32_t)(2 * cc)) ^ sw) << 4), o[0], o[1], o[2], o[3]);
    st_shared_v4(row_addr + ((((uint32_t)(2 * cc + 1)) ^ sw) << 4), o[4], o[5], o[6], o[7]);
  }
}

// The whole weight decoded to bf16 once per call, for the 256-token path:
// thread b decodes 64-weight block b with the same tables and arithmetic as
// the in-GEMM decoders (bit-identical values), 32 or 64 code bytes in, 128
// bytes out.
template <int WF>
__global__ void __launch_bounds__(256) expand_bf16_kernel(const TcParams p, const uint8_t* codes,
                                                          int64_t nblocks, uint4* out) {
  const int64_t b = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (b >= nblocks) return;
  uint32_t v[32];
  if (WF == 3) {
    const uint32_t g0 = (uint32_t)((2 * b) >> p.g_shift), g1 = (uint32_t)((2 * b + 1) >> p.g_shift);
    aff8_regs<4>(codes + 64 * b, 0u, 0, __ldg(p.asc + g0), __ldg(p.abi + g0), __ldg(p.asc + g1),
                 __ldg(p.abi + g1), v);
  } else {
    Nf4Planes tA, tB;
    if (WF == 2) {
      const uint32_t g0 = (uint32_t)((2 * b) >> p.g_shift), g1 = (uint32_t)((2 * b + 1) >> p.g_shift);
      tA = affine_planes(__ldg(p.asc + g0), __ldg(p.abi + g0));
      tB = g1 == g0 ? tA : affine_planes(__ldg(p.asc + g1), __ldg(p.abi + g1));
    } else {
      float sc;
      if (WF == 1) {
        sc = __ldg(p.sb + b);
      } else {
        const uint32_t g = p.c_shift >= 0 ? (uint32_t)(b >> p.c_shift) : (uint32_t)(b / p.C);
        sc = decode_block_scale(__ldg(p.qcodes + b), __ldg(p.t + g), __ldg(p.mu));
      }
      tA = nf4_planes(sc);
      tB = tA;
    }
    decode_row_regs(codes + 32 * b, codes + 32 * b + 16, tA, tB, v);
  }
  uint4* dst = out + 8 * b;
#pragma unroll
  for (int j = 0; j < 8; ++j) dst[j] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

// TMA bulk tensor store of a shared-memory box (3D map: weight-side
// column, token, split); coordinates past the tensor edge are not written.
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int32_t x, int32_t y,
                                             int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(tmap),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_and_wait_read() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// TMEM accumulator columns [c_begin, c_end) (tokens) of this warp's 32
// lanes (weight-side rows 32*quad + lane) -> the group's staging area `ep`
// laid out as two boxes [ncols tokens][64 weight-side columns] (rows 0..63
// and 64..127 of the tile), bf16 outputs or fp32 split-K partials.
template <bool PARTIAL>
__device__ __forceinline__ void epilogue_stage(uint32_t tmem, int quad, int lane, int c_begin,
                                               int c_end, int ncols, uint8_t* ep) {
  constexpr int ES = PARTIAL ? 4 : 2;
  const int half = quad >> 1, col64 = (quad & 1) * 32 + lane;
  uint8_t* base = ep + ((size_t)half * ncols * 64 + col64) * ES;
#pragma unroll 1
  for (int c0 = c_begin; c0 < c_end; c0 += 32) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c0, v);
    tmem_ld_wait();
    uint8_t* dst = base + (size_t)(c0 - c_begin) * 64 * ES;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (c0 + j < c_end) {
        if (PARTIAL)
          *reinterpret_cast<uint32_t*>(dst) = v[j];
        else
          *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(__uint_as_float(v[j]));
      }
      dst += 64 * ES;
    }
  }
}

// Columns of the token tile each epilogue group stores.
template <int BN>
constexpr int cols_per_group() {
  return BN >= 64 ? BN / epi_groups(BN) : BN;
}

// WF: weight format, a template parameter so the decoder loop carries no
// format branches (0 NF4 double-quant, 1 NF4 legacy fp32 scales, 2 affine
// 4-bit, 3 affine 8-bit, 4 weights decoded to bf16 before the launch)
template <bool DX, int BN, int WF>
__global__ void __launch_bounds__(Cfg<DX, BN, wf_bits(WF)>::kThreads,
                                  Cfg<DX, BN, wf_bits(WF)>::kMinCtas)
    tc_qlinear_kernel(const __grid_constant__ CUtensorMap tm_act,
                      const __grid_constant__ CUtensorMap tm_pk,
                      const __grid_constant__ CUtensorMap tm_aact,
                      const __grid_constant__ CUtensorMap tm_aw,
                      const __grid_constant__ CUtensorMap tm_out, const TcParams p) {
  using C = Cfg<DX, BN, wf_bits(WF)>;
  constexpr int NIN = C::NIN, NDEC = C::NDEC;
  constexpr uint32_t kIdesc = idesc_bf16(kBM, BN, DX);
  constexpr int DW = dec_warps(BN);
  constexpr int DG = C::DG;
  static_assert((BN >= 64 ? epi_groups(BN) : 1) * 2 * cols_per_group<BN>() * 64 * 4 <= C::kRing,
                "epilogue staging must fit in the ring buffers");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* act = smem;                        // NIN x BN*128
  uint8_t* pk = act + NIN * C::kAct;          // NIN x 4 KB (4-bit) or 8 KB (8-bit)
  uint8_t* wdec = pk + NIN * C::kPk;          // input gradient: NDEC x 16 KB
  uint8_t* adw = wdec + C::kWdec;             // 16 KB
  uint8_t* adx = adw + kWTile;                // G > 1: adapter token tile
  uint64_t* bars = (uint64_t*)(adx + C::kAdx);
  uint64_t* full_in = bars;                   // TMA landed (on the group's first slot)
  uint64_t* in_empty = bars + NIN;            // MMA done with the step of this stage
  uint64_t* dec_full = bars + 2 * NIN;        // decoded tile written (4 warps)
  uint64_t* acc_full = bars + 2 * NIN + NDEC;
  uint64_t* ad_full = acc_full + 1;           // G > 1: adapter operands landed
  volatile uint32_t* tmem_slot = (volatile uint32_t*)(ad_full + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Tile order: CTAs go in groups of up to kGroupM weight tiles, sweeping
  // every token tile of the group before the next group starts, so that a
  // wave's weight slabs and token tiles both stay in L2 (with the plain
  // order every wave re-read the whole weight; for a bf16 weight copy larger
  // than L2 that came from DRAM every time).
  int mt, nt;
  {
    constexpr int64_t kGroupM = 16;
    const int64_t MT = gridDim.x, NT = gridDim.y;
    const int64_t lin = (int64_t)blockIdx.y * MT + blockIdx.x;
    const int64_t per_group = kGroupM * NT;
    const int64_t first = (lin / per_group) * kGroupM;
    const int64_t gsz = MT - first < kGroupM ? MT - first : kGroupM;
    const int64_t r = lin % per_group;
    mt = (int)(first + r % gsz);
    nt = (int)(r / gsz);
  }
  const int m0 = mt * kBM;
  const int64_t n0 = (int64_t)nt * BN;
  const int split = blockIdx.z;
  const int kb_lo = split * p.kb_per_split;
  const int kb_hi = min(p.KB, kb_lo + p.kb_per_split);
  const int nk = kb_hi - kb_lo;               // weight K steps of this CTA (+ the adapter
                                              // step, last, in split 0)

  if (threadIdx.x == 0) {
    // A kernel queued behind this one with a programmatic dependency (the
    // split-K reduction) may start now; it waits for this grid itself.
    griddep_launch_dependents();
    for (int s = 0; s < NIN; ++s) {
      mbar_init(smem_u32(&full_in[s]), 1);
      mbar_init(smem_u32(&in_empty[s]), 1);
    }
    for (int d = 0; d < NDEC; ++d) {
      mbar_init(smem_u32(&dec_full[d]), DW);  // the warps of one decoder group
    }
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(ad_full), 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_act);
    prefetch_tensormap(&tm_pk);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      constexpr int G = C::G;
      int issued = 0;  // K steps whose copies were issued
      bool ad_issued = false;
      int s0 = 0;          // first slot of the group (running)
      uint32_t ph = 0;     // ring cycle parity of the group
      for (int it0 = 0; it0 < nk; it0 += G) {
        const int sl = s0 + G - 1;  // group = slots s0 .. sl
        if ((it0 & (8 * G - 1)) == 0 && *abort_flag) break;
        if (!mbar_wait(smem_u32(&in_empty[sl]), ph ^ 1u, p.wait_ns, p.err, 0x101)) {
          *abort_flag = 1;
          break;
        }
        const uint32_t fb = smem_u32(&full_in[s0]);
        const int kb = kb_lo + it0;
        mbar_arrive_expect_tx(fb, G * (C::kAct + C::kPk));
        tma_load_3d(smem_u32(act + s0 * C::kAct), &tm_act, fb, 0, (int32_t)n0, kb);
        if (!DX) {
          tma_load_3d(smem_u32(pk + s0 * C::kPk), &tm_pk, fb, 0, m0, kb);
        } else if (WF == 4) {  // W^T tile, MN-major: two 64-column boxes
          tma_load_3d(smem_u32(pk + s0 * C::kPk), &tm_pk, fb, m0, 0, kb);
          tma_load_3d(smem_u32(pk + s0 * C::kPk + kWTile / 2), &tm_pk, fb, m0 + 64, 0, kb);
        } else {
          tma_load_3d(smem_u32(pk + s0 * C::kPk), &tm_pk, fb, WF == 3 ? m0 : m0 / 2, 0, kb);
        }
        issued = it0 + G;
        s0 += G;
        if (s0 == NIN) { s0 = 0; ph ^= 1u; }
      }
      if (split == 0 && !*abort_flag) {
        // Adapter step: U / V and the scaled factor come from the launch
        // just before this one, which may still be running.
        uint32_t fb, a_dst;
        bool ok = true;
        if (G > 1) {
          fb = smem_u32(ad_full);
          a_dst = smem_u32(adx);
        } else {
          const int s = nk % NIN;  // G == 1 here: s0 == s, ph its cycle
          ok = mbar_wait(smem_u32(&in_empty[s]), ph ^ 1u, p.wait_ns, p.err, 0x102);
          fb = smem_u32(&full_in[s]);
          a_dst = smem_u32(act + s * C::kAct);
        }
        if (!ok) {
          *abort_flag = 1;
        } else {
          griddep_wait();
          mbar_arrive_expect_tx(fb, C::kAct + kWTile);
          tma_load_2d(a_dst, &tm_aact, fb, 0, (int32_t)n0);
          if (!DX) {
            tma_load_2d(smem_u32(adw), &tm_aw, fb, 0, m0);
          } else {
            tma_load_2d(smem_u32(adw), &tm_aw, fb, m0, 0);
            tma_load_2d(smem_u32(adw + kWTile / 2), &tm_aw, fb, m0 + 64, 0);
          }
          if (G > 1) ad_issued = true;
          else issued = nk + 1;
        }
      }
      if (*abort_flag) {  // let copies in flight land before the CTA exits
        const int first = issued - NIN < 0 ? 0 : issued - NIN;
        for (int it = first - first % G; it < issued; it += G)
          mbar_wait(smem_u32(&full_in[it % NIN]), (it / NIN) & 1, p.wait_ns, nullptr, 0);
        if (ad_issued) mbar_wait(smem_u32(ad_full), 0, p.wait_ns, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // The loop is one thread's dependent chain, so it keeps it short:
    // running ring positions instead of divisions, descriptors built once,
    // both barriers tested together (the bounded blocking wait only when a
    // test fails), the abort flag read every eighth step.
    if (lane == 0) {
      constexpr int G = C::G;
      const uint32_t act0 = smem_u32(act);
      const uint64_t bdesc0 = sdesc(act0, 16, 1024);
      const uint64_t adesc0 = sdesc(smem_u32(wdec), 8192, 1024);
      const uint32_t pk_s0 = smem_u32(pk);
      int s = 0, d = 0;
      uint32_t ph_in = 0, ph_dec = 0;
      bool ok = true;
      for (int it = 0; it < nk; ++it) {
        if ((it & 7) == 0 && *abort_flag) { ok = false; break; }
        // The decoders waited for this step's TMA group (token and packed
        // tiles land on the same barrier) before they arrived on dec_full,
        // so dec_full alone orders the MMA after both copies.
        // pre-decoded weights: the step's TMA group (both operands) is
        // all the MMA waits for; otherwise the decoded tile
        const uint32_t db = WF == 4 ? smem_u32(&full_in[s - s % G]) : smem_u32(&dec_full[d]);
        if (!mbar_wait(db, WF == 4 ? ph_in : ph_dec, p.wait_ns, p.err, 0x202)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bd = bdesc0 + (uint64_t)((uint32_t)(s * C::kAct) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          if (WF == 4) {
            const uint32_t a_s = pk_s0 + (uint32_t)(s * C::kPk);
            if (!DX)  // W tile K-major (128-byte rows, 128-byte swizzle)
              umma_bf16(tmem, sdesc(a_s, 16, 1024) + 2 * kk, bd + 2 * kk, kIdesc, acc);
            else      // W^T tile MN-major, as the decoded tile below
              umma_bf16(tmem, sdesc(a_s, 8192, 1024) + (uint64_t)((uint32_t)(kk * 2048) >> 4),
                        bd + 2 * kk, kIdesc, acc);
          } else if (!DX) {
            umma_bf16_ta(tmem, tmem + (uint32_t)(C::kAccCols + d * 32 + kk * 8), bd + 2 * kk,
                         kIdesc, acc);
          } else {
            umma_bf16(tmem, adesc0 + (uint64_t)((uint32_t)(d * kWTile + kk * 2048) >> 4),
                      bd + 2 * kk, kIdesc, acc);
          }
        }
        umma_commit(smem_u32(&in_empty[s]));  // frees the in-ring stage and, NDEC steps on, the decoded slot
        if (++s == NIN) { s = 0; ph_in ^= 1u; }
        if (++d == NDEC) { d = 0; ph_dec ^= 1u; }
      }
      if (ok && split == 0) {  // adapter step (s is now nk % NIN)
        const uint32_t fb = G > 1 ? smem_u32(ad_full) : smem_u32(&full_in[s]);
        const uint32_t b0 = G > 1 ? smem_u32(adx) : act0 + (uint32_t)(s * C::kAct);
        if (*abort_flag || !mbar_wait(fb, G > 1 ? 0u : ph_in, p.wait_ns, p.err, 0x203)) {
          *abort_flag = 1;
        } else {
          tc_fence_after();
          const uint32_t a0 = smem_u32(adw);
          for (int kk = 0; kk < p.r_slices; ++kk) {
            const uint64_t ad = DX ? sdesc(a0 + kk * 2048, 8192, 1024) : sdesc(a0 + kk * 32, 16, 1024);
            umma_bf16(tmem, ad, sdesc(b0 + kk * 32, 16, 1024), kIdesc, (nk > 0 || kk > 0) ? 1u : 0u);
          }
        }
      }
      umma_commit(smem_u32(acc_full));
    }
    __syncwarp();
  } else if (WF == 4) {
    // weights decoded before the launch: the decoder warps only run the
    // epilogue, once the accumulator is complete
    if (!mbar_wait(smem_u32(acc_full), 0, p.wait_ns, p.err, 0x401)) *abort_flag = 1;
  } else {
    // ------------------------------------------------------------ decoders
    // DG groups of DW warps; group g decodes the steps it = g, g + DG, ...
    // Forward: the thread decodes weight row 32*(warp%4) + lane, its own
    // TMEM lane, and stores the block's 32 bf16 pairs with one tcgen05.st.
    // Input gradient: unit u writes one swizzled 128-byte row of the
    // MN-major shared-memory tile (64 weights of W row kb*64 + u%64).
    // With eight warps per group, warps wi and wi + 4 of the group share the
    // rows (units) and take the low (half 0) and high (half 1) 32 weights.
    const int group = (warp - 2) / DW;
    const int wi = (warp - 2) % DW;
    const int half = wi >> 2;  // always 0 with four warps per group
    const int quad = warp & 3;
    const int u = DX ? (((int)threadIdx.x - 64 - 32 * DW * group) & 127) : 32 * quad + lane;
    constexpr bool legacy = WF == 1;  // fp32 block scales stored as they are
    constexpr bool affine = WF >= 2;  // affine groups: (scale, bias); WF 3: 8-bit codes
    const float mu = (legacy || affine) ? 0.0f : __ldg(p.mu);
    const uint32_t bpr = (uint32_t)(p.I / kBK);  // blocks per W row
    auto block_of = [&](int kb) -> uint32_t {
      if (!DX) return (uint32_t)(m0 + u) * bpr + (uint32_t)kb;
      return (uint32_t)(kb * kBK + (u & 63)) * bpr + (uint32_t)(m0 / kBK) + (uint32_t)(u >> 6);
    };
    // scale group of block b (a shift when the group size is a power of two)
    auto group_of = [&](uint32_t b) -> uint32_t {
      return p.c_shift >= 0 ? (b >> p.c_shift) : b / p.C;
    };
    // affine group of the first weight this thread decodes in block b (32
    // weights per half block: group (2 b + half) >> log2(G / 32))
    auto agroup_of = [&](uint32_t b) -> uint32_t { return (2u * b + (uint32_t)half) >> p.g_shift; };
    // Per step: NF4 (q_b, t_g); legacy (-, s_b); affine (scale bits, bias).
    auto load_scale = [&](uint32_t b, uint32_t& q, float& t) {
      if (affine) {
        const uint32_t gi = agroup_of(b);
        q = __float_as_uint(__ldg(p.asc + gi));
        t = __ldg(p.abi + gi);
      } else if (legacy) {
        t = __ldg(p.sb + b);
      } else {
        q = __ldg(p.qcodes + b);
        t = __ldg(p.t + group_of(b));
      }
    };
    const uint32_t row_off = (uint32_t)((u >> 6) * (kWTile / 2) + (u & 63) * 128);
    const uint32_t sw = (uint32_t)(u & 7);
    // Packed tile as TMA wrote it: forward 128 rows x 32 B with the 32-byte
    // swizzle (16-byte half c of row y at c ^ bit 2 of y), input gradient
    // 64 rows x 64 B with the 64-byte swizzle (chunk c of row y at
    // c ^ bits 1..2 of y).  Eight consecutive lanes then hit eight
    // different bank groups.
    uint32_t pk_lo, pk_hi;
    if (!DX) {
      const uint32_t x = (uint32_t)(u >> 2) & 1u;
      pk_lo = (uint32_t)u * 32 + ((0u ^ x) << 4);
      pk_hi = (uint32_t)u * 32 + ((1u ^ x) << 4);
    } else {
      const uint32_t o = (uint32_t)(u & 63), h = (uint32_t)(u >> 6), x = (o >> 1) & 3u;
      pk_lo = o * 64 + (((2 * h) ^ x) << 4);
      pk_hi = o * 64 + (((2 * h + 1) ^ x) << 4);
    }
    const uint32_t tm_row = tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)C::kAccCols;
    // Scale inputs (q_b, t_g) of this group's next kPf steps are in flight
    // while it decodes: a rotating window of loads kPf steps ahead hides
    // the global-memory latency behind kPf tile decodes.
    constexpr int kPf = 4;
    uint32_t qw[kPf];
    float tw[kPf];
#pragma unroll
    for (int j = 0; j < kPf; ++j) {
      const int itj = group + j * DG;
      qw[j] = 128u;
      tw[j] = 0.0f;
      if (itj < nk) load_scale(block_of(kb_lo + itj), qw[j], tw[j]);
    }
    bool ok = true;
    // running ring positions of this group's steps (it = group, group + DG, ...)
    int s = group % NIN, d = group % NDEC;
    uint32_t ph_in = 0;
    for (int it = group; it < nk; it += DG) {
      const float sc = affine ? __uint_as_float(qw[0]) : legacy ? tw[0] : decode_block_scale(qw[0], tw[0], mu);
      const float bi = tw[0];  // affine bias
      const uint32_t bcur = block_of(kb_lo + it);
#pragma unroll
      for (int j = 0; j + 1 < kPf; ++j) {
        qw[j] = qw[j + 1];
        tw[j] = tw[j + 1];
      }
      {
        const int itn = it + kPf * DG;
        if (itn < nk) load_scale(block_of(kb_lo + itn), qw[kPf - 1], tw[kPf - 1]);
      }
      if (((it >> 1) & 3) == 0 && __any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      // Decoded slot d was last used by step it - NDEC; the MMA releases a
      // step by committing to its in-ring stage barrier (NDEC <= NIN, so
      // that barrier cannot have moved on by a further phase yet).
      const uint32_t fb = smem_u32(&full_in[s - s % C::G]);
      uint32_t eb = 0, ep = 0;
      if (it >= NDEC) {
        const int j = it - NDEC;
        eb = smem_u32(&in_empty[j % NIN]);
        ep = (uint32_t)((j / NIN) & 1);
      }
      bool w_ok = mbar_test(fb, ph_in) & (eb == 0 || mbar_test(eb, ep));
      if (!w_ok)
        w_ok = (eb == 0 || mbar_wait(eb, ep, p.wait_ns, p.err, 0x301)) &&
               mbar_wait(fb, ph_in, p.wait_ns, p.err, 0x302);
      if (!__all_sync(0xffffffffu, w_ok)) { *abort_flag = 1; ok = false; break; }
      const uint8_t* src = pk + s * C::kPk;
      if (WF == 3) {
        // 8-bit codes: per-weight arithmetic; a whole-row thread with groups
        // of 32 reads the second group's scale and bias here
        float sc1 = sc, bi1 = bi;
        if (DW == 4 && p.g_shift == 0) {
          const uint32_t g2 = 2u * bcur + 1u;
          sc1 = __ldg(p.asc + g2);
          bi1 = __ldg(p.abi + g2);
        }
        if (!DX) {
          tc_fence_after();
          const uint8_t* row = src + (uint32_t)u * 64;
          const uint32_t x = ((uint32_t)u >> 1) & 3u;
          if (DW == 4) {
            uint32_t v[32];
            aff8_regs<4>(row, x, 0, sc, bi, sc1, bi1, v);
            tmem_st_32x32b_x32(tm_row + (uint32_t)(d * 32), v);
          } else {
            uint32_t v[16];
            aff8_regs<2>(row, x, 2 * half, sc, bi, sc, bi, v);
            tmem_st_32x32b_x16(tm_row + (uint32_t)(d * 32 + 16 * half), v);
          }
          tmem_st_wait();
          tc_fence_before();
        } else {
          const uint32_t o = (uint32_t)(u & 63), hh = (uint32_t)(u >> 6);
          const uint8_t* row = src + o * 128;
          const uint32_t daddr = smem_u32(wdec + d * kWTile) + row_off;
          if (DW == 4)
            aff8_smem<4>(row, o & 7u, (int)hh, 0, sc, bi, sc1, bi1, daddr, sw);
          else
            aff8_smem<2>(row, o & 7u, (int)hh, 2 * half, sc, bi, sc, bi, daddr, sw);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&dec_full[d]));
        s += DG;
        if (s >= NIN) { s -= NIN; ph_in ^= 1u; }
        d += DG;
        if (d >= NDEC) d -= NDEC;
        continue;
      }
      // decode tables: one per block, or (whole-row threads, affine groups
      // of 32) one per half block, the second group's scale and bias read here
      const Nf4Planes tA = affine ? affine_planes(sc, bi) : nf4_planes(sc);
      Nf4Planes tB = tA;
      if (DW == 4 && affine && p.g_shift == 0) {
        const uint32_t g2 = 2u * bcur + 1u;
        tB = affine_planes(__ldg(p.asc + g2), __ldg(p.abi + g2));
      }
      if (!DX) {
        tc_fence_after();
        if (DW == 4) {
          uint32_t v[32];
          decode_row_regs(src + pk_lo, src + pk_hi, tA, tB, v);
          tmem_st_32x32b_x32(tm_row + (uint32_t)(d * 32), v);
        } else {
          uint32_t v[16];
          decode_half_regs(src + (half ? pk_hi : pk_lo), tA, v);
          tmem_st_32x32b_x16(tm_row + (uint32_t)(d * 32 + 16 * half), v);
        }
        tmem_st_wait();
        tc_fence_before();
      } else {
        if (DW == 4)
          decode_row_smem(src + pk_lo, src + pk_hi, tA, tB, smem_u32(wdec + d * kWTile) + row_off, sw);
        else
          decode_half_smem(src + (half ? pk_hi : pk_lo), tA, smem_u32(wdec + d * kWTile) + row_off,
                           sw, half);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&dec_full[d]));
      s += DG;
      if (s >= NIN) { s -= NIN; ph_in ^= 1u; }
      d += DG;
      if (d >= NDEC) d -= NDEC;
    }
    // the accumulator is complete once acc_full fires
    const bool acc_ok = mbar_wait(smem_u32(acc_full), 0, p.wait_ns, p.err, 0x401);
    if (!ok || !acc_ok) *abort_flag = 1;
  }
  // All roles are past the main loop: the ring buffers are free and the
  // abort flag is final (and the same for every thread after this barrier).
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp >= 2 && *abort_flag == 0) {
    // ---------------------------------------------------------- epilogue
    // Warp w reads TMEM lanes 32*(w%4) .. +31; the epilogue groups (four
    // warps each) split the token columns (group 0 alone when the tile is
    // narrower than 64).  Each group stages its columns in the freed ring
    // buffers and one thread writes them with two TMA stores (weight-side
    // rows 0..63, 64..127).
    const int group = (warp - 2) >> 2;
    constexpr int kColsPerGroup = cols_per_group<BN>();
    const int c_begin = BN >= 64 ? group * kColsPerGroup : 0;
    const int c_end = BN >= 64 ? c_begin + kColsPerGroup : (group == 0 ? BN : 0);
    if (group < epi_groups(BN) && c_end > c_begin) {
      const int es = p.partial ? 4 : 2;
      uint8_t* ep = smem + (size_t)group * 2 * kColsPerGroup * 64 * es;
      if (p.partial)
        epilogue_stage<true>(tmem, warp & 3, lane, c_begin, c_end, kColsPerGroup, ep);
      else
        epilogue_stage<false>(tmem, warp & 3, lane, c_begin, c_end, kColsPerGroup, ep);
      fence_proxy_async_smem();
      named_bar_sync(1 + group, 128);
      if (((warp - 2) & 3) == 0 && lane == 0) {
        const int32_t y = (int32_t)(n0 + c_begin);
        tma_store_3d(&tm_out, smem_u32(ep), m0, y, split);
        tma_store_3d(&tm_out, smem_u32(ep + (size_t)kColsPerGroup * 64 * es), m0 + 64, y, split);
        bulk_commit_and_wait_read();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  // The grid counts as finished only after the launch it depends on has:
  // whatever runs next in the stream sees that launch's writes too.
  if (threadIdx.x == 0) griddep_wait();
}

// ------------------------------------------------------------------ host

using EncodeTiled = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiled)f;
  }
  return fn;
}

// 2D row-major tensor [rows x cols] of `esize`-byte elements, box [br x bc].
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
              uint64_t rows, uint32_t bc, uint32_t br, CUtensorMapSwizzle swz) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)esize};
  cuuint32_t box[2] = {bc, br};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3D view {d0, d1, d2} of `esize`-byte elements with byte strides s1 (dim
// 1) and s2 (dim 2), box {b0, b1, b2}: the token and packed tiles of b2
// consecutive K steps in one copy, landing as b2 consecutive tiles.
bool make_map3(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t d0, uint64_t d1,
               uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
               CUtensorMapSwizzle swz) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3D output map [splits][rows][cols] of `esize`-byte elements, box
// [1][br][64] (one 64-column half of a tile), no swizzle.
bool make_out_map(CUtensorMap* m, const void* base, bool fp32, uint64_t cols, uint64_t rows,
                  uint64_t splits, uint32_t br) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const uint64_t es = fp32 ? 4 : 2;
  cuuint64_t dims[3] = {cols, rows, splits};
  cuuint64_t strides[2] = {cols * es, cols * rows * es};
  cuuint32_t box[3] = {64, br, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms_cached() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// The launch waits for the kernel before it in the stream only where the
// adapter step needs that kernel's output (programmatic dependent launch):
// the weight stream starts while U / V are still being computed.
template <bool DX, int BN, int WF>
cudaError_t launch_bn(dim3 grid, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                      const CUtensorMap& d, const CUtensorMap& o, const TcParams& p,
                      cudaStream_t st) {
  using Cf = Cfg<DX, BN, wf_bits(WF)>;
  auto kern = tc_qlinear_kernel<DX, BN, WF>;
  static bool attr_set = false;  // once per instantiation (keeps graph capture free of it)
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const double flops = 2.0 * (double)p.R * (double)p.Mw * (double)p.KB * kBK +
                       2.0 * (double)p.R * (double)p.Mw * (double)p.rank;
  const int slot = timing_begin(st, DX ? 1 : 0, flops);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(Cf::kThreads);
  cfg.dynamicSmemBytes = (size_t)Cf::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  // a timing event between the two launches would separate them anyway
  cfg.attrs = attr;
  cfg.numAttrs = slot < 0 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, b, c, d, o, p);
  timing_end(slot, st);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <bool DX, int WF>
cudaError_t launch_plan_wf(const TcPlan& pl, dim3 grid, const CUtensorMap& a, const CUtensorMap& b,
                           const CUtensorMap& c, const CUtensorMap& d, const CUtensorMap& o,
                           const TcParams& p, cudaStream_t st) {
  switch (pl.bn) {
    case 16: return launch_bn<DX, 16, WF>(grid, a, b, c, d, o, p, st);
    case 32: return launch_bn<DX, 32, WF>(grid, a, b, c, d, o, p, st);
    case 64: return launch_bn<DX, 64, WF>(grid, a, b, c, d, o, p, st);
    case 128: return launch_bn<DX, 128, WF>(grid, a, b, c, d, o, p, st);
    default: return launch_bn<DX, 256, WF>(grid, a, b, c, d, o, p, st);
  }
}

template <bool DX>
cudaError_t launch_plan(const TcPlan& pl, dim3 grid, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& c, const CUtensorMap& d, const CUtensorMap& o,
                        const TcParams& p, cudaStream_t st) {
  if (p.pre) return launch_bn<DX, 256, 4>(grid, a, b, c, d, o, p, st);
  if (p.asc) return p.pbits == 8 ? launch_plan_wf<DX, 3>(pl, grid, a, b, c, d, o, p, st)
                                 : launch_plan_wf<DX, 2>(pl, grid, a, b, c, d, o, p, st);
  if (p.sb) return launch_plan_wf<DX, 1>(pl, grid, a, b, c, d, o, p, st);
  return launch_plan_wf<DX, 0>(pl, grid, a, b, c, d, o, p, st);
}

int group_cols(int bn) { return bn >= 64 ? bn / epi_groups(bn) : bn; }

bool ptr_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool common_supported(const WView& w, int64_t R) {
  if (w.fmt == QLORA_FMT_NF4_DQ) {
    if (w.block != kBK || w.group < 1) return false;
  } else if (w.fmt == QLORA_FMT_NF4_FP32SCALE) {
    if (w.block != kBK) return false;
  } else if (w.fmt == QLORA_FMT_AFFINE) {
    if ((w.bits != 4 && w.bits != 8) || (w.block != 32 && w.block != 64 && w.block != 128))
      return false;
  } else {
    return false;
  }
  if (R <= 0 || R > (int64_t)INT32_MAX - 256) return false;
  if (w.I % 128 != 0 || w.O % 128 != 0) return false;
  if (w.O > INT32_MAX || w.I > INT32_MAX) return false;
  if ((w.O * w.I) / kBK >= (int64_t)UINT32_MAX) return false;
  if (!ptr_aligned(w.codes, 16)) return false;
  return encode_fn() != nullptr;
}

size_t partial_bytes(const TcPlan& pl, int64_t R, int64_t Mw) {
  return pl.splits > 1 ? align_up((size_t)pl.splits * (size_t)R * (size_t)Mw * 4, 256) : 0;
}

}  // namespace

TcPlan tc_plan(int64_t Mw, int64_t KB, int64_t R) {
  TcPlan pl;
  const int sms = num_sms_cached();
  const int64_t mt = Mw / kBM;
  // Token tile: the smallest power of two >= R (16..256); at large R, halve
  // it (down to 64) while the grid fills less than 3/4 of a wave, rather
  // than split K (a 256-token tile reads half the weight bytes per flop of
  // a 128-token one and wins down to ~0.85 of a wave).
  int bn = 16;
  while (bn < 256 && bn < R) bn *= 2;
  while (bn > 64 && 4 * mt * ((R + bn - 1) / bn) < 3 * (int64_t)sms) bn /= 2;
  pl.bn = bn;
  pl.stages = 0;
  const int64_t tiles = mt * ((R + bn - 1) / bn);
  // Below one wave of tiles, split K so that the grid is one full wave
  // (two CTAs per SM up to 128-token tiles), at least 4 K steps per split.
  int64_t splits = 1;
  if (tiles > 0 && tiles < sms) {
    splits = ((bn >= 256 ? 1 : 2) * (int64_t)sms) / tiles;
    const int64_t max_splits = KB / 4 > 0 ? KB / 4 : 1;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
  }
  pl.kb_per_split = (int)((KB + splits - 1) / splits);
  pl.splits = (int)((KB + pl.kb_per_split - 1) / pl.kb_per_split);
  return pl;
}

bool tc_fwd_supported(const WView& w, const void* X, const void* Y, int64_t R) {
  return common_supported(w, R) && ptr_aligned(X, 16) && ptr_aligned(Y, 16);
}

bool tc_dx_supported(const WView& w, const void* dY, const void* dX, int64_t R) {
  return common_supported(w, R) && ptr_aligned(dY, 16) && ptr_aligned(dX, 16);
}

// From this many tokens on (with 256-token tiles and no K split) the input
// gradient decodes the weight to bf16 once per call and the GEMM reads it
// with TMA: the decode and its shared-memory tile leave the MMA's critical
// path, for 2.5 extra HBM bytes per weight per call, which the GEMM's 2 R
// flops per weight repay well before this token count.  Measured on the
// 14B layer: input-gradient kernel 1154-1165 vs 966-969 TFLOP/s, step
// 923-925 vs 901-905 TFLOP/s under the power cap.  The forward, whose
// in-GEMM decode writes TMEM rather than shared memory, gained ~3% per
// kernel but lost it to the lower clock under the power cap (step 908-910),
// so it keeps the in-GEMM decode (QLORA_TC_PRE_FWD=1 switches it over).
constexpr int64_t kPreMinTokens = 2048;

#ifndef QLORA_TC_PRE_FWD
#define QLORA_TC_PRE_FWD 0
#endif
bool tc_pre(bool dx, const TcPlan& pl, int64_t R) {
  return (dx || QLORA_TC_PRE_FWD) && pl.bn == 256 && pl.splits == 1 && R >= kPreMinTokens;
}

size_t wbuf_bytes(const WView& w) { return align_up((size_t)w.O * (size_t)w.I * 2, 256); }

// Workspace: U_pad / V_pad bf16 [R x 64], the adapter weight operand bf16
// (fwd: [O x 64]; dX: [64 x I]), split-K partials, and (from kPreMinTokens
// tokens) the bf16 copy of the decoded weight [O x I].
size_t tc_fwd_ws(const WView& w, int64_t R) {
  const TcPlan pl = tc_plan(w.O, w.I / kBK, R);
  return align_up((size_t)R * 128, 256) + align_up((size_t)w.O * 128, 256) +
         partial_bytes(pl, R, w.O) + (tc_pre(false, pl, R) ? wbuf_bytes(w) : 0);
}

size_t tc_dx_ws(const WView& w, int64_t R) {
  const TcPlan pl = tc_plan(w.I, w.O / kBK, R);
  return align_up((size_t)R * 128, 256) + align_up((size_t)w.I * 128, 256) +
         partial_bytes(pl, R, w.I) + (tc_pre(true, pl, R) ? wbuf_bytes(w) : 0);
}

namespace {

// Decode inputs of the weight (the same for both directions).
void fill_weight_params(const WView& w, TcParams& p) {
  p.C = (uint32_t)(w.group < 1 ? 1 : w.group);
  p.c_shift = ((p.C & (p.C - 1)) == 0) ? __builtin_ctz(p.C) : -1;
  p.qcodes = w.qcodes;
  p.t = w.t;
  p.mu = w.mu;
  p.sb = w.fmt == QLORA_FMT_NF4_FP32SCALE ? w.scale : nullptr;
  p.asc = w.fmt == QLORA_FMT_AFFINE ? w.scale : nullptr;
  p.abi = w.fmt == QLORA_FMT_AFFINE ? w.bias : nullptr;
  p.g_shift = w.block == 128 ? 2 : w.block == 64 ? 1 : 0;
  p.pbits = w.bits;
}

// The bf16 weight copy of the tensor-core workspace.
uint16_t* wbuf_of(void* tcws, int64_t R, int64_t Mw, const TcPlan& pl) {
  return (uint16_t*)((char*)tcws + align_up((size_t)R * 128, 256) + align_up((size_t)Mw * 128, 256) +
                     partial_bytes(pl, R, Mw));
}

}  // namespace

cudaError_t tc_prepare(bool dx, const WView& w, int64_t R, void* tcws, cudaStream_t st) {
  const int64_t Mw = dx ? w.I : w.O;
  const TcPlan pl = dx ? tc_plan(w.I, w.O / kBK, R) : tc_plan(w.O, w.I / kBK, R);
  if (!tc_pre(dx, pl, R)) return cudaSuccess;
  TcParams p = {};
  fill_weight_params(w, p);
  const int64_t nb = w.O * w.I / kBK;
  uint4* out = (uint4*)wbuf_of(tcws, R, Mw, pl);
  const unsigned grid = (unsigned)((nb + 255) / 256);
  if (w.fmt == QLORA_FMT_AFFINE) {
    if (w.bits == 8)
      expand_bf16_kernel<3><<<grid, 256, 0, st>>>(p, w.codes, nb, out);
    else
      expand_bf16_kernel<2><<<grid, 256, 0, st>>>(p, w.codes, nb, out);
  } else if (w.fmt == QLORA_FMT_NF4_FP32SCALE) {
    expand_bf16_kernel<1><<<grid, 256, 0, st>>>(p, w.codes, nb, out);
  } else {
    expand_bf16_kernel<0><<<grid, 256, 0, st>>>(p, w.codes, nb, out);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_tc_fwd(const WView& w, const void* X, int64_t R, const float* U,
                          const float* B, int32_t r, float s, void* Y, void* tcws,
                          uint32_t* hdr, cudaStream_t st) {
  const int64_t O = w.O, I = w.I;
  const TcPlan pl = tc_plan(O, I / kBK, R);
  uint16_t* upad = (uint16_t*)tcws;
  uint16_t* bpad = (uint16_t*)((char*)tcws + align_up((size_t)R * 128, 256));
  float* part = (float*)((char*)bpad + align_up((size_t)O * 128, 256));
  // upad (bf16 U) and bpad (bf16(s B)) were written by the rowdot launch that made U
  (void)U;
  (void)B;
  (void)s;
  cudaError_t e = cudaSuccess;
  CUtensorMap m_act, m_pk, m_aact, m_aw;
  const uint32_t bn = (uint32_t)pl.bn;
  // X as {64 columns, R rows, I/64 K steps}; codes as {32 bytes, O rows, I/64 K steps}
  const uint32_t g = (uint32_t)tma_group(pl.bn);
  const bool pre = tc_pre(false, pl, R);
  // pre-decoded: the bf16 weight as {64 columns, O rows, I/64 K steps}, 16 KB boxes
  if (!make_map3(&m_act, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, (uint64_t)R, (uint64_t)(I / 64),
                 (uint64_t)I * 2, 128, 64, bn, g, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !(pre ? make_map3(&m_pk, wbuf_of(tcws, R, O, pl), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64,
                        (uint64_t)O, (uint64_t)(I / 64), (uint64_t)I * 2, 128, 64, 128, 1,
                        CU_TENSOR_MAP_SWIZZLE_128B)
      : w.bits == 8
            ? make_map3(&m_pk, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, (uint64_t)O,
                        (uint64_t)(I / 64), (uint64_t)I, 64, 64, 128, g, CU_TENSOR_MAP_SWIZZLE_64B)
            : make_map3(&m_pk, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 32, (uint64_t)O,
                        (uint64_t)(I / 64), (uint64_t)(I / 2), 32, 32, 128, g,
                        CU_TENSOR_MAP_SWIZZLE_32B)) ||
      !make_map(&m_aact, upad, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, R, 64, bn, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&m_aw, bpad, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, O, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcParams p;
  p.R = R;
  p.Mw = (int32_t)O;
  p.KB = (int32_t)(I / kBK);
  p.I = (int32_t)I;
  p.kb_per_split = pl.kb_per_split;
  p.r_slices = (r + 15) / 16;
  p.rank = r;
  fill_weight_params(w, p);
  p.pre = pre ? 1 : 0;
  p.partial = pl.splits > 1;
  p.out = pl.splits > 1 ? (void*)part : Y;
  p.err = hdr;
  p.wait_ns = kWaitLimitNs;
  CUtensorMap m_out;
  if (!make_out_map(&m_out, p.out, pl.splits > 1, (uint64_t)O, (uint64_t)R, (uint64_t)pl.splits,
                    (uint32_t)group_cols(pl.bn)))
    return cudaErrorInvalidValue;
  dim3 grid((unsigned)(O / kBM), (unsigned)((R + pl.bn - 1) / pl.bn), (unsigned)pl.splits);
  e = launch_plan<false>(pl, grid, m_act, m_pk, m_aact, m_aw, m_out, p, st);
  if (e != cudaSuccess || pl.splits == 1) return e;
  return launch_splitk_reduce(part, pl.splits, R, O, true, Y, st, 1.0f, !timing_enabled());
}

cudaError_t launch_tc_dx(const WView& w, const void* dY, int64_t R, const float* V,
                         const float* A, int32_t r, float s, void* dX, void* tcws, uint32_t* hdr,
                         cudaStream_t st) {
  const int64_t O = w.O, I = w.I;
  const TcPlan pl = tc_plan(I, O / kBK, R);
  uint16_t* vpad = (uint16_t*)tcws;
  uint16_t* apad = (uint16_t*)((char*)tcws + align_up((size_t)R * 128, 256));
  float* part = (float*)((char*)apad + align_up((size_t)I * 128, 256));
  // vpad (bf16 V) and apad (bf16(s A)) were written by the rowdot launch that made V
  (void)V;
  (void)A;
  (void)s;
  cudaError_t e = cudaSuccess;
  CUtensorMap m_act, m_pk, m_aact, m_aw;
  const uint32_t bn = (uint32_t)pl.bn;
  // dY as {64 columns, R rows, O/64 K steps}; codes as {I/2 bytes, 64 rows, O/64 K steps}
  const uint32_t g = (uint32_t)tma_group(pl.bn);
  const bool pre = tc_pre(true, pl, R);
  // pre-decoded: the bf16 weight as {I columns, 64 rows, O/64 K steps}, two
  // 64 x 64 boxes per step (the MN-major W^T tile)
  if (!make_map3(&m_act, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, (uint64_t)R, (uint64_t)(O / 64),
                 (uint64_t)O * 2, 128, 64, bn, g, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !(pre ? make_map3(&m_pk, wbuf_of(tcws, R, I, pl), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        (uint64_t)I, 64, (uint64_t)(O / 64), (uint64_t)I * 2, (uint64_t)64 * I * 2,
                        64, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B)
      : w.bits == 8
            ? make_map3(&m_pk, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)I, 64,
                        (uint64_t)(O / 64), (uint64_t)I, (uint64_t)64 * I, 128, 64, g,
                        CU_TENSOR_MAP_SWIZZLE_128B)
            : make_map3(&m_pk, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)(I / 2), 64,
                        (uint64_t)(O / 64), (uint64_t)(I / 2), (uint64_t)64 * (I / 2), 64, 64, g,
                        CU_TENSOR_MAP_SWIZZLE_64B)) ||
      !make_map(&m_aact, vpad, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, R, 64, bn, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&m_aw, apad, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, I, 64, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcParams p;
  p.R = R;
  p.Mw = (int32_t)I;
  p.KB = (int32_t)(O / kBK);
  p.I = (int32_t)I;
  p.kb_per_split = pl.kb_per_split;
  p.r_slices = (r + 15) / 16;
  p.rank = r;
  fill_weight_params(w, p);
  p.pre = pre ? 1 : 0;
  p.partial = pl.splits > 1;
  p.out = pl.splits > 1 ? (void*)part : dX;
  p.err = hdr;
  p.wait_ns = kWaitLimitNs;
  CUtensorMap m_out;
  if (!make_out_map(&m_out, p.out, pl.splits > 1, (uint64_t)I, (uint64_t)R, (uint64_t)pl.splits,
                    (uint32_t)group_cols(pl.bn)))
    return cudaErrorInvalidValue;
  dim3 grid((unsigned)(I / kBM), (unsigned)((R + pl.bn - 1) / pl.bn), (unsigned)pl.splits);
  e = launch_plan<true>(pl, grid, m_act, m_pk, m_aact, m_aw, m_out, p, st);
  if (e != cudaSuccess || pl.splits == 1) return e;
  return launch_splitk_reduce(part, pl.splits, R, I, true, dX, st, 1.0f, !timing_enabled());
}

// Failure-detection self test: one thread waits on an mbarrier that nothing
// arrives on; the bounded wait gives up and records QLORA_ERR_TIMEOUT.
__global__ void wait_selftest_kernel(uint32_t* hdr, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    mbar_wait(smem_u32(&bar), 0, limit_ns, hdr, 0x901);
  }
}

cudaError_t launch_wait_selftest(uint32_t* ws_header, uint64_t limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(ws_header, limit_ns);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
