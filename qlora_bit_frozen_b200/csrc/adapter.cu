// adapter.cu -- the LoRA side products of the QLoRA linear layer.
//
// "QLoRA on Mac", "Design / Q-LoRA layer": the adapter branch is
// (alpha/r)(x A^T) B^T with fp32 A, B.  Forward needs U = X A^T; the
// backward chain rule needs V = dY B, dA = s V^T X and dB = s dY^T U.
// Each reads one activation matrix once and touches an r-wide factor, so
// they are bound by HBM bandwidth on X / dY.
//
//  * bf16 activations (the tensor-core configurations): rowdot_mma_kernel
//    and coldot_mma_kernel run the products on mma.sync with the fp32
//    factor split into two bf16 halves (16 significant bits kept); few-row
//    cases split the reduction across blocks and the last block to finish
//    adds the partials in a fixed order.  rowdot also writes the bf16 copy
//    of U / V zero-padded to 64 columns and (extra blocks of the same
//    launch) the zero-padded bf16(s B) / bf16(s A) operand of the
//    tensor-core kernel's adapter step.
//  * fp32 activations (fp32 compute mode) and unaligned inputs: the FMA
//    forms rowdot_kernel / coldot_kernel, fp32 throughout.
#include "common.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int kThreads = 256;

// 16-byte global -> shared copy, asynchronous; bytes past src_bytes are
// filled with zeros (src_bytes = 0 for padding rows/columns).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ----------------------------------------------------------------- loads

template <typename T, int E>
struct Raw {
  static constexpr int kBytes = E * (int)sizeof(T);
  static constexpr int W = (kBytes + 3) / 4;
  uint32_t w[W];
  __device__ __forceinline__ void load(const T* p, int nvalid, bool vec_ok) {
    if (vec_ok && nvalid >= E) {
      if constexpr (kBytes == 32) {
        const uint4 a = *reinterpret_cast<const uint4*>(p);
        const uint4 b = *reinterpret_cast<const uint4*>(p + 16 / (int)sizeof(T));
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
      } else if constexpr (kBytes == 16) {
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
      } else if constexpr (kBytes == 8) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        w[0] = v.x; w[1] = v.y;
      } else if constexpr (kBytes == 4) {
        w[0] = *reinterpret_cast<const uint32_t*>(p);
      } else {
        w[0] = *reinterpret_cast<const unsigned short*>(p);
      }
    } else {
      float x[E];
#pragma unroll
      for (int i = 0; i < E; ++i) x[i] = i < nvalid ? to_f32<T>(p[i]) : 0.0f;
      set(x);
    }
  }
  __device__ __forceinline__ void set(const float (&x)[E]) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int i = 0; i < W; ++i) {
        const uint32_t lo = __float_as_uint(x[2 * i]) >> 16;
        const uint32_t hi = 2 * i + 1 < E ? (__float_as_uint(x[2 * i + 1]) & 0xFFFF0000u) : 0u;
        w[i] = lo | hi;
      }
    } else {
#pragma unroll
      for (int i = 0; i < W; ++i) w[i] = __float_as_uint(x[i]);
    }
  }
  __device__ __forceinline__ float at(int i) const {
    if constexpr (sizeof(T) == 2)
      return __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
    else
      return __uint_as_float(w[i]);
  }
};

// ---------------------------------------------------------------- pad job

// Zero-padded bf16 copy of an r-wide fp32 factor times mul:
//   mode 0: dst[rows x 64] from src[rows x r]   (bf16(s B), [O x 64])
//   mode 1: dst[64 x cols] from src[r x cols]   (bf16(s A), [64 x I])
struct PadJob {
  const float* src;
  uint16_t* dst;
  int64_t extent;  // rows (mode 0) or cols (mode 1)
  int r;
  int mode;
  float mul;
  int blocks;  // launch blocks reserved for this job (0 = none)
};

__device__ void run_pad_job(const PadJob& j, int64_t blk) {
  const int64_t total = 64 * j.extent;
  for (int64_t e = blk * kThreads * 8 + threadIdx.x; e < min(total, (blk + 1) * kThreads * 8);
       e += kThreads) {
    float v;
    if (j.mode == 0) {
      const int64_t m = e >> 6;
      const int c = (int)(e & 63);
      v = c < j.r ? __fmul_rn(j.mul, j.src[m * j.r + c]) : 0.0f;
    } else {
      const int64_t row = e / j.extent;
      v = row < j.r ? __fmul_rn(j.mul, j.src[e]) : 0.0f;
    }
    j.dst[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// ------------------------------------------------------------------ rowdot

// Block = 8 warps = (8 / KS) row groups x KS column groups.  A warp owns RW
// rows and the 256-wide K steps kg, kg + KS, ...; each lane loads 8
// consecutive elements of each of its rows per step (all rows' loads in
// flight together) and reads the matching 8 x r factor values through L1
// (they are shared by the RW rows).  Lane partials are combined with a
// butterfly, column groups (KS > 1, for few rows) in shared memory in a fixed
// order.
template <typename T, int RMAX, int RW, int KS>
__global__ void __launch_bounds__(kThreads) rowdot_kernel(const T* __restrict__ P, int64_t R,
                                                          int64_t K, const float* __restrict__ L,
                                                          int l_is_kr, int r,
                                                          float* __restrict__ out,
                                                          uint16_t* __restrict__ out_pad,
                                                          int row_blocks, PadJob job) {
  // the tensor-core kernel queued next may start its weight stream now
  if (threadIdx.x == 0) griddep_launch_dependents();
  if ((int)blockIdx.x >= row_blocks) {
    run_pad_job(job, (int64_t)blockIdx.x - row_blocks);
    return;
  }
  constexpr int EPL = 8;
  constexpr int STEP = 32 * EPL;  // 256 columns per warp step
  constexpr int RG = 8 / KS;      // row groups per block
  __shared__ float red[KS > 1 ? KS : 1][RW][RMAX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = warp % RG, kg = warp / RG;
  const int64_t row0 = ((int64_t)blockIdx.x * RG + rg) * RW;
  const bool vec_ok = (K % EPL) == 0 && ((uintptr_t)P % (EPL * sizeof(T))) == 0;
  const bool l_vec = ((uintptr_t)L % 16) == 0 && (l_is_kr ? (r % 4) == 0 : (K % 4) == 0);
  float acc[RW][RMAX];
#pragma unroll
  for (int q = 0; q < RW; ++q)
#pragma unroll
    for (int j = 0; j < RMAX; ++j) acc[q][j] = 0.0f;

  for (int64_t k0 = (int64_t)kg * STEP; k0 < K; k0 += (int64_t)KS * STEP) {
    const int64_t k = k0 + lane * EPL;
    const int nk = (int)max((int64_t)0, min((int64_t)EPL, K - k));
    Raw<T, EPL> x[RW];
#pragma unroll
    for (int q = 0; q < RW; ++q) {
      const int64_t m = row0 + q;
      x[q].load(P + m * K + k, m < R ? nk : 0, vec_ok);
    }
    if (nk == 0) continue;
#pragma unroll
    for (int j = 0; j < RMAX; ++j) {
      if (j < r) {
        float l[EPL];
        if (!l_is_kr) {  // L[j * K + k]
          const float* lp = L + (int64_t)j * K + k;
          if (l_vec && nk == EPL) {
            const float4 a = __ldg(reinterpret_cast<const float4*>(lp));
            const float4 b = __ldg(reinterpret_cast<const float4*>(lp + 4));
            l[0] = a.x; l[1] = a.y; l[2] = a.z; l[3] = a.w;
            l[4] = b.x; l[5] = b.y; l[6] = b.z; l[7] = b.w;
          } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) l[e] = e < nk ? __ldg(lp + e) : 0.0f;
          }
        } else {  // L[k * r + j]
#pragma unroll
          for (int e = 0; e < EPL; ++e) l[e] = e < nk ? __ldg(L + (k + e) * r + j) : 0.0f;
        }
#pragma unroll
        for (int q = 0; q < RW; ++q)
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[q][j] = fmaf(x[q].at(e), l[e], acc[q][j]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < RW; ++q)
#pragma unroll
    for (int j = 0; j < RMAX; ++j)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[q][j] += __shfl_xor_sync(0xffffffffu, acc[q][j], o);
  if constexpr (KS > 1) {
    if (lane == 0)
#pragma unroll
      for (int q = 0; q < RW; ++q)
#pragma unroll
        for (int j = 0; j < RMAX; ++j) red[kg][q][j] = acc[q][j];
    __syncthreads();
    if (kg != 0) return;
#pragma unroll
    for (int q = 0; q < RW; ++q)
#pragma unroll
      for (int j = 0; j < RMAX; ++j) {
        float v = red[0][q][j];
#pragma unroll
        for (int g = 1; g < KS; ++g) v += red[g][q][j];
        acc[q][j] = v;
      }
  }
#pragma unroll
  for (int q = 0; q < RW; ++q) {
    const int64_t m = row0 + q;
    if (m >= R) continue;
    float a0 = 0.0f, a1 = 0.0f;  // columns lane and lane + 32, picked without dynamic indexing
#pragma unroll
    for (int j = 0; j < RMAX; ++j) {
      if (j == lane) a0 = acc[q][j];
      if (j == lane + 32) a1 = acc[q][j];
    }
    if (lane < r) out[m * r + lane] = a0;
    if (lane + 32 < r) out[m * r + lane + 32] = a1;
    if (out_pad) {
      out_pad[m * 64 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(lane < r ? a0 : 0.0f));
      out_pad[m * 64 + lane + 32] =
          __bfloat16_as_ushort(__float2bfloat16_rn(lane + 32 < r ? a1 : 0.0f));
    }
  }
}

// ------------------------------------------------------------------ coldot

template <int RMAX>
constexpr int col_cpt() {
  return RMAX <= 8 ? 8 : RMAX <= 16 ? 4 : RMAX <= 32 ? 2 : 1;  // CPT * RMAX = 64
}
constexpr int kRowLanes = kThreads / 32;
constexpr int kUnroll = 8;

// Block (x, y) = column range x (32 threads x CPT columns) over row slice y,
// 8 row lanes per column thread, 8 rows in flight per lane.  The row lanes
// are summed in shared memory; the slice sums go to `part`; the last block
// of column range x to finish (ticket counter) adds the slices in slice
// order, scales by s and writes the result: dA as [r x N] (out_nr = 0) or
// dB as [N x r] (out_nr = 1).  With one slice it writes directly.
template <typename T, int RMAX>
__global__ void __launch_bounds__(kThreads) coldot_kernel(const T* __restrict__ P, int64_t R,
                                                          int64_t N, const float* __restrict__ aux,
                                                          int r, int64_t rows_per_split,
                                                          int splits, float s, int out_nr,
                                                          float* __restrict__ part,
                                                          unsigned* __restrict__ tickets,
                                                          float* __restrict__ out) {
  constexpr int CPT = col_cpt<RMAX>();
  constexpr int NV = CPT * RMAX;  // accumulators per thread (64)
  __shared__ float red[4][NV][32];  // 32 KB: row-lane reduction staging
  __shared__ unsigned is_last;
  const int c = threadIdx.x & 31, tr = threadIdx.x >> 5;
  const int64_t nb = (int64_t)blockIdx.x * (32 * CPT);
  const int64_t n0 = nb + (int64_t)c * CPT;
  const int64_t m_lo = (int64_t)blockIdx.y * rows_per_split;
  const int64_t m_hi = min(R, m_lo + rows_per_split);
  const bool vec_ok = (N % CPT) == 0 && ((uintptr_t)P % (CPT * sizeof(T))) == 0;
  const int nvalid = (int)max((int64_t)0, min((int64_t)CPT, N - n0));
  const bool aux_vec = (r % 4) == 0 && ((uintptr_t)aux % 16) == 0;
  float acc[CPT][RMAX];
#pragma unroll
  for (int cc = 0; cc < CPT; ++cc)
#pragma unroll
    for (int j = 0; j < RMAX; ++j) acc[cc][j] = 0.0f;

  for (int64_t m = m_lo + tr; m < m_hi; m += kRowLanes * kUnroll) {
    Raw<T, CPT> p[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t mu = m + (int64_t)u * kRowLanes;
      p[u].load(P + mu * N + n0, mu < m_hi ? nvalid : 0, vec_ok);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t mu = m + (int64_t)u * kRowLanes;
      if (mu >= m_hi) break;
      const float* arow = aux + mu * r;
#pragma unroll
      for (int j = 0; j < RMAX; j += 4) {
        if (j < r) {
          float a[4];
          if (aux_vec) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(arow + j));
            a[0] = f.x; a[1] = f.y; a[2] = f.z; a[3] = f.w;
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = j + i < r ? __ldg(arow + j + i) : 0.0f;
          }
#pragma unroll
          for (int cc = 0; cc < CPT; ++cc)
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (j + i < RMAX) acc[cc][j + i] = fmaf(a[i], p[u].at(cc), acc[cc][j + i]);
        }
      }
    }
  }
  // sum the 8 row lanes (warps): 8 -> 4 -> 2 -> 1 through shared memory
#pragma unroll
  for (int half = 4; half >= 1; half >>= 1) {
    __syncthreads();
    if (tr >= half && tr < 2 * half) {
#pragma unroll
      for (int cc = 0; cc < CPT; ++cc)
#pragma unroll
        for (int j = 0; j < RMAX; ++j) red[tr - half][cc * RMAX + j][c] = acc[cc][j];
    }
    __syncthreads();
    if (tr < half) {
#pragma unroll
      for (int cc = 0; cc < CPT; ++cc)
#pragma unroll
        for (int j = 0; j < RMAX; ++j) acc[cc][j] += red[tr][cc * RMAX + j][c];
    }
  }
  if (splits == 1) {
    if (tr == 0)
#pragma unroll
      for (int j = 0; j < RMAX; ++j)
#pragma unroll
        for (int cc = 0; cc < CPT; ++cc)
          if (j < r && cc < nvalid) {
            const int64_t n = n0 + cc;
            out[out_nr ? n * r + j : (int64_t)j * N + n] = s * acc[cc][j];
          }
    return;
  }
  if (tr == 0) {
    float* dst = part + (int64_t)blockIdx.y * r * N;
#pragma unroll
    for (int j = 0; j < RMAX; ++j)
#pragma unroll
      for (int cc = 0; cc < CPT; ++cc)
        if (j < r && cc < nvalid) dst[(int64_t)j * N + n0 + cc] = acc[cc][j];
    __threadfence();
  }
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(&tickets[blockIdx.x], 1u) == (unsigned)splits - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // this block's columns [nb, nb + 32 * CPT) x r: sum the slices in order
  const int ncols = (int)min((int64_t)(32 * CPT), N - nb);
  const int64_t rN = (int64_t)r * N;
  for (int e = threadIdx.x; e < ncols * r; e += kThreads) {
    const int j = e / ncols, cc = e - j * ncols;
    const int64_t idx = (int64_t)j * N + nb + cc;
    float v = 0.0f;
    int k = 0;
    for (; k + 8 <= splits; k += 8) {
      float t[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) t[u] = __ldcg(part + (int64_t)(k + u) * rN + idx);
#pragma unroll
      for (int u = 0; u < 8; ++u) v += t[u];
    }
    for (; k < splits; ++k) v += __ldcg(part + (int64_t)k * rN + idx);
    const int64_t n = nb + cc;
    out[out_nr ? n * r + j : idx] = s * v;
  }
  if (threadIdx.x == 0) tickets[blockIdx.x] = 0;  // ready for the next call
}

// ------------------------------------------- pipelined kernels (16-byte rows)
//
// Used when every row of P starts on a 16-byte boundary.  A block streams
// tiles of P (and of the r-wide factor) through a 4-stage cp.async ring in
// shared memory, so each block keeps ~3 tiles of loads in flight whatever
// its register use; threads compute from shared memory.


// ------------------------------------------------------ tensor-core path
//
// The same products on the tensor cores (mma.sync m16n8k16, bf16 operands,
// fp32 accumulation).  The activation operand is exact in bf16.  The fp32
// factor x is split into bf16 hi = bf16(x) and lo = bf16(x - hi) (x - hi is
// exact in fp32) and both halves are multiplied: the factor keeps 16
// significant bits (relative error <= 2^-16), against 24 in the FMA form.
// That removes the r FMAs per activation element from the issue slots; the
// kernels are then bound by HBM on the activation, not by instructions.

constexpr int kMmaStages = 4;
constexpr int kMaxTickets = 1024;  // zeroed counters the caller provides

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
// c += A (16 x 16, row) * B (16 x 8, col)
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// (x, y) -> bf16 pairs hi = (bf16(x), bf16(y)) and lo = bf16 of the remainders
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x, y);
  lo = pack_bf16x2(x - __uint_as_float(hi << 16), y - __uint_as_float(hi & 0xFFFF0000u));
}
// B fragment pair of one n-tile from an fp32 factor tile, hi/lo halves
// accumulated into c.  f(k, n) gives the factor entry (0 outside).
template <typename F>
__device__ __forceinline__ void mma_split(float (&c)[4], const uint32_t (&a)[4], int k0, int n,
                                          F f) {
  uint32_t h0, l0, h1, l1;
  split_bf16(f(k0, n), f(k0 + 1, n), h0, l0);
  split_bf16(f(k0 + 8, n), f(k0 + 9, n), h1, l1);
  mma16816(c, a, h0, h1);
  mma16816(c, a, l0, l1);
}

// dst[row * tstr + col] = sum over q < nsplit (in q order) of
// part[q * slice + (row0 + row) * NP + col] for rows < nrows, the whole
// block cooperating: four consecutive columns per thread and eight slices
// in flight, so the last block's reduction is not a chain of dependent
// L2 loads.  part was written by other blocks of this grid: read via L2.
template <int NP>
__device__ __forceinline__ void sum_slices(const float* __restrict__ part, int64_t slice,
                                           int64_t row0, int nrows, int rows, int nsplit,
                                           float* dst, int tstr) {
  for (int e4 = threadIdx.x; e4 < rows * (NP / 4); e4 += kThreads) {
    const int row = e4 / (NP / 4), col = (e4 % (NP / 4)) * 4;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (row < nrows) {
      const float* p = part + (row0 + row) * NP + col;
      int q = 0;
      for (; q + 8 <= nsplit; q += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldcg(reinterpret_cast<const float4*>(p + (q + u) * slice));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          acc.x += v[u].x;
          acc.y += v[u].y;
          acc.z += v[u].z;
          acc.w += v[u].w;
        }
      }
      for (; q < nsplit; ++q) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p + q * slice));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
    }
    dst[row * tstr + col] = acc.x;
    dst[row * tstr + col + 1] = acc.y;
    dst[row * tstr + col + 2] = acc.z;
    dst[row * tstr + col + 3] = acc.w;
  }
}

// c += A * (B_hi + B_lo) for one n-tile from a split tile in shared memory:
// hi row n at t + n * ls, lo row n at t + lo_off + n * ls (bf16, k contiguous).
__device__ __forceinline__ void mma_pairs(float (&c)[4], const uint32_t (&a)[4], const uint16_t* t,
                                          int ls, int lo_off, int n, int kb) {
  const uint16_t* h = t + n * ls + kb;
  const uint16_t* l = h + lo_off;
  mma16816(c, a, *reinterpret_cast<const uint32_t*>(h), *reinterpret_cast<const uint32_t*>(h + 8));
  mma16816(c, a, *reinterpret_cast<const uint32_t*>(l), *reinterpret_cast<const uint32_t*>(l + 8));
}

// Split an r-wide fp32 factor into bf16 hi / lo rows, n-major:
// dst[j * ld + k] = hi, dst[(NP + j) * ld + k] = lo of F(k, j), where
// F(k, j) = src[k * r + j] (nr = 1, [n x r]) or src[j * n + k] (nr = 0,
// [r x n]); zero for j >= r or k >= n, up to the row length ld.
__global__ void split_factor_kernel(const float* __restrict__ src, int64_t n, int r, int nr, int NP,
                                    int64_t ld, uint16_t* __restrict__ dst) {
  const int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 2;  // (j, k) pair start
  if (e >= (int64_t)NP * ld) return;
  const int64_t j = e / ld, k = e - j * ld;
  auto f = [&](int64_t kk) -> float {
    if (j >= r || kk >= n) return 0.0f;
    return nr ? src[kk * r + j] : src[j * n + kk];
  };
  uint32_t h, l;
  split_bf16(f(k), f(k + 1), h, l);
  *reinterpret_cast<uint32_t*>(dst + j * ld + k) = h;
  *reinterpret_cast<uint32_t*>(dst + ((int64_t)NP + j) * ld + k) = l;
}

// rowdot on the tensor cores: out[m, j] = sum_k P[m, k] L(k, j).
// Block = 8 warps = 4 row groups (16 rows each, 64 rows per block) x 2 K
// groups (alternate 16-column chunks); a stage holds KT = 128 columns of
// the 64 rows (rows padded by 16 bytes: conflict-free ldmatrix) and the
// matching factor tile, as given: [r x KT] rows when L is [r x K] (A),
// [KT x r] when L is [K x r] (B).  Grid = row blocks x K splits; with
// several splits each writes a partial and the last block of a row block
// to finish (ticket) adds them in split order.  The final values go out as
// fp32 [R x r] and, optionally, bf16 zero-padded to 64 columns.
// Ranks above 16 use 64-column stages (a smaller factor tile): three blocks
// per SM instead of one.
constexpr int rowmma_kt(int nt) { return nt >= 4 ? 64 : 128; }
constexpr int colmma_rt(int nt) { return nt >= 4 ? 32 : 64; }

// Factor modes: FM 0 fp32 [r x K] rows (A), FM 1 fp32 [K x r] (B), FM 2 the
// factor already split into bf16 hi / lo rows [2][NP][lstride] (n-major,
// zero past r and K) by split_factor_kernel: B fragments are then plain
// bf16 pairs, no per-warp split arithmetic.
template <int NT, int FM>
struct RowMma {
  static constexpr bool LKR = FM == 1;
  static constexpr int RB = 64, KT = rowmma_kt(NT);
  static constexpr int PCH = KT / 8;                   // 16-byte chunks per P row
  static constexpr int NP = 8 * NT;                    // padded rank
  static constexpr int PSTR = KT * 2 + 16;             // bytes per P row in smem
  static constexpr int PB = RB * PSTR;
  static constexpr int LSTRF = KT + 8;                 // floats per L row ([r x K] case)
  static constexpr int LSTRH = KT + 8;                 // bf16 per split row (FM 2)
  static constexpr int LB = FM == 2 ? 2 * NP * LSTRH * 2 : LKR ? KT * NP * 4 : NP * LSTRF * 4;
  static constexpr int STAGE = PB + LB;
  static constexpr int TSTR = NP + 1;                  // result tile row stride (floats)
  static constexpr int RED = 4 * 32 * NT * 4 * 4;      // K-group combine buffer
  static constexpr int TILE = RB * TSTR * 4;
  static constexpr int SMEM = kMmaStages * STAGE + (RED > TILE ? RED : TILE);
};

template <int NT, int FM>
__global__ void __launch_bounds__(kThreads) rowdot_mma_kernel(
    const __nv_bfloat16* __restrict__ P, int64_t R, int64_t K, const float* __restrict__ L,
    int64_t lstride, int r, int row_blocks, int ksplit, int tiles_per_split,
    float* __restrict__ out, uint16_t* __restrict__ out_pad, float* __restrict__ part,
    unsigned* __restrict__ tickets, PadJob job) {
  constexpr bool LKR = FM == 1;
  // the tensor-core kernel queued next may start its weight stream now
  if (threadIdx.x == 0) griddep_launch_dependents();
  if ((int)blockIdx.x >= row_blocks * ksplit) {
    run_pad_job(job, (int64_t)blockIdx.x - row_blocks * ksplit);
    return;
  }
  using C = RowMma<NT, FM>;
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = (int)blockIdx.x % row_blocks, ks = (int)blockIdx.x / row_blocks;
  const int64_t m0 = (int64_t)rb * C::RB;
  const int ntiles = (int)((K + C::KT - 1) / C::KT);
  const int t_lo = ks * tiles_per_split, t_hi = min(ntiles, t_lo + tiles_per_split);

  auto issue = [&](int t) {
    const uint32_t ps = (uint32_t)__cvta_generic_to_shared(sm + ((t - t_lo) % kMmaStages) * C::STAGE);
    const uint32_t ls = ps + C::PB;
    const int64_t k0 = (int64_t)t * C::KT;
    // P: 64 rows x PCH chunks of 16 bytes
#pragma unroll
    for (int i = 0; i < C::RB * C::PCH / kThreads; ++i) {
      const int c = threadIdx.x + kThreads * i, row = c / C::PCH, ch = c % C::PCH;
      const int64_t m = m0 + row, k = k0 + ch * 8;
      const int64_t rem = (K - k) * 2;
      const uint32_t nb = (m < R && rem > 0) ? (uint32_t)min((int64_t)16, rem) : 0u;
      cp_async16(ps + (uint32_t)(row * C::PSTR + ch * 16), nb ? (const void*)(P + m * K + k) : (const void*)P, nb);
    }
    if (FM == 2) {  // split rows: 2 x NP rows of KT bf16
      const uint16_t* Ls = reinterpret_cast<const uint16_t*>(L);
      for (int c = threadIdx.x; c < 2 * C::NP * (C::KT / 8); c += kThreads) {
        const int row = c / (C::KT / 8), ch = c % (C::KT / 8);
        const int64_t k = k0 + ch * 8;
        const int64_t rem = (lstride - k) * 2;
        const uint32_t nb = rem > 0 ? (uint32_t)min((int64_t)16, rem) : 0u;
        cp_async16(ls + (uint32_t)(row * C::LSTRH + ch * 8) * 2,
                   nb ? (const void*)(Ls + row * lstride + k) : (const void*)Ls, nb);
      }
    } else if (LKR) {  // contiguous [KT x r] floats
      const int64_t base = k0 * r, total = K * (int64_t)r;
      const int nch = (C::KT * r) / 4;
      for (int c = threadIdx.x; c < nch; c += kThreads) {
        const int64_t e = base + (int64_t)c * 4;
        const int64_t rem = (total - e) * 4;
        const uint32_t nb = rem > 0 ? (uint32_t)min((int64_t)16, rem) : 0u;
        cp_async16(ls + (uint32_t)c * 16, nb ? (const void*)(L + e) : (const void*)L, nb);
      }
    } else {  // NP rows of KT floats, rows >= r zero
      for (int c = threadIdx.x; c < C::NP * (C::KT / 4); c += kThreads) {
        const int j = c / (C::KT / 4), ch = c % (C::KT / 4);
        const int64_t k = k0 + ch * 4;
        const int64_t rem = (K - k) * 4;
        const uint32_t nb = (j < r && rem > 0) ? (uint32_t)min((int64_t)16, rem) : 0u;
        cp_async16(ls + (uint32_t)(j * C::LSTRF + ch * 4) * 4,
                   nb ? (const void*)(L + (int64_t)j * K + k) : (const void*)L, nb);
      }
    }
  };

  const int rg = warp & 3, kg = warp >> 2;
  const int g = lane >> 2, tq = lane & 3;
  float c[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0.0f;

#pragma unroll
  for (int i = 0; i < kMmaStages - 1; ++i) {
    if (t_lo + i < t_hi) issue(t_lo + i);
    cp_async_commit();
  }
  for (int t = t_lo; t < t_hi; ++t) {
    cp_async_wait<kMmaStages - 2>();
    __syncthreads();
    if (t + kMmaStages - 1 < t_hi) issue(t + kMmaStages - 1);
    cp_async_commit();
    const uint8_t* stage = sm + ((t - t_lo) % kMmaStages) * C::STAGE;
    const uint32_t ps = (uint32_t)__cvta_generic_to_shared(stage);
    const float* ls = (const float*)(stage + C::PB);
#pragma unroll
    for (int q = 0; q < C::KT / 32; ++q) {
      const int kc = 2 * q + kg;  // 16-column chunk
      uint32_t a[4];
      ldsm_x4(ps + (uint32_t)((16 * rg + (lane & 15)) * C::PSTR + (kc * 16 + (lane >> 4) * 8) * 2), a);
      const int kb = kc * 16 + 2 * tq;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (FM == 2)
          mma_pairs(c[n], a, reinterpret_cast<const uint16_t*>(ls), C::LSTRH, C::NP * C::LSTRH,
                    8 * n + g, kb);
        else if (LKR)
          mma_split(c[n], a, kb, 8 * n + g,
                    [&](int k, int j) { return j < r ? ls[k * r + j] : 0.0f; });
        else
          mma_split(c[n], a, kb, 8 * n + g, [&](int k, int j) { return ls[j * C::LSTRF + k]; });
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  // combine the two K groups, then stage the 64 x NP result tile
  float* red = (float*)(sm + kMmaStages * C::STAGE);
  if (kg == 1) {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[((rg * 32 + lane) * NT + n) * 4 + e] = c[n][e];
  }
  __syncthreads();
  if (kg == 0) {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) c[n][e] += red[((rg * 32 + lane) * NT + n) * 4 + e];
  }
  __syncthreads();
  float* tile = red;  // [64][TSTR]
  if (kg == 0) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = 8 * n + 2 * tq, row = 16 * rg + g;
      tile[row * C::TSTR + col] = c[n][0];
      tile[row * C::TSTR + col + 1] = c[n][1];
      tile[(row + 8) * C::TSTR + col] = c[n][2];
      tile[(row + 8) * C::TSTR + col + 1] = c[n][3];
    }
  }
  __syncthreads();
  if (ksplit > 1) {
    for (int e = threadIdx.x; e < C::RB * C::NP; e += kThreads) {
      const int row = e / C::NP, col = e % C::NP;
      const int64_t m = m0 + row;
      if (m < R) part[((int64_t)ks * R + m) * C::NP + col] = tile[row * C::TSTR + col];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&tickets[rb], 1u) == (unsigned)(ksplit - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    sum_slices<C::NP>(part, R * C::NP, m0, (int)min((int64_t)C::RB, R - m0), C::RB, ksplit, tile,
                      C::TSTR);
    if (threadIdx.x == 0) tickets[rb] = 0;  // ready for the next launch
    __syncthreads();
  }
  for (int e = threadIdx.x; e < C::RB * 64; e += kThreads) {
    const int row = e >> 6, col = e & 63;
    const int64_t m = m0 + row;
    if (m >= R) continue;
    const float v = col < r ? tile[row * C::TSTR + col] : 0.0f;
    if (col < r) out[m * r + col] = v;
    if (out_pad) out_pad[m * 64 + col] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// coldot on the tensor cores: out(j, n) = s sum_m aux[m, j] P[m, n].
// D[n, j] = sum_m P^T[n, m] aux[m, j]: the P tile [64 rows x 128 columns]
// is read transposed by ldmatrix.trans.  Block = 8 warps x 16 columns;
// grid = column blocks x row splits, the last block of a column block to
// finish (ticket) adds the split partials in split order, scales by s and
// writes dA as [r x N] (out_nr = 0) or dB as [N x r] (out_nr = 1).
// Aux modes: FM 0 fp32 [R x r]; FM 2 split into bf16 hi / lo rows (as for
// the rowdot factor).
template <int NT, int FM>
struct ColMma {
  static constexpr int NC = 128, RT = colmma_rt(NT);
  static constexpr int NP = 8 * NT;
  static constexpr int PSTR = NC * 2 + 16;
  static constexpr int PB = RT * PSTR;
  static constexpr int ASTRH = RT + 8;                 // bf16 per split row (FM 2)
  static constexpr int AB = FM == 2 ? 2 * NP * ASTRH * 2 : RT * NP * 4;  // aux tile
  static constexpr int STAGE = PB + AB;
  static constexpr int TSTR = NP + 1;
  static constexpr int TILE = NC * TSTR * 4;
  static constexpr int SMEM = kMmaStages * STAGE + TILE;
};

// One coldot product: out(j, n) = s sum_m aux[m, j] P[m, n] over column
// blocks x row splits, with its own partial buffer and ticket counters.
struct ColJob {
  const __nv_bfloat16* P;
  int64_t R, N;
  const float* aux;
  int64_t astride;
  int r, col_blocks, splits, tiles_per_split;
  float s;
  int out_nr;
  float* out;
  float* part;
  unsigned* tickets;
};

// Grid = the blocks of job a, then those of job b (col_blocks = 0: none):
// the two side products of a backward pass, dA and dB, share one launch.
template <int NT, int FM>
__global__ void __launch_bounds__(kThreads) coldot_mma_kernel(const ColJob ja, const ColJob jb) {
  // the input-gradient GEMM queued next may start its weight stream now
  if (threadIdx.x == 0) griddep_launch_dependents();
  using C = ColMma<NT, FM>;
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ int s_last;
  const int na = ja.col_blocks * ja.splits;
  const bool first = (int)blockIdx.x < na;
  const ColJob& jo = first ? ja : jb;
  const int lb = first ? (int)blockIdx.x : (int)blockIdx.x - na;
  const __nv_bfloat16* __restrict__ P = jo.P;
  const int64_t R = jo.R, N = jo.N, astride = jo.astride;
  const float* __restrict__ aux = jo.aux;
  const int r = jo.r, splits = jo.splits, tiles_per_split = jo.tiles_per_split;
  const float s = jo.s;
  const int out_nr = jo.out_nr;
  float* __restrict__ out = jo.out;
  float* __restrict__ part = jo.part;
  unsigned* __restrict__ tickets = jo.tickets;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = lb % jo.col_blocks, sp = lb / jo.col_blocks;
  const int64_t n0 = (int64_t)cb * C::NC;
  const int ntiles = (int)((R + C::RT - 1) / C::RT);
  const int t_lo = sp * tiles_per_split, t_hi = min(ntiles, t_lo + tiles_per_split);

  auto issue = [&](int t) {
    const uint32_t ps = (uint32_t)__cvta_generic_to_shared(sm + ((t - t_lo) % kMmaStages) * C::STAGE);
    const uint32_t as = ps + C::PB;
    const int64_t mt = (int64_t)t * C::RT;
#pragma unroll
    for (int i = 0; i < C::RT * 16 / kThreads; ++i) {  // RT rows x 16 chunks
      const int c = threadIdx.x + kThreads * i, row = c >> 4, ch = c & 15;
      const int64_t m = mt + row, n = n0 + ch * 8;
      const int64_t rem = (N - n) * 2;
      const uint32_t nb = (m < R && rem > 0) ? (uint32_t)min((int64_t)16, rem) : 0u;
      cp_async16(ps + (uint32_t)(row * C::PSTR + ch * 16), nb ? (const void*)(P + m * N + n) : (const void*)P, nb);
    }
    if (FM == 2) {  // split rows: 2 x NP rows of RT bf16
      const uint16_t* As = reinterpret_cast<const uint16_t*>(aux);
      for (int c = threadIdx.x; c < 2 * C::NP * (C::RT / 8); c += kThreads) {
        const int row = c / (C::RT / 8), ch = c % (C::RT / 8);
        const int64_t m = mt + ch * 8;
        const int64_t rem = (astride - m) * 2;
        const uint32_t nb = rem > 0 ? (uint32_t)min((int64_t)16, rem) : 0u;
        cp_async16(as + (uint32_t)(row * C::ASTRH + ch * 8) * 2,
                   nb ? (const void*)(As + row * astride + m) : (const void*)As, nb);
      }
    } else {
      const int64_t base = mt * r, total = R * (int64_t)r;  // contiguous [RT x r]
      const int nch = (C::RT * r) / 4;
      for (int c = threadIdx.x; c < nch; c += kThreads) {
        const int64_t e = base + (int64_t)c * 4;
        const int64_t rem = (total - e) * 4;
        const uint32_t nb = rem > 0 ? (uint32_t)min((int64_t)16, rem) : 0u;
        cp_async16(as + (uint32_t)c * 16, nb ? (const void*)(aux + e) : (const void*)aux, nb);
      }
    }
  };

  const int g = lane >> 2, tq = lane & 3;
  float c[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) c[n][0] = c[n][1] = c[n][2] = c[n][3] = 0.0f;
#pragma unroll
  for (int i = 0; i < kMmaStages - 1; ++i) {
    if (t_lo + i < t_hi) issue(t_lo + i);
    cp_async_commit();
  }
  // ldmatrix.trans source rows: matrix q = lane / 8 covers columns
  // 8 (q & 1) .. +7 and rows 8 (q >> 1) .. +7 of the 16 x 16 block
  const int lrow = (lane & 7) + 8 * (lane >> 4), lcol = 16 * warp + 8 * ((lane >> 3) & 1);
  for (int t = t_lo; t < t_hi; ++t) {
    cp_async_wait<kMmaStages - 2>();
    __syncthreads();
    if (t + kMmaStages - 1 < t_hi) issue(t + kMmaStages - 1);
    cp_async_commit();
    const uint8_t* stage = sm + ((t - t_lo) % kMmaStages) * C::STAGE;
    const uint32_t ps = (uint32_t)__cvta_generic_to_shared(stage);
    const float* as = (const float*)(stage + C::PB);
#pragma unroll
    for (int kc = 0; kc < C::RT / 16; ++kc) {
      uint32_t a[4];
      ldsm_x4_t(ps + (uint32_t)((kc * 16 + lrow) * C::PSTR + lcol * 2), a);
      const int kb = kc * 16 + 2 * tq;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (FM == 2)
          mma_pairs(c[n], a, reinterpret_cast<const uint16_t*>(as), C::ASTRH, C::NP * C::ASTRH,
                    8 * n + g, kb);
        else
          mma_split(c[n], a, kb, 8 * n + g,
                    [&](int k, int j) { return j < r ? as[k * r + j] : 0.0f; });
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  float* tile = (float*)(sm + kMmaStages * C::STAGE);  // [NC][TSTR]: D[n][j]
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int col = 8 * n + 2 * tq, row = 16 * warp + g;
    tile[row * C::TSTR + col] = c[n][0];
    tile[row * C::TSTR + col + 1] = c[n][1];
    tile[(row + 8) * C::TSTR + col] = c[n][2];
    tile[(row + 8) * C::TSTR + col + 1] = c[n][3];
  }
  __syncthreads();
  if (splits > 1) {
    for (int e = threadIdx.x; e < C::NC * C::NP; e += kThreads) {
      const int row = e / C::NP, col = e % C::NP;
      const int64_t n = n0 + row;
      if (n < N) part[((int64_t)sp * N + n) * C::NP + col] = tile[row * C::TSTR + col];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&tickets[cb], 1u) == (unsigned)(splits - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    sum_slices<C::NP>(part, N * C::NP, n0, (int)min((int64_t)C::NC, N - n0), C::NC, splits, tile,
                      C::TSTR);
    if (threadIdx.x == 0) tickets[cb] = 0;  // ready for the next launch
    __syncthreads();
  }
  if (out_nr) {  // dB [N x r]: consecutive threads along j then n
    for (int e = threadIdx.x; e < C::NC * r; e += kThreads) {
      const int row = e / r, j = e % r;
      const int64_t n = n0 + row;
      if (n < N) out[n * r + j] = s * tile[row * C::TSTR + j];
    }
  } else {  // dA [r x N]: consecutive threads along n
    for (int e = threadIdx.x; e < C::NC * r; e += kThreads) {
      const int j = e / C::NC, row = e % C::NC;
      const int64_t n = n0 + row;
      if (n < N) out[(int64_t)j * N + n] = s * tile[row * C::TSTR + j];
    }
  }
}

// dst[j * K + k] = src[k * r + j]: B [K x r] -> B^T [r x K].
__global__ void transpose_kr_kernel(const float* __restrict__ src, int64_t K, int r,
                                    float* __restrict__ dst) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // e = j * K + k
  if (e >= (int64_t)r * K) return;
  const int64_t j = e / K, k = e - j * K;
  dst[e] = src[k * r + j];
}

inline unsigned cdiv(int64_t a, int64_t b) { return (unsigned)((a + b - 1) / b); }

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <typename T, int RMAX, int RW, int KS>
void rowdot_go(unsigned grid, const void* P, int64_t R, int64_t K, const float* L, bool l_is_kr,
               int r, float* out, uint16_t* pad, int row_blocks, PadJob job, cudaStream_t st) {
  rowdot_kernel<T, RMAX, RW, KS><<<grid, kThreads, 0, st>>>((const T*)P, R, K, L, l_is_kr, r, out,
                                                            pad, row_blocks, job);
}

template <typename T, int RMAX>
cudaError_t rowdot_dispatch(const void* P, int64_t R, int64_t K, const float* L, bool l_is_kr,
                            int r, float* out, uint16_t* pad, PadJob job, cudaStream_t st) {
  // Many rows: one column group, RW rows per warp (RW * RMAX <= 64) while
  // that leaves >= one block per SM.  Few rows: the 8 warps split K.
  constexpr int RWMAX = 64 / RMAX < 4 ? 64 / RMAX : 4;
  const int sms = sm_count();
  int row_blocks = 0;
  unsigned grid = 0;
  if (R <= 64) {
    row_blocks = (int)R;  // one row per block, 8 warps over K
    grid = (unsigned)(row_blocks + job.blocks);
    if (grid) rowdot_go<T, RMAX, 1, 8>(grid, P, R, K, L, l_is_kr, r, out, pad, row_blocks, job, st);
  } else {
    int rw = RWMAX;
    while (rw > 1 && (R + 8 * rw - 1) / (8 * rw) < sms) rw /= 2;
    row_blocks = (int)cdiv(R, 8 * rw);
    grid = (unsigned)(row_blocks + job.blocks);
    if (rw >= 4)
      rowdot_go<T, RMAX, RWMAX, 1>(grid, P, R, K, L, l_is_kr, r, out, pad, row_blocks, job, st);
    else if (rw == 2)
      rowdot_go<T, RMAX, (RWMAX >= 2 ? 2 : 1), 1>(grid, P, R, K, L, l_is_kr, r, out, pad,
                                                  row_blocks, job, st);
    else
      rowdot_go<T, RMAX, 1, 1>(grid, P, R, K, L, l_is_kr, r, out, pad, row_blocks, job, st);
  }
  if (grid == 0) return cudaSuccess;
  count_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t rowdot_r(const void* P, int64_t R, int64_t K, const float* L, bool l_is_kr, int r,
                     float* out, uint16_t* pad, PadJob job, cudaStream_t st) {
  if (r <= 8) return rowdot_dispatch<T, 8>(P, R, K, L, l_is_kr, r, out, pad, job, st);
  if (r <= 16) return rowdot_dispatch<T, 16>(P, R, K, L, l_is_kr, r, out, pad, job, st);
  if (r <= 32) return rowdot_dispatch<T, 32>(P, R, K, L, l_is_kr, r, out, pad, job, st);
  return rowdot_dispatch<T, 64>(P, R, K, L, l_is_kr, r, out, pad, job, st);
}

template <typename Kern>
cudaError_t set_smem_once(Kern k, int bytes, bool& done) {
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done = true;
  return e;
}

struct ColPlan {
  int splits;
  int64_t rows_per_split;
  unsigned colblocks;
};

ColPlan col_plan(int64_t R, int64_t N, int r) {
  const int cpt = r <= 8 ? 8 : r <= 16 ? 4 : r <= 32 ? 2 : 1;
  ColPlan c;
  c.colblocks = cdiv(N, 32 * cpt);
  int64_t splits = ((int64_t)sm_count() + c.colblocks - 1) / c.colblocks;  // ~one wave
  const int64_t max_splits = (R + 127) / 128;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  c.rows_per_split = R > 0 ? (R + splits - 1) / splits : 1;
  c.splits = (int)(R > 0 ? (R + c.rows_per_split - 1) / c.rows_per_split : 1);
  return c;
}

template <typename T, int RMAX>
void coldot_launch(const void* P, int64_t R, int64_t N, const float* aux, int r, const ColPlan& c,
                   float s, bool out_nr, float* part, unsigned* tickets, float* out,
                   cudaStream_t st) {
  dim3 grid(c.colblocks, (unsigned)c.splits);
  coldot_kernel<T, RMAX><<<grid, kThreads, 0, st>>>((const T*)P, R, N, aux, r, c.rows_per_split,
                                                    c.splits, s, out_nr ? 1 : 0, part, tickets,
                                                    out);
}

template <typename T>
void coldot_r(const void* P, int64_t R, int64_t N, const float* aux, int r, const ColPlan& c,
              float s, bool out_nr, float* part, unsigned* tickets, float* out, cudaStream_t st) {
  if (r <= 8) coldot_launch<T, 8>(P, R, N, aux, r, c, s, out_nr, part, tickets, out, st);
  else if (r <= 16) coldot_launch<T, 16>(P, R, N, aux, r, c, s, out_nr, part, tickets, out, st);
  else if (r <= 32) coldot_launch<T, 32>(P, R, N, aux, r, c, s, out_nr, part, tickets, out, st);
  else coldot_launch<T, 64>(P, R, N, aux, r, c, s, out_nr, part, tickets, out, st);
}

struct MmaPlan {
  int blocks;          // row blocks (rowdot) or column blocks (coldot)
  int splits;          // K splits (rowdot) or row splits (coldot)
  int tiles_per_split;
};

// ~two waves of 256-thread blocks; a split only where the blocks alone
// leave SMs idle, and only with ticket counters to spare.
MmaPlan mma_plan(int64_t blocks, int64_t ntiles, bool can_split) {
  MmaPlan pl;
  pl.blocks = (int)blocks;
  int64_t splits = 1;
  if (can_split && blocks > 0 && blocks <= kMaxTickets && blocks < sm_count()) {
    splits = (2 * (int64_t)sm_count()) / blocks;
    if (splits > ntiles) splits = ntiles;
    if (splits < 1) splits = 1;
  }
  pl.tiles_per_split = (int)((ntiles + splits - 1) / splits);
  if (pl.tiles_per_split < 1) pl.tiles_per_split = 1;
  pl.splits = (int)((ntiles + pl.tiles_per_split - 1) / pl.tiles_per_split);
  if (pl.splits < 1) pl.splits = 1;
  return pl;
}

int rank_tiles(int r) { return r <= 8 ? 1 : r <= 16 ? 2 : r <= 32 ? 4 : 8; }

MmaPlan rowdot_mma_plan(int64_t R, int64_t K, int r, bool can_split) {
  return mma_plan(cdiv(R, 64), cdiv(K, rowmma_kt(rank_tiles(r))), can_split);
}
MmaPlan coldot_mma_plan(int64_t R, int64_t N, int r, bool can_split) {
  return mma_plan(cdiv(N, 128), cdiv(R, colmma_rt(rank_tiles(r))), can_split);
}

bool rowdot_mma_ok(const void* P, bool bf16, int64_t K, const float* L) {
  return bf16 && (K % 8) == 0 && ((uintptr_t)P % 16) == 0 && ((uintptr_t)L % 16) == 0;
}

template <int NT, int FM>
cudaError_t rowdot_mma_go(const __nv_bfloat16* P, int64_t R, int64_t K, const float* L,
                          int64_t lstride, int r, const MmaPlan& pl, float* out, uint16_t* pad,
                          float* part, unsigned* tickets, PadJob job, cudaStream_t st) {
  using C = RowMma<NT, FM>;
  static bool attr = false;
  auto kern = rowdot_mma_kernel<NT, FM>;
  cudaError_t e = set_smem_once(kern, C::SMEM, attr);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(pl.blocks * pl.splits + job.blocks);
  if (grid == 0) return cudaSuccess;
  kern<<<grid, kThreads, C::SMEM, st>>>(P, R, K, L, lstride, r, pl.blocks, pl.splits,
                                        pl.tiles_per_split, out, pad, part, tickets, job);
  count_launch();
  return cudaGetLastError();
}

template <int FM>
cudaError_t rowdot_mma_r(const __nv_bfloat16* P, int64_t R, int64_t K, const float* L,
                         int64_t lstride, int r, const MmaPlan& pl, float* out, uint16_t* pad,
                         float* part, unsigned* tickets, PadJob job, cudaStream_t st) {
  switch (rank_tiles(r)) {
    case 1: return rowdot_mma_go<1, FM>(P, R, K, L, lstride, r, pl, out, pad, part, tickets, job, st);
    case 2: return rowdot_mma_go<2, FM>(P, R, K, L, lstride, r, pl, out, pad, part, tickets, job, st);
    case 4: return rowdot_mma_go<4, FM>(P, R, K, L, lstride, r, pl, out, pad, part, tickets, job, st);
    default: return rowdot_mma_go<8, FM>(P, R, K, L, lstride, r, pl, out, pad, part, tickets, job, st);
  }
}

// Split the r-wide factor of one product into bf16 hi / lo rows in `dst`
// (row length ld = extent rounded up to 8).
cudaError_t split_factor(const float* src, int64_t extent, int r, bool nr, uint16_t* dst,
                         int64_t* ld, cudaStream_t st) {
  const int NP = 8 * rank_tiles(r);
  *ld = (extent + 7) / 8 * 8;
  const int64_t pairs = (int64_t)NP * *ld / 2;
  split_factor_kernel<<<cdiv(pairs, 256), 256, 0, st>>>(src, extent, r, nr ? 1 : 0, NP, *ld, dst);
  count_launch();
  return cudaGetLastError();
}

ColJob col_job(const __nv_bfloat16* P, int64_t R, int64_t N, const float* aux, int64_t astride,
               int r, const MmaPlan& pl, float s, bool out_nr, float* out, float* part,
               unsigned* tickets) {
  ColJob j;
  j.P = P;
  j.R = R;
  j.N = N;
  j.aux = aux;
  j.astride = astride;
  j.r = r;
  j.col_blocks = pl.blocks;
  j.splits = pl.splits;
  j.tiles_per_split = pl.tiles_per_split;
  j.s = s;
  j.out_nr = out_nr ? 1 : 0;
  j.out = out;
  j.part = part;
  j.tickets = tickets;
  return j;
}

template <int NT, int FM>
cudaError_t coldot_mma_pair_go(const ColJob& ja, const ColJob& jb, cudaStream_t st) {
  using C = ColMma<NT, FM>;
  static bool attr = false;
  auto kern = coldot_mma_kernel<NT, FM>;
  cudaError_t e = set_smem_once(kern, C::SMEM, attr);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(ja.col_blocks * ja.splits + jb.col_blocks * jb.splits);
  kern<<<grid, kThreads, C::SMEM, st>>>(ja, jb);
  count_launch();
  return cudaGetLastError();
}

template <int NT, int FM>
cudaError_t coldot_mma_go(const __nv_bfloat16* P, int64_t R, int64_t N, const float* aux,
                          int64_t astride, int r, const MmaPlan& pl, float s, bool out_nr,
                          float* out, float* part, unsigned* tickets, cudaStream_t st) {
  ColJob none = {};
  return coldot_mma_pair_go<NT, FM>(
      col_job(P, R, N, aux, astride, r, pl, s, out_nr, out, part, tickets), none, st);
}


}  // namespace

cudaError_t launch_rowdot(const void* P, bool bf16, int64_t R, int64_t K, const float* L,
                          bool l_is_kr, int32_t r, float* out, cudaStream_t st, uint16_t* pad,
                          const float* side_src, int64_t side_extent, int side_mode,
                          float side_mul, uint16_t* side_dst, float* lt_ws, float* part_ws,
                          unsigned* tickets, uint16_t* split_ws) {
  PadJob job{side_src, side_dst, side_extent, r, side_mode, side_mul, 0};
  if (side_dst && side_extent > 0) job.blocks = (int)cdiv(64 * side_extent, kThreads * 8);
  if (R > 0 && rowdot_mma_ok(P, bf16, K, L)) {  // tensor cores, either factor layout
    const MmaPlan pl = rowdot_mma_plan(R, K, r, part_ws != nullptr && tickets != nullptr);
    const __nv_bfloat16* Pb = (const __nv_bfloat16*)P;
    // A [K x r] factor is read in place, except over large activations
    // with scratch for it: there one transposing launch (r*K floats) is
    // repaid by the faster row-major factor path (measured 25-40% on
    // 8192 x 4096 and 16384 x 17408 activations).
    // Above rank 8, one small launch splits the factor into bf16 hi / lo
    // rows once, instead of every warp of every block splitting it again.
    if (split_ws && rank_tiles(r) >= 2 && ((uintptr_t)split_ws % 16) == 0) {
      int64_t ld = 0;
      cudaError_t e = split_factor(L, K, r, l_is_kr, split_ws, &ld, st);
      if (e != cudaSuccess) return e;
      return rowdot_mma_r<2>(Pb, R, K, (const float*)split_ws, ld, r, pl, out, pad, part_ws,
                             tickets, job, st);
    }
    if (l_is_kr && lt_ws && R * K >= (int64_t)32 << 20 && ((uintptr_t)lt_ws % 16) == 0) {
      transpose_kr_kernel<<<cdiv((int64_t)r * K, 256), 256, 0, st>>>(L, K, r, lt_ws);
      count_launch();
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      return rowdot_mma_r<0>(Pb, R, K, lt_ws, 0, r, pl, out, pad, part_ws, tickets, job, st);
    }
    if (l_is_kr) return rowdot_mma_r<1>(Pb, R, K, L, 0, r, pl, out, pad, part_ws, tickets, job, st);
    return rowdot_mma_r<0>(Pb, R, K, L, 0, r, pl, out, pad, part_ws, tickets, job, st);
  }
  // With scratch for it, a factor given as [K x r] is transposed first so
  // every path below reads factor rows ([r x K]) contiguously.
  const float* Lr = L;
  bool lkr = l_is_kr;
  if (l_is_kr && lt_ws && R > 0) {
    transpose_kr_kernel<<<cdiv((int64_t)r * K, 256), 256, 0, st>>>(L, K, r, lt_ws);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Lr = lt_ws;
    lkr = false;
  }
  if (bf16) return rowdot_r<__nv_bfloat16>(P, R, K, Lr, lkr, r, out, pad, job, st);
  return rowdot_r<float>(P, R, K, Lr, lkr, r, out, pad, job, st);
}

namespace {

bool coldot_mma_ok(const void* P, bool bf16, int64_t R, int64_t N, const float* aux) {
  return bf16 && R > 0 && (N % 8) == 0 && ((uintptr_t)P % 16) == 0 && ((uintptr_t)aux % 16) == 0;
}

}  // namespace

size_t adapter_split_ws(int64_t extent, int32_t r) {
  if (rank_tiles(r) < 2) return 0;
  return align_up((size_t)2 * 8 * rank_tiles(r) * (size_t)((extent + 7) / 8 * 8) * 2, 256);
}

size_t rowdot_ws(int64_t R, int64_t K, int32_t r) {
  const MmaPlan pl = rowdot_mma_plan(R, K, r, true);
  return pl.splits > 1 ? align_up((size_t)pl.splits * (size_t)R * 8 * rank_tiles(r) * 4, 256) : 0;
}

// Workspace: the larger of the tensor-core path (split partials) and the
// FMA path (tickets + slice sums).
size_t coldot_ws(int64_t R, int64_t N, int32_t r) {
  const ColPlan c = col_plan(R, N, r);
  size_t a = c.splits <= 1 ? 0
                           : align_up((size_t)c.colblocks * 4, 256) +
                                 align_up((size_t)c.splits * (size_t)r * (size_t)N * 4, 256);
  const MmaPlan mp = coldot_mma_plan(R, N, r, true);
  const size_t b =
      mp.splits > 1 ? align_up((size_t)mp.splits * (size_t)N * 8 * rank_tiles(r) * 4, 256) : 0;
  return a > b ? a : b;
}

cudaError_t launch_coldot(const void* P, bool bf16, int64_t R, int64_t N, const float* aux,
                          int32_t r, float s, bool out_nr, float* out, void* ws,
                          cudaStream_t st, unsigned* tickets, uint16_t* split_ws) {
  if (N == 0) return cudaSuccess;
  if (R == 0) return cudaMemsetAsync(out, 0, (size_t)r * (size_t)N * 4, st);
  if (coldot_mma_ok(P, bf16, R, N, aux)) {  // tensor cores
    const MmaPlan pl = coldot_mma_plan(R, N, r, tickets != nullptr);
    const __nv_bfloat16* Pb = (const __nv_bfloat16*)P;
    float* part = (float*)ws;
    if (split_ws && rank_tiles(r) >= 2 && ((uintptr_t)split_ws % 16) == 0) {
      int64_t ld = 0;
      cudaError_t e = split_factor(aux, R, r, true, split_ws, &ld, st);
      if (e != cudaSuccess) return e;
      const float* sp = (const float*)split_ws;
      switch (rank_tiles(r)) {
        case 2: return coldot_mma_go<2, 2>(Pb, R, N, sp, ld, r, pl, s, out_nr, out, part, tickets, st);
        case 4: return coldot_mma_go<4, 2>(Pb, R, N, sp, ld, r, pl, s, out_nr, out, part, tickets, st);
        default: return coldot_mma_go<8, 2>(Pb, R, N, sp, ld, r, pl, s, out_nr, out, part, tickets, st);
      }
    }
    switch (rank_tiles(r)) {
      case 1: return coldot_mma_go<1, 0>(Pb, R, N, aux, 0, r, pl, s, out_nr, out, part, tickets, st);
      case 2: return coldot_mma_go<2, 0>(Pb, R, N, aux, 0, r, pl, s, out_nr, out, part, tickets, st);
      case 4: return coldot_mma_go<4, 0>(Pb, R, N, aux, 0, r, pl, s, out_nr, out, part, tickets, st);
      default: return coldot_mma_go<8, 0>(Pb, R, N, aux, 0, r, pl, s, out_nr, out, part, tickets, st);
    }
  }
  const ColPlan c = col_plan(R, N, r);
  unsigned* slice_tickets = (unsigned*)ws;
  float* part = (float*)((char*)ws + align_up((size_t)c.colblocks * 4, 256));
  if (c.splits > 1) {
    cudaError_t e = cudaMemsetAsync(slice_tickets, 0, (size_t)c.colblocks * 4, st);
    if (e != cudaSuccess) return e;
  }
  if (bf16)
    coldot_r<__nv_bfloat16>(P, R, N, aux, r, c, s, out_nr, part, slice_tickets, out, st);
  else
    coldot_r<float>(P, R, N, aux, r, c, s, out_nr, part, slice_tickets, out, st);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_coldot_pair(const void* PA, int64_t NA, const float* auxA, bool out_nrA,
                               float* outA, void* wsA, uint16_t* splitA, const void* PB,
                               int64_t NB, const float* auxB, bool out_nrB, float* outB, void* wsB,
                               uint16_t* splitB, int64_t R, int32_t r, float s, cudaStream_t st,
                               unsigned* tickets, bool* done) {
  *done = false;
  if (R <= 0 || NA <= 0 || NB <= 0 || !tickets) return cudaSuccess;
  if (!coldot_mma_ok(PA, true, R, NA, auxA) || !coldot_mma_ok(PB, true, R, NB, auxB))
    return cudaSuccess;
  const MmaPlan pa = coldot_mma_plan(R, NA, r, true), pb = coldot_mma_plan(R, NB, r, true);
  if (pa.blocks + pb.blocks > kMaxTickets) return cudaSuccess;
  const __nv_bfloat16* A = (const __nv_bfloat16*)PA;
  const __nv_bfloat16* B = (const __nv_bfloat16*)PB;
  *done = true;
  if (rank_tiles(r) >= 2 && splitA && splitB && ((uintptr_t)splitA % 16) == 0 &&
      ((uintptr_t)splitB % 16) == 0) {
    int64_t lda = 0, ldb = 0;
    cudaError_t e = split_factor(auxA, R, r, true, splitA, &lda, st);
    if (e == cudaSuccess) e = split_factor(auxB, R, r, true, splitB, &ldb, st);
    if (e != cudaSuccess) return e;
    const ColJob ja = col_job(A, R, NA, (const float*)splitA, lda, r, pa, s, out_nrA, outA,
                              (float*)wsA, tickets);
    const ColJob jb = col_job(B, R, NB, (const float*)splitB, ldb, r, pb, s, out_nrB, outB,
                              (float*)wsB, tickets + pa.blocks);
    switch (rank_tiles(r)) {
      case 2: return coldot_mma_pair_go<2, 2>(ja, jb, st);
      case 4: return coldot_mma_pair_go<4, 2>(ja, jb, st);
      default: return coldot_mma_pair_go<8, 2>(ja, jb, st);
    }
  }
  const ColJob ja = col_job(A, R, NA, auxA, 0, r, pa, s, out_nrA, outA, (float*)wsA, tickets);
  const ColJob jb = col_job(B, R, NB, auxB, 0, r, pb, s, out_nrB, outB, (float*)wsB,
                            tickets + pa.blocks);
  switch (rank_tiles(r)) {
    case 1: return coldot_mma_pair_go<1, 0>(ja, jb, st);
    case 2: return coldot_mma_pair_go<2, 0>(ja, jb, st);
    case 4: return coldot_mma_pair_go<4, 0>(ja, jb, st);
    default: return coldot_mma_pair_go<8, 0>(ja, jb, st);
  }
}

}  // namespace qlora
