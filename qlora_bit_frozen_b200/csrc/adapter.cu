// adapter.cu -- the LoRA side products of the QLoRA linear layer, in fp32.
//
// "QLoRA on Mac", "Design / Q-LoRA layer": the adapter branch is
// (alpha/r)(x A^T) B^T with fp32 A, B.  Forward needs U = X A^T; the
// backward chain rule needs V = dY B, dA = s V^T X and dB = s dY^T U.
// All four read one activation matrix once and touch an r-wide factor, so
// they are bound by HBM bandwidth on X / dY, not by arithmetic:
//
//  * rowdot: out[m, j] = sum_k P[m, k] L(k, j) (U with L = A^T, V with L = B).
//    Each warp owns 2 rows; lanes stride K four elements at a time; a
//    256-wide chunk of L is staged in shared memory once per block and read
//    as conflict-free float4; the 32 lane partials are combined with a
//    butterfly.  Also writes the bf16 copy zero-padded to 64 columns that
//    the tensor-core kernels use as their extra K step.
//  * coldot: partial[split][j][n] = sum over the split's rows of
//    aux[m, j] P[m, n] (dA with aux = V, P = X; dB with aux = U, P = dY).
//    One thread per two columns, the aux rows broadcast from shared memory;
//    the splits are then summed in split order (deterministic) and scaled
//    by s, writing dA as [r x I] and dB as [O x r].
#include "common.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int kRowThreads = 256;
constexpr int kRowsPerWarp = 2;
constexpr int kRowsPerBlock = kRowsPerWarp * (kRowThreads / 32);

template <typename T>
struct Vec4;
template <>
struct Vec4<float> {
  __device__ static void load(const float* p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
};
template <>
struct Vec4<__nv_bfloat16> {
  __device__ static void load(const __nv_bfloat16* p, float (&x)[4]) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
    x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  }
};

// K chunk staged per block: RMAX x KC floats stay within 32 KB.
template <int RMAX>
constexpr int kc_for() {
  return RMAX <= 32 ? 256 : 128;
}

template <typename T, int RMAX>
__global__ void __launch_bounds__(kRowThreads) rowdot_kernel(const T* __restrict__ P, int64_t R,
                                                             int64_t K, const float* __restrict__ L,
                                                             int l_is_kr, int r,
                                                             float* __restrict__ out,
                                                             uint16_t* __restrict__ out_pad) {
  constexpr int kKC = kc_for<RMAX>();
  __shared__ __align__(16) float Ls[RMAX * kKC];  // Ls[j * kKC + k]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = ((int64_t)blockIdx.x * (kRowThreads / 32) + warp) * kRowsPerWarp;
  const bool vec = (K % 4) == 0;
  float acc[kRowsPerWarp][RMAX];
#pragma unroll
  for (int q = 0; q < kRowsPerWarp; ++q)
#pragma unroll
    for (int j = 0; j < RMAX; ++j) acc[q][j] = 0.0f;

  for (int64_t k0 = 0; k0 < K; k0 += kKC) {
    const int kc = (int)min((int64_t)kKC, K - k0);
    __syncthreads();
    for (int e = threadIdx.x; e < kc * r; e += kRowThreads) {
      int j, k;
      float v;
      if (l_is_kr) {
        k = e / r;
        j = e - k * r;
        v = L[(k0 + k) * r + j];
      } else {
        j = e / kc;
        k = e - j * kc;
        v = L[(int64_t)j * K + k0 + k];
      }
      Ls[j * kKC + k] = v;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kKC / 128; ++t) {
      const int kk = t * 128 + lane * 4;
      if (kk >= kc) break;
      float x[kRowsPerWarp][4];
#pragma unroll
      for (int q = 0; q < kRowsPerWarp; ++q) {
        const int64_t m = row0 + q;
        if (m < R && vec && kk + 4 <= kc) {
          Vec4<T>::load(P + m * K + k0 + kk, x[q]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            x[q][e] = (m < R && kk + e < kc) ? to_f32<T>(P[m * K + k0 + kk + e]) : 0.0f;
        }
      }
      const int kmax = kc - kk;  // entries of Ls past kc are stale: mask them
#pragma unroll
      for (int j = 0; j < RMAX; ++j) {
        if (j < r) {
          const float4 l = *reinterpret_cast<const float4*>(&Ls[j * kKC + kk]);
          const float lv[4] = {l.x, kmax > 1 ? l.y : 0.0f, kmax > 2 ? l.z : 0.0f,
                               kmax > 3 ? l.w : 0.0f};
#pragma unroll
          for (int q = 0; q < kRowsPerWarp; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[q][j] = fmaf(x[q][e], lv[e], acc[q][j]);
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kRowsPerWarp; ++q)
#pragma unroll
    for (int j = 0; j < RMAX; ++j)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[q][j] += __shfl_xor_sync(0xffffffffu, acc[q][j], o);
#pragma unroll
  for (int q = 0; q < kRowsPerWarp; ++q) {
    const int64_t m = row0 + q;
    if (m >= R) continue;
    // lane l writes columns l and l + 32 (selected without dynamic indexing)
    float a0 = 0.0f, a1 = 0.0f;
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

constexpr int kColThreads = 256;
constexpr int kColsPerThread = 2;
constexpr int kColsPerBlock = kColThreads * kColsPerThread;
constexpr int kMC = 64;  // aux rows staged per chunk

template <typename T, int RMAX>
__global__ void __launch_bounds__(kColThreads) coldot_kernel(const T* __restrict__ P, int64_t R,
                                                             int64_t N, const float* __restrict__ aux,
                                                             int r, int64_t rows_per_split,
                                                             float* __restrict__ part) {
  __shared__ __align__(16) float As[kMC * RMAX];  // As[mm * RMAX + j]
  const int64_t n = ((int64_t)blockIdx.x * kColThreads + threadIdx.x) * kColsPerThread;
  const int64_t m_lo = (int64_t)blockIdx.y * rows_per_split;
  const int64_t m_hi = min(R, m_lo + rows_per_split);
  const bool pair = (n + 1 < N) && ((N & 1) == 0);
  float acc[kColsPerThread][RMAX];
#pragma unroll
  for (int c = 0; c < kColsPerThread; ++c)
#pragma unroll
    for (int j = 0; j < RMAX; ++j) acc[c][j] = 0.0f;
  for (int64_t m0 = m_lo; m0 < m_hi; m0 += kMC) {
    const int mc = (int)min((int64_t)kMC, m_hi - m0);
    __syncthreads();
    for (int e = threadIdx.x; e < mc * RMAX; e += kColThreads) {
      const int mm = e / RMAX, j = e - mm * RMAX;
      As[e] = j < r ? aux[(m0 + mm) * r + j] : 0.0f;
    }
    __syncthreads();
    if (n < N) {
      for (int mm = 0; mm < mc; ++mm) {
        float p0, p1 = 0.0f;
        const T* row = P + (m0 + mm) * N + n;
        if (pair) {
          if constexpr (sizeof(T) == 2) {
            const uint32_t v = *reinterpret_cast<const uint32_t*>(row);
            p0 = __uint_as_float(v << 16);
            p1 = __uint_as_float(v & 0xFFFF0000u);
          } else {
            const float2 v = *reinterpret_cast<const float2*>(row);
            p0 = v.x;
            p1 = v.y;
          }
        } else {
          p0 = to_f32<T>(row[0]);
          if (n + 1 < N) p1 = to_f32<T>(row[1]);
        }
#pragma unroll
        for (int j = 0; j < RMAX; j += 4) {
          const float4 a = *reinterpret_cast<const float4*>(&As[mm * RMAX + j]);
          acc[0][j] = fmaf(a.x, p0, acc[0][j]);
          acc[0][j + 1] = fmaf(a.y, p0, acc[0][j + 1]);
          acc[0][j + 2] = fmaf(a.z, p0, acc[0][j + 2]);
          acc[0][j + 3] = fmaf(a.w, p0, acc[0][j + 3]);
          acc[1][j] = fmaf(a.x, p1, acc[1][j]);
          acc[1][j + 1] = fmaf(a.y, p1, acc[1][j + 1]);
          acc[1][j + 2] = fmaf(a.z, p1, acc[1][j + 2]);
          acc[1][j + 3] = fmaf(a.w, p1, acc[1][j + 3]);
        }
      }
    }
  }
  float* dst = part + (int64_t)blockIdx.y * r * N;
#pragma unroll
  for (int j = 0; j < RMAX; ++j) {
    if (j < r) {
      if (n < N) dst[(int64_t)j * N + n] = acc[0][j];
      if (n + 1 < N) dst[(int64_t)j * N + n + 1] = acc[1][j];
    }
  }
}

// out = s * sum over splits (in order) of part[split][j][n];
// out_nr == 0: out[j * N + n] (dA);  1: out[n * r + j] (dB).
__global__ void coldot_reduce_kernel(const float* __restrict__ part, int splits, int64_t N, int r,
                                     float s, int out_nr, float* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // e = j * N + n
  if (e >= (int64_t)r * N) return;
  float acc = 0.0f;
  for (int k = 0; k < splits; ++k) acc += part[(int64_t)k * r * N + e];
  const int64_t j = e / N, n = e - j * N;
  out[out_nr ? n * r + j : e] = s * acc;
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

template <typename T, int RMAX>
void rowdot_launch(const void* P, int64_t R, int64_t K, const float* L, bool l_is_kr, int r,
                   float* out, uint16_t* pad, cudaStream_t st) {
  rowdot_kernel<T, RMAX><<<cdiv(R, kRowsPerBlock), kRowThreads, 0, st>>>(
      (const T*)P, R, K, L, l_is_kr ? 1 : 0, r, out, pad);
}

template <typename T, int RMAX>
void coldot_launch(const void* P, int64_t R, int64_t N, const float* aux, int r, int64_t rps,
                   int splits, float* part, cudaStream_t st) {
  dim3 grid(cdiv(N, kColsPerBlock), (unsigned)splits);
  coldot_kernel<T, RMAX><<<grid, kColThreads, 0, st>>>((const T*)P, R, N, aux, r, rps, part);
}

struct ColPlan {
  int splits;
  int64_t rows_per_split;
};

ColPlan col_plan(int64_t R, int64_t N) {
  ColPlan c;
  const int64_t colblocks = (N + kColsPerBlock - 1) / kColsPerBlock;
  int64_t splits = (2 * (int64_t)sm_count() + colblocks - 1) / colblocks;
  if (splits < 1) splits = 1;
  int64_t rps = (R + splits - 1) / splits;
  rps = (rps + kMC - 1) / kMC * kMC;
  if (rps < kMC) rps = kMC;
  c.rows_per_split = rps;
  c.splits = (int)(R > 0 ? (R + rps - 1) / rps : 1);
  return c;
}

}  // namespace

// out[m, j] = sum_k P[m, k] * L(k, j);  L(k, j) = L[k*r + j] if l_is_kr else L[j*K + k].
// pad (nullable): bf16 copy [R x 64], columns r..63 zero.
cudaError_t launch_rowdot(const void* P, bool bf16, int64_t R, int64_t K, const float* L,
                          bool l_is_kr, int32_t r, float* out, cudaStream_t st, uint16_t* pad) {
  if (R == 0) return cudaSuccess;
  if (bf16) {
    if (r <= 8) rowdot_launch<__nv_bfloat16, 8>(P, R, K, L, l_is_kr, r, out, pad, st);
    else if (r <= 16) rowdot_launch<__nv_bfloat16, 16>(P, R, K, L, l_is_kr, r, out, pad, st);
    else if (r <= 32) rowdot_launch<__nv_bfloat16, 32>(P, R, K, L, l_is_kr, r, out, pad, st);
    else rowdot_launch<__nv_bfloat16, 64>(P, R, K, L, l_is_kr, r, out, pad, st);
  } else {
    if (r <= 8) rowdot_launch<float, 8>(P, R, K, L, l_is_kr, r, out, pad, st);
    else if (r <= 16) rowdot_launch<float, 16>(P, R, K, L, l_is_kr, r, out, pad, st);
    else if (r <= 32) rowdot_launch<float, 32>(P, R, K, L, l_is_kr, r, out, pad, st);
    else rowdot_launch<float, 64>(P, R, K, L, l_is_kr, r, out, pad, st);
  }
  count_launch();
  return cudaGetLastError();
}

size_t coldot_ws(int64_t R, int64_t N, int32_t r) {
  const ColPlan c = col_plan(R, N);
  return align_up((size_t)c.splits * (size_t)r * (size_t)N * 4, 256);
}

// out = s * aux^T P:  out(j, n) = s * sum_m aux[m, j] * P[m, n];
// out_nr == false: out is [r x N] (dA);  true: out is [N x r] (dB).
cudaError_t launch_coldot(const void* P, bool bf16, int64_t R, int64_t N, const float* aux,
                          int32_t r, float s, bool out_nr, float* out, void* ws,
                          cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  const ColPlan c = col_plan(R, N);
  float* part = (float*)ws;
  if (R == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, (size_t)r * (size_t)N * 4, st);
    return e;
  }
  if (bf16) {
    if (r <= 8) coldot_launch<__nv_bfloat16, 8>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
    else if (r <= 16) coldot_launch<__nv_bfloat16, 16>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
    else if (r <= 32) coldot_launch<__nv_bfloat16, 32>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
    else coldot_launch<__nv_bfloat16, 64>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
  } else {
    if (r <= 8) coldot_launch<float, 8>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
    else if (r <= 16) coldot_launch<float, 16>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
    else if (r <= 32) coldot_launch<float, 32>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
    else coldot_launch<float, 64>(P, R, N, aux, r, c.rows_per_split, c.splits, part, st);
  }
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  coldot_reduce_kernel<<<cdiv((int64_t)r * N, 256), 256, 0, st>>>(part, c.splits, N, r, s,
                                                                    out_nr ? 1 : 0, out);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
