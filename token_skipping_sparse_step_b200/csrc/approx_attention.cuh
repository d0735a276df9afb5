// Saliency-aware approximate attention of one layer ("DyLLM: Efficient
// Diffusion LLM Inference via Saliency-based Token Selection and Partial
// Attention", technical summary section 2.B.2): the rows whose values moved
// since the previous step (the salient ones) get exact attention rows, and
// every other row moves its cached context by the change of those values
// weighted by its cached attention probabilities, C_i += sum_a P_{i,j_a} dV_{j_a}
// (per head), at O(L x |changed|) instead of O(L^2).
//
// Two kernels on one stream, in this order:
//   approx_update_kernel      every row i: C_i += sum over the changed rows of
//                             P[i, j_a] (V - V_prev)[j_a]  (reads the cached P)
//   approx_exact_rows_kernel  every changed row: exact softmax(q k^T / sqrt(hd))
//                             over all L keys, its P row rewritten (float32,
//                             normalised) and its context overwritten with P V
// The update also touches the changed rows, whose contexts the second kernel
// then replaces; it reads their P rows before the second kernel rewrites them.
//
// Layouts: q, k, v, v_prev, c [B, L, H, hd] storage type; p [B, H, L, L]
// float32; the changed rows of sequence b are idx[b*L .. b*L + count[b] - 1],
// strictly ascending positions in [0, L) (the output of compact_below_kernel).
// A count outside [0, L] or a position that breaks that order sets the check
// flag and is skipped; no access leaves the buffers.
#pragma once

#include "common.cuh"

namespace esd {

constexpr int kApxRows = 16;     // context rows (queries) per CTA
constexpr int kApxChunk = 32;    // changed rows / keys staged per shared-memory chunk
constexpr int kApxThreads = 128;
constexpr int kApxMaxHd = 128;
constexpr int kApxRowsPerWarp = kApxRows / (kApxThreads / 32);

__device__ __forceinline__ int apx_count(const int32_t* __restrict__ count, int b, int L, int* flag) {
  const int n = count[b];
  if (n < 0 || n > L) {
    raise_flag(flag, kFlagCheck);
    return 0;
  }
  return n;
}

// position of entry a (< count) of a sequence's changed list, or -1 with the
// check flag raised when it is outside [0, L) or not above its predecessor
__device__ __forceinline__ int apx_changed_pos(const int32_t* __restrict__ idx, int a, int L, int* flag) {
  const int j = idx[a];
  if (j < 0 || j >= L || (a > 0 && idx[a - 1] >= j)) {
    raise_flag(flag, kFlagCheck);
    return -1;
  }
  return j;
}

__device__ __forceinline__ size_t apx_off(int b, int j, int h, int d, int L, int H, int hd) {
  return (((size_t)b * L + j) * H + h) * hd + d;
}

// Grid (ceil(L / kApxRows), H, B). Thread (g, dd) = (tid / hd, tid % hd) owns
// output column dd of rows g, g + G, ... (G = kApxThreads / hd groups).
template <typename T>
__global__ void __launch_bounds__(kApxThreads)
    approx_update_kernel(const T* __restrict__ v, const T* __restrict__ v_prev, const float* __restrict__ p,
                         const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int L, int H, int hd,
                         T* __restrict__ c, int* flag) {
  using S = Storage<T>;
  __shared__ int pos[kApxChunk];
  __shared__ float dv[kApxChunk][kApxMaxHd + 1];
  __shared__ float pp[kApxRows][kApxChunk + 1];
  const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * kApxRows;
  const int n = apx_count(count, b, L, flag);
  if (n == 0) return;
  const int32_t* ib = idx + (size_t)b * L;
  const int G = kApxThreads / hd;
  const int g = threadIdx.x / hd, dd = threadIdx.x - g * hd;
  const bool active = g < G;
  const size_t prow = ((size_t)b * H + h) * L;  // row index of P[b, h, 0, :]
  float acc[kApxRows];
#pragma unroll
  for (int u = 0; u < kApxRows; ++u) acc[u] = 0.f;

  for (int a0 = 0; a0 < n; a0 += kApxChunk) {
    const int na = min(kApxChunk, n - a0);
    if (threadIdx.x < kApxChunk)
      pos[threadIdx.x] = (int)threadIdx.x < na ? apx_changed_pos(ib, a0 + threadIdx.x, L, flag) : -1;
    __syncthreads();
    for (int e = threadIdx.x; e < kApxChunk * hd; e += kApxThreads) {
      const int a = e / hd, d = e - a * hd, j = pos[a];
      float x = 0.f;
      if (j >= 0) {
        const size_t o = apx_off(b, j, h, d, L, H, hd);
        x = S::to_f(v[o]) - S::to_f(v_prev[o]);
      }
      dv[a][d] = x;
    }
    for (int e = threadIdx.x; e < kApxRows * kApxChunk; e += kApxThreads) {
      const int r = e / kApxChunk, a = e - r * kApxChunk;
      const int i = i0 + r, j = pos[a];
      pp[r][a] = (i < L && j >= 0) ? p[(prow + i) * L + j] : 0.f;
    }
    __syncthreads();
    if (active) {
      for (int a = 0; a < na; ++a) {
        const float x = dv[a][dd];
#pragma unroll
        for (int u = 0; u < kApxRows; ++u) {
          const int r = g + G * u;
          if (r < kApxRows) acc[u] = fmaf(pp[r][a], x, acc[u]);
        }
      }
    }
    __syncthreads();
  }
  if (!active) return;
#pragma unroll
  for (int u = 0; u < kApxRows; ++u) {
    const int r = g + G * u, i = i0 + r;
    if (r < kApxRows && i < L) {
      const size_t o = apx_off(b, i, h, dd, L, H, hd);
      c[o] = S::from_f(S::to_f(c[o]) + acc[u]);
    }
  }
}

// Grid (ceil(L / kApxRows), H, B); CTA x takes entries [16x, 16x + 16) of the
// changed list (CTAs past the count return). Pass 1 writes the raw scores of
// its rows into their P rows and keeps each row's running maximum and sum of
// exponentials (warp w owns rows w, w + 4, w + 8, w + 12; lane = key within
// the chunk); pass 2 turns the scores into probabilities in place (each
// thread re-reads what it wrote) and accumulates P V from staged V chunks.
template <typename T>
__global__ void __launch_bounds__(kApxThreads)
    approx_exact_rows_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                             const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int L, int H,
                             int hd, float scale, T* __restrict__ c, float* __restrict__ p, int* flag) {
  using S = Storage<T>;
  __shared__ int pos[kApxRows];
  __shared__ float qs[kApxRows][kApxMaxHd];
  __shared__ float ks[kApxChunk][kApxMaxHd + 1];
  __shared__ float ps[kApxRows][kApxChunk + 1];
  const int b = blockIdx.z, h = blockIdx.y, a0 = blockIdx.x * kApxRows;
  const int n = apx_count(count, b, L, flag);
  if (a0 >= n) return;
  const int32_t* ib = idx + (size_t)b * L;
  if (threadIdx.x < kApxRows) {
    const int a = a0 + threadIdx.x;
    pos[threadIdx.x] = a < n ? apx_changed_pos(ib, a, L, flag) : -1;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kApxRows * hd; e += kApxThreads) {
    const int r = e / hd, d = e - r * hd, j = pos[r];
    qs[r][d] = j >= 0 ? S::to_f(q[apx_off(b, j, h, d, L, H, hd)]) * scale : 0.f;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t prow = ((size_t)b * H + h) * L;
  float m[kApxRowsPerWarp], s[kApxRowsPerWarp];
#pragma unroll
  for (int u = 0; u < kApxRowsPerWarp; ++u) {
    m[u] = -INFINITY;
    s[u] = 0.f;
  }

  // pass 1: scores
  for (int j0 = 0; j0 < L; j0 += kApxChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kApxChunk * hd; e += kApxThreads) {
      const int jj = e / hd, d = e - jj * hd, j = j0 + jj;
      ks[jj][d] = j < L ? S::to_f(k[apx_off(b, j, h, d, L, H, hd)]) : 0.f;
    }
    __syncthreads();
    const int j = j0 + lane;
#pragma unroll
    for (int u = 0; u < kApxRowsPerWarp; ++u) {
      const int r = warp + 4 * u;
      float sc = 0.f;
      for (int d = 0; d < hd; ++d) sc = fmaf(qs[r][d], ks[lane][d], sc);
      const float x = j < L ? sc : -INFINITY;
      const float nm = fmaxf(m[u], warp_max(x));
      const float es = warp_sum(j < L ? expf(x - nm) : 0.f);
      s[u] = s[u] * expf(m[u] - nm) + es;
      m[u] = nm;
      if (j < L && pos[r] >= 0) p[(prow + pos[r]) * L + j] = sc;
    }
  }

  // pass 2: probabilities and P V
  const int G = kApxThreads / hd;
  const int g = threadIdx.x / hd, dd = threadIdx.x - g * hd;
  const bool active = g < G;
  float acc[kApxRows];
#pragma unroll
  for (int u = 0; u < kApxRows; ++u) acc[u] = 0.f;
  for (int j0 = 0; j0 < L; j0 += kApxChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kApxChunk * hd; e += kApxThreads) {
      const int jj = e / hd, d = e - jj * hd, j = j0 + jj;
      ks[jj][d] = j < L ? S::to_f(v[apx_off(b, j, h, d, L, H, hd)]) : 0.f;
    }
    const int j = j0 + lane;
#pragma unroll
    for (int u = 0; u < kApxRowsPerWarp; ++u) {
      const int r = warp + 4 * u;
      float pr = 0.f;
      if (j < L && pos[r] >= 0) {
        const size_t o = (prow + pos[r]) * L + j;
        pr = expf(p[o] - m[u]) / s[u];
        p[o] = pr;
      }
      ps[r][lane] = pr;
    }
    __syncthreads();
    if (active) {
      const int nj = min(kApxChunk, L - j0);
      for (int jj = 0; jj < nj; ++jj) {
        const float x = ks[jj][dd];
#pragma unroll
        for (int u = 0; u < kApxRows; ++u) {
          const int r = g + G * u;
          if (r < kApxRows) acc[u] = fmaf(ps[r][jj], x, acc[u]);
        }
      }
    }
  }
  if (!active) return;
#pragma unroll
  for (int u = 0; u < kApxRows; ++u) {
    const int r = g + G * u;
    if (r < kApxRows && pos[r] >= 0) c[apx_off(b, pos[r], h, dd, L, H, hd)] = S::from_f(acc[u]);
  }
}

}  // namespace esd
