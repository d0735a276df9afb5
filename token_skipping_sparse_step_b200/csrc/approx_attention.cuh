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
// Both are SIMT float32: 16 rows of one head per CTA, operands staged in
// shared memory in 32-row chunks and read as float4, several independent
// accumulators per thread.
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
constexpr int kApxKs = kApxMaxHd + 4;  // staged K / V / dV row stride (floats): float4 reads conflict-free
constexpr int kApxPt = kApxRows + 4;   // transposed probability tile stride: float4-aligned rows
constexpr int kApxPre = kApxChunk * kApxMaxHd / kApxThreads;  // staged elements per thread

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

// Output mapping shared by both kernels: thread (g, dd) = (tid / hd, tid % hd)
// owns column dd of the rp consecutive rows [g * rp, (g + 1) * rp), with
// 1 <= groups = min(pow2 floor of kApxThreads / hd, kApxRows) and
// rp = kApxRows / groups; threads with g >= groups only stage data.
struct ApxOut {
  int g, dd, rp;
  bool active;
  __device__ __forceinline__ ApxOut(int hd) {
    int groups = 1;
    while (groups * 2 * hd <= kApxThreads && groups * 2 <= kApxRows) groups *= 2;
    g = threadIdx.x / hd;
    dd = threadIdx.x - g * hd;
    rp = kApxRows / groups;
    active = g < groups;
  }
};

// acc[u] += pt[g*rp + u] * x for u < rp (pt: one float4-aligned row of a
// transposed probability tile; float4 reads when rp >= 4)
__device__ __forceinline__ void apx_accumulate(float (&acc)[kApxRows], const float* pt, int rp, float x) {
#pragma unroll
  for (int u = 0; u < kApxRows; u += 4) {
    if (u < rp) {
      float4 pv;
      if (rp >= 4) {
        pv = *reinterpret_cast<const float4*>(pt + u);
      } else {
        pv.x = pt[u];
        pv.y = u + 1 < rp ? pt[u + 1] : 0.f;
        pv.z = 0.f;
        pv.w = 0.f;
      }
      acc[u] = fmaf(pv.x, x, acc[u]);
      acc[u + 1] = fmaf(pv.y, x, acc[u + 1]);
      acc[u + 2] = fmaf(pv.z, x, acc[u + 2]);
      acc[u + 3] = fmaf(pv.w, x, acc[u + 3]);
    }
  }
}

// Grid (ceil(L / kApxRows), H, B): rows [16x, 16x + 16) of head y, sequence z.
template <typename T>
__global__ void __launch_bounds__(kApxThreads)
    approx_update_kernel(const T* __restrict__ v, const T* __restrict__ v_prev, const float* __restrict__ p,
                         const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int L, int H, int hd,
                         T* __restrict__ c, int* flag) {
  using S = Storage<T>;
  __shared__ int pos[kApxChunk];
  __shared__ __align__(16) float dv[kApxChunk][kApxKs];
  __shared__ __align__(16) float pt[kApxChunk][kApxPt];  // pt[a][r] = P[i0 + r, pos[a]]
  const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * kApxRows;
  const int n = apx_count(count, b, L, flag);
  if (n == 0) return;
  const int32_t* ib = idx + (size_t)b * L;
  const ApxOut om(hd);
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
      pt[a][r] = (i < L && j >= 0) ? p[(prow + i) * L + j] : 0.f;
    }
    __syncthreads();
    if (om.active)
      for (int a = 0; a < na; ++a) apx_accumulate(acc, &pt[a][om.g * om.rp], om.rp, dv[a][om.dd]);
    __syncthreads();
  }
  if (!om.active) return;
#pragma unroll
  for (int u = 0; u < kApxRows; ++u) {
    const int i = i0 + om.g * om.rp + u;
    if (u < om.rp && i < L) {
      const size_t o = apx_off(b, i, h, om.dd, L, H, hd);
      c[o] = S::from_f(S::to_f(c[o]) + acc[u]);
    }
  }
}

// Register staging of a chunk of 32 key rows of one head: thread (g, d) =
// (tid / hd4, tid % hd4) holds column d of keys g, g + kp, g + 2 kp, ...
// (kp = kApxThreads / hd4 >= 1 keys side by side); columns past hd and keys
// past L are zero, so that every cell [0, 32) x [0, hd4) of the tile is written.
struct ApxStage {
  int kp, g, d, hd4;
  bool on;
  size_t stride;  // elements between the keys one thread holds
  __device__ __forceinline__ ApxStage(int hd, int H) {
    hd4 = (hd + 3) & ~3;
    kp = kApxThreads / hd4;
    g = threadIdx.x / hd4;
    d = threadIdx.x - g * hd4;
    on = g < kp;
    stride = (size_t)kp * H * hd;
  }
};

template <typename T>
__device__ __forceinline__ void apx_load_chunk(float (&pre)[kApxPre], const ApxStage sg, const T* __restrict__ src,
                                               int b, int j0, int h, int L, int H, int hd) {
  const bool col = sg.on && sg.d < hd;
  const T* base = src + apx_off(b, 0, h, col ? sg.d : 0, L, H, hd) + (size_t)(j0 + sg.g) * H * hd;
#pragma unroll
  for (int u = 0; u < kApxPre; ++u) {
    const int jj = sg.g + sg.kp * u;
    pre[u] = (col && jj < kApxChunk && j0 + jj < L) ? Storage<T>::to_f(base[sg.stride * u]) : 0.f;
  }
}

__device__ __forceinline__ void apx_store_chunk(float (*ks)[kApxKs], const float (&pre)[kApxPre],
                                                const ApxStage sg) {
  if (!sg.on) return;
#pragma unroll
  for (int u = 0; u < kApxPre; ++u) {
    const int jj = sg.g + sg.kp * u;
    if (jj < kApxChunk) ks[jj][sg.d] = pre[u];
  }
}

// Grid (ceil(L / kApxRows), H, B); CTA x takes entries [16x, 16x + 16) of the
// changed list (CTAs past the count return). Pass 1 writes the raw scores of
// its rows into their P rows and keeps each row's running maximum and sum of
// exponentials (warp w owns rows w, w + 4, w + 8, w + 12; lane = key within
// the chunk); pass 2 turns the scores into probabilities in place (each
// thread re-reads what it wrote) and accumulates P V from staged V chunks.
// Each pass stages the next chunk in registers while the current one is used.
template <typename T>
__global__ void __launch_bounds__(kApxThreads)
    approx_exact_rows_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                             const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int L, int H,
                             int hd, float scale, T* __restrict__ c, float* __restrict__ p, int* flag) {
  using S = Storage<T>;
  __shared__ int pos[kApxRows];
  __shared__ __align__(16) float qs[kApxRows][kApxMaxHd];
  __shared__ __align__(16) float ks[kApxChunk][kApxKs];
  __shared__ __align__(16) float pt[kApxChunk][kApxPt];  // pt[jj][r] = P[pos[r], j0 + jj]
  const int b = blockIdx.z, h = blockIdx.y, a0 = blockIdx.x * kApxRows;
  const int n = apx_count(count, b, L, flag);
  if (a0 >= n) return;
  const int32_t* ib = idx + (size_t)b * L;
  const ApxStage sg(hd, H);
  const int hd4 = sg.hd4;
  float pre[kApxPre];
  apx_load_chunk<T>(pre, sg, k, b, 0, h, L, H, hd);
  if (threadIdx.x < kApxRows) {
    const int a = a0 + threadIdx.x;
    pos[threadIdx.x] = a < n ? apx_changed_pos(ib, a, L, flag) : -1;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kApxRows * hd4; e += kApxThreads) {
    const int r = e / hd4, d = e - r * hd4, j = pos[r];
    qs[r][d] = (j >= 0 && d < hd) ? S::to_f(q[apx_off(b, j, h, d, L, H, hd)]) * scale : 0.f;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t prow = ((size_t)b * H + h) * L;
  int prw[kApxRowsPerWarp];  // positions of this warp's rows
  float m[kApxRowsPerWarp], s[kApxRowsPerWarp];
#pragma unroll
  for (int u = 0; u < kApxRowsPerWarp; ++u) {
    prw[u] = pos[warp + 4 * u];
    m[u] = -INFINITY;
    s[u] = 0.f;
  }

  // pass 1: scores
  for (int j0 = 0; j0 < L; j0 += kApxChunk) {
    __syncthreads();
    apx_store_chunk(ks, pre, sg);
    __syncthreads();
    if (j0 + kApxChunk < L) apx_load_chunk<T>(pre, sg, k, b, j0 + kApxChunk, h, L, H, hd);
    float sc[kApxRowsPerWarp];
#pragma unroll
    for (int u = 0; u < kApxRowsPerWarp; ++u) sc[u] = 0.f;
    for (int d = 0; d < hd4; d += 4) {
      const float4 kv = *reinterpret_cast<const float4*>(&ks[lane][d]);
#pragma unroll
      for (int u = 0; u < kApxRowsPerWarp; ++u) {
        const float4 qv = *reinterpret_cast<const float4*>(&qs[warp + 4 * u][d]);
        sc[u] = fmaf(qv.x, kv.x, sc[u]);
        sc[u] = fmaf(qv.y, kv.y, sc[u]);
        sc[u] = fmaf(qv.z, kv.z, sc[u]);
        sc[u] = fmaf(qv.w, kv.w, sc[u]);
      }
    }
    const int j = j0 + lane;
#pragma unroll
    for (int u = 0; u < kApxRowsPerWarp; ++u) {
      const float x = j < L ? sc[u] : -INFINITY;
      const float nm = fmaxf(m[u], warp_max(x));
      const float es = warp_sum(j < L ? expf(x - nm) : 0.f);
      s[u] = s[u] * expf(m[u] - nm) + es;
      m[u] = nm;
      if (j < L && prw[u] >= 0) p[(prow + prw[u]) * L + j] = sc[u];
    }
  }

  // pass 2: probabilities and P V
  const ApxOut om(hd);
  float acc[kApxRows];
#pragma unroll
  for (int u = 0; u < kApxRows; ++u) acc[u] = 0.f;
  apx_load_chunk<T>(pre, sg, v, b, 0, h, L, H, hd);
  for (int j0 = 0; j0 < L; j0 += kApxChunk) {
    __syncthreads();
    apx_store_chunk(ks, pre, sg);
    const int j = j0 + lane;
#pragma unroll
    for (int u = 0; u < kApxRowsPerWarp; ++u) {
      float pr = 0.f;
      if (j < L && prw[u] >= 0) {
        const size_t o = (prow + prw[u]) * L + j;
        pr = expf(p[o] - m[u]) / s[u];
        p[o] = pr;
      }
      pt[lane][warp + 4 * u] = pr;
    }
    __syncthreads();
    if (j0 + kApxChunk < L) apx_load_chunk<T>(pre, sg, v, b, j0 + kApxChunk, h, L, H, hd);
    if (om.active) {
      const int nj = min(kApxChunk, L - j0);
      for (int jj = 0; jj < nj; ++jj) apx_accumulate(acc, &pt[jj][om.g * om.rp], om.rp, ks[jj][om.dd]);
    }
  }
  if (!om.active) return;
#pragma unroll
  for (int u = 0; u < kApxRows; ++u) {
    if (u < om.rp) {
      const int j = pos[om.g * om.rp + u];
      if (j >= 0) c[apx_off(b, j, h, om.dd, L, H, hd)] = S::from_f(acc[u]);
    }
  }
}

}  // namespace esd
