// Saliency-aware approximate attention of one layer ("DyLLM: Efficient
// Diffusion LLM Inference via Saliency-based Token Selection and Partial
// Attention", technical summary section 2.B.2): the rows whose values moved
// since the previous step (the salient ones) get exact attention rows, and
// every other row moves its cached context by the change of those values
// weighted by its cached attention probabilities, C_i += sum_a P_{i,j_a} dV_{j_a}
// (per head), at O(L x |changed|) instead of O(L^2).
//
// float32 models: two SIMT kernels on one stream, in this order:
//   approx_update_kernel      every row i: C_i += sum over the changed rows of
//                             P[i, j_a] (V - V_prev)[j_a]  (reads the cached P)
//   approx_exact_rows_kernel  every changed row: exact softmax(q k^T / sqrt(hd))
//                             over all L keys, its P row rewritten (float32,
//                             normalised) and its context overwritten with P V
// The update also touches the changed rows, whose contexts the second kernel
// then replaces; it reads their P rows before the second kernel rewrites them.
// 16 rows of one head per CTA, operands staged in shared memory in 32-row
// chunks and read as float4, several independent accumulators per thread.
// bf16 models: the tensor-core kernels at the end of this file, same order.
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

// ------------------------------------------------------------------ bf16
// The bf16 models run the same arithmetic on tensor cores:
//   approx_update_mma_kernel  every row i: C_out_i = C_in_i + sum_a P[i, j_a]
//                             (V - V_prev)[j_a], per head, as a tensor-core
//                             product (mma.sync m16n8k16, bf16 operands, fp32
//                             sums): the moved rows' columns of the cached
//                             probabilities (rounded to bf16) times the staged
//                             change of their values (rounded to bf16);
//   the moved rows' exact attention on the SM-pair attention kernel (which
//   also reports each moved row's maximum and sum of its scores), then
//   prob_rows_mma_kernel  each moved row's P row = 2^(score - max) / sum,
//                         the scores recomputed on tensor cores.
// Moved lists in slot form: slot a < count[b] of sequence b holds position
// idx[b*L + a]; slot_rows_kernel gathers rows by slot or scatters them back.

constexpr int kAuRows = 64;   // context rows per CTA (4 warps x 16)
constexpr int kAuKeys = 32;   // moved rows per staged chunk

__device__ __forceinline__ uint32_t au_swz(int row, int chunk) {  // byte offset in a [rows][256 B] tile
  return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}
__device__ __forceinline__ void au_ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                             uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void au_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9},"
      " {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t au_pack(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Grid (ceil(L / 64), H, B), 128 threads; warp w owns rows [16 w, 16 w + 16)
// of the CTA's 64. v, v_prev, c_in, c_out: [B*L, d] as [B, L, H, 128]; v_prev
// row b*L + a (vprev_slots) or b*L + idx_a. p: [B, H, L, L] float32. The
// moved positions are staged in shared memory in blocks of kAuPos; within a
// block, the next chunk's loads (its rows of V and V_prev, and this thread's
// P values) are in flight while the current chunk's products run.
constexpr int kAuPos = 1024;

struct AuLoads {
  uint4 nv[4], ov[4];  // this thread's 32 dims of V and V_prev of one moved row
  float pf[16];        // P values of the A fragments of the chunk's two k-steps
};

__device__ __forceinline__ void au_issue(AuLoads& ld, const float* pa, const float* pb, bool va, bool vb,
                                         const int* pos, int base, int na, const __nv_bfloat16* v,
                                         const __nv_bfloat16* v_prev, bool vprev_slots, int slot0, size_t vrow0,
                                         int tid, int t4, size_t d, int h) {
  // V rows: moved row kk = tid / 4 of the chunk, dims [32 (tid % 4), +32)
  const int kk = tid >> 2, c0 = (tid & 3) * 32;
  const int j = kk < na ? pos[base + kk] : -1;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    ld.nv[q] = make_uint4(0u, 0u, 0u, 0u);
    ld.ov[q] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (j >= 0) {
    const __nv_bfloat16* vr = v + (vrow0 + j) * d + h * 128 + c0;
    const __nv_bfloat16* pr = v_prev + (vrow0 + (vprev_slots ? slot0 + base + kk : j)) * d + h * 128 + c0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      ld.nv[q] = *reinterpret_cast<const uint4*>(vr + 8 * q);
      ld.ov[q] = *reinterpret_cast<const uint4*>(pr + 8 * q);
    }
  }
  // P: columns ks*16 + 2 t4 (+1, +8, +9) of rows ra (pa) and rb (pb)
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int kc = ks * 16 + 2 * t4 + (e & 1) + ((e >> 1) << 3);
      const int jj = kc < na ? pos[base + kc] : -1;
      ld.pf[ks * 8 + e] = (va && jj >= 0) ? __ldg(pa + jj) : 0.0f;
      ld.pf[ks * 8 + 4 + e] = (vb && jj >= 0) ? __ldg(pb + jj) : 0.0f;
    }
  }
}

__global__ void __launch_bounds__(128)
approx_update_mma_kernel(const float* __restrict__ p, const __nv_bfloat16* __restrict__ v,
                         const __nv_bfloat16* __restrict__ v_prev, int vprev_slots, const int32_t* __restrict__ idx,
                         const int32_t* __restrict__ count, int L, int H, const __nv_bfloat16* c_in,
                         __nv_bfloat16* c_out, int* flag) {
  __shared__ int pos[kAuPos];
  __shared__ __align__(128) uint8_t sdv[2][kAuKeys * 256];  // change of V [32 moved rows][128 dims] bf16, swizzled
  grid_launch_dependents();
  grid_dependency_wait();  // (no-ops unless launched with dependent launch)
  const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * kAuRows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const size_t d = (size_t)H * 128;
  const int n = apx_count(count, b, L, flag);
  const int32_t* ib = idx + (size_t)b * L;
  const int ra = i0 + warp * 16 + g, rb = ra + 8;  // this thread's two rows of every fragment
  const bool va = ra < L, vb = rb < L;
  const float* pa = p + (((size_t)b * H + h) * L + (va ? ra : 0)) * (size_t)L;
  const float* pb = p + (((size_t)b * H + h) * L + (vb ? rb : 0)) * (size_t)L;
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  const uint32_t sbase = smem_u32(sdv);

  for (int s0 = 0; s0 < n; s0 += kAuPos) {
    const int ns = min(kAuPos, n - s0);
    __syncthreads();  // the previous block's positions are no longer read
    for (int a = tid; a < ns; a += 128) pos[a] = apx_changed_pos(ib, s0 + a, L, flag);
    __syncthreads();
    const int nch = (ns + kAuKeys - 1) / kAuKeys;
    AuLoads cur;
    au_issue(cur, pa, pb, va, vb, pos, 0, min(kAuKeys, ns), v, v_prev, vprev_slots != 0, s0, (size_t)b * L, tid, t4,
             d, h);
    for (int c = 0; c < nch; ++c) {
      const int buf = c & 1;
      // the chunk's change of V into its staged tile, its P values into A fragments
      {
        const int kk = tid >> 2, c0 = (tid & 3) * 32;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162* n2 = reinterpret_cast<const __nv_bfloat162*>(&cur.nv[q]);
          const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&cur.ov[q]);
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fn = __bfloat1622float2(n2[e]), fo = __bfloat1622float2(o2[e]);
            w[e] = au_pack(fn.x - fo.x, fn.y - fo.y);
          }
          *reinterpret_cast<uint4*>(sdv[buf] + au_swz(kk, (c0 >> 3) + q)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      uint32_t af[2][4];
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const float* f = cur.pf + ks * 8;
        af[ks][0] = au_pack(f[0], f[1]);  // row ra, columns 2 t4, +1
        af[ks][1] = au_pack(f[4], f[5]);  // row rb
        af[ks][2] = au_pack(f[2], f[3]);  // row ra, columns 2 t4 + 8, +9
        af[ks][3] = au_pack(f[6], f[7]);  // row rb
      }
      __syncthreads();
      if (c + 1 < nch) {
        const int base = (c + 1) * kAuKeys;
        au_issue(cur, pa, pb, va, vb, pos, base, min(kAuKeys, ns - base), v, v_prev, vprev_slots != 0, s0,
                 (size_t)b * L, tid, t4, d, h);
      }
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
        for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-dim tiles
          const int key = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int chunk = dp * 2 + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          au_ldsm_x4_t(sbase + (uint32_t)(buf * kAuKeys * 256) + au_swz(key, chunk), b0, b1, b2, b3);
          au_mma(o[2 * dp], af[ks][0], af[ks][1], af[ks][2], af[ks][3], b0, b1);
          au_mma(o[2 * dp + 1], af[ks][0], af[ks][1], af[ks][2], af[ks][3], b2, b3);
        }
      }
    }
  }
  // C_out = C_in + the sums, rows ra and rb, dims 8 dn + 2 t4 (+1)
#pragma unroll
  for (int dn = 0; dn < 16; ++dn) {
    const int col = dn * 8 + 2 * t4;
    if (va) {
      const size_t e = ((size_t)b * L + ra) * d + h * 128 + col;
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(c_in + e));
      *reinterpret_cast<__nv_bfloat162*>(c_out + e) = __floats2bfloat162_rn(c.x + o[dn][0], c.y + o[dn][1]);
    }
    if (vb) {
      const size_t e = ((size_t)b * L + rb) * d + h * 128 + col;
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(c_in + e));
      *reinterpret_cast<__nv_bfloat162*>(c_out + e) = __floats2bfloat162_rn(c.x + o[dn][2], c.y + o[dn][3]);
    }
  }
}

// The moved rows' probability rows: P[b, h, idx_a, key] = 2^(s - m) / l with
// s = q_a k_key / sqrt(128) log2 e and (m, l) = stat[(b*L + a) H + h], the
// row maximum and sum the attention kernel reported for the same scores.
// Grid (ceil(R / 64), H, B * ks), 128 threads (4 warps x 16 rows); split
// z % ks takes an equal share of the 64-key tiles; q: the moved rows'
// queries in slot form, R rows per sequence; k: [B*L, d]. Q fragments
// stay in registers; K tiles of 64 keys stream through a double-buffered
// shared tile (cp.async); S with mma.sync m16n8k16 (bf16 in, fp32 sums); each
// store instruction writes 8 rows x 32 contiguous bytes.
constexpr int kPrRows = 64;
constexpr int kPrKeys = 64;

__device__ __forceinline__ void au_ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void au_cp16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
// [64 rows][128 bf16] tile (row stride ld elements) into swizzled shared memory; rows >= valid zero
__device__ __forceinline__ void au_load_tile(uint32_t sbase, const __nv_bfloat16* g, size_t ld, int valid, int tid) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = tid + i * 128;  // 1024 chunks of 16 B
    const int row = c >> 4, chunk = c & 15;
    const bool ok = row < valid;
    au_cp16(sbase + au_swz(row, chunk), ok ? g + (size_t)row * ld + chunk * 8 : g, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(128)
prob_rows_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                     const float2* __restrict__ stat, float* __restrict__ p, int R, int L, int H, float scale_log2,
                     int ks, int* flag) {
  __shared__ __align__(128) uint8_t sq[kPrRows * 256];
  __shared__ __align__(128) uint8_t sk[2][kPrKeys * 256];
  grid_launch_dependents();
  grid_dependency_wait();  // (no-ops unless launched with dependent launch)
  const int b = blockIdx.z / ks, split = blockIdx.z % ks, h = blockIdx.y, a0 = blockIdx.x * kPrRows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int n = min(apx_count(count, b, L, flag), R);
  if (a0 >= n) return;
  const size_t ld = (size_t)H * 128;
  const uint32_t sqb = smem_u32(sq), skb = smem_u32(sk);
  const int ntiles = (L + kPrKeys - 1) / kPrKeys, tps = (ntiles + ks - 1) / ks;
  const int t0 = split * tps, t1 = min(ntiles, t0 + tps);
  if (t0 >= t1) return;  // (before any copy into shared memory is issued)
  au_load_tile(sqb, q + ((size_t)b * R + a0) * ld + h * 128, ld, n - a0, tid);
  const __nv_bfloat16* kg = k + (size_t)b * L * ld + h * 128;
  au_load_tile(skb, kg + (size_t)t0 * kPrKeys * ld, ld, L - t0 * kPrKeys, tid);
  // this thread's two rows: slot a, P row pointer and statistics
  float* prow[2] = {nullptr, nullptr};
  float mrow[2] = {0.0f, 0.0f}, irow[2] = {0.0f, 0.0f};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int a = a0 + warp * 16 + g + 8 * u;
    if (a < n) {
      const int j = apx_changed_pos(idx + (size_t)b * L, a, L, flag);
      if (j >= 0) {
        const float2 st = stat[((size_t)b * L + a) * H + h];
        prow[u] = p + (((size_t)b * H + h) * L + j) * (size_t)L;
        mrow[u] = st.x;
        irow[u] = 1.0f / st.y;
      }
    }
  }
  uint32_t qa[8][4];
  for (int t = t0; t < t1; ++t) {
    const int buf = (t - t0) & 1;
    if (t + 1 < t1) {
      au_load_tile(skb + (uint32_t)((buf ^ 1) * kPrKeys * 256), kg + (size_t)(t + 1) * kPrKeys * ld, ld,
                   L - (t + 1) * kPrKeys, tid);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    if (t == t0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int row = warp * 16 + (lane & 15);
        const int chunk = kk * 2 + (lane >> 4);
        au_ldsm_x4(sqb + au_swz(row, chunk), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }
    float sv[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[i][0] = sv[i][1] = sv[i][2] = sv[i][3] = 0.0f;
    const uint32_t kt = skb + (uint32_t)(buf * kPrKeys * 256);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // pairs of 8-key tiles
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int chunk = kk * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        au_ldsm_x4(kt + au_swz(key, chunk), b0, b1, b2, b3);
        au_mma(sv[2 * np], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
        au_mma(sv[2 * np + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!prow[u]) continue;
#pragma unroll
      for (int nn = 0; nn < 8; ++nn) {
        const int key = t * kPrKeys + nn * 8 + 2 * t4;
        const float e0 = exp2f(fmaf(sv[nn][2 * u], scale_log2, -mrow[u])) * irow[u];
        const float e1 = exp2f(fmaf(sv[nn][2 * u + 1], scale_log2, -mrow[u])) * irow[u];
        if (key + 1 < L && (L & 1) == 0) {
          __stcs(reinterpret_cast<float2*>(prow[u] + key), make_float2(e0, e1));
        } else {
          if (key < L) __stcs(prow[u] + key, e0);
          if (key + 1 < L) __stcs(prow[u] + key + 1, e1);
        }
      }
    }
    __syncthreads();  // the K buffer is refilled two tiles later
  }
}

// Rows of d bf16 (d a multiple of 8) between slot and position form: gather
// dst[b*sld + a] = src[b*L + idx_a], scatter dst[b*L + idx_a] = src[b*sld + a],
// for every slot a < min(count[b], sld). Grid (sld, B), 128 threads.
template <bool kScatter>
__global__ void __launch_bounds__(128)
slot_rows_kernel(__nv_bfloat16* __restrict__ dst, const __nv_bfloat16* __restrict__ src,
                 const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int L, int sld, int d,
                 int* flag) {
  grid_launch_dependents();
  grid_dependency_wait();  // (no-ops unless launched with dependent launch)
  const int b = blockIdx.y, a = blockIdx.x;
  const int n = apx_count(count, b, L, flag);
  if (a >= n) return;
  const int j = apx_changed_pos(idx + (size_t)b * L, a, L, flag);
  if (j < 0) return;
  const size_t sr = kScatter ? (size_t)b * sld + a : (size_t)b * L + j;
  const size_t dr = kScatter ? (size_t)b * L + j : (size_t)b * sld + a;
  const uint4* s4 = reinterpret_cast<const uint4*>(src + sr * d);
  uint4* d4 = reinterpret_cast<uint4*>(dst + dr * d);
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) d4[i] = s4[i];
}

}  // namespace esd
