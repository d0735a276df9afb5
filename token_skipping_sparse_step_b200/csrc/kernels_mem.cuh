// Memory-bound kernels of the step: embedding gather, RMS statistic, importance
// score, per-sequence top-k, row gather with H-cache scatter, remasking and the
// final reduction of the max-softmax head.
#pragma once

#include "common.cuh"

namespace esd {

// ---------------------------------------------------------------------------
// x[r, :] = E[tok[r], :]   (one warp per row, 16-byte accesses)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tok, const T* __restrict__ emb,
                             T* __restrict__ x, int rows, int d, int vocab, int* flag) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  int t = tok[warp];
  T* dst = x + (size_t)warp * d;
  if (t < 0 || t >= vocab) {
    if (lane == 0) raise_flag(flag, kFlagCheck);
    for (int c = lane * 8; c < d; c += 256) {
      float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      Storage<T>::store8(dst + c, z);
    }
    return;
  }
  const T* src = emb + (size_t)t * d;
  for (int c = lane * 8; c < d; c += 256) copy8(dst + c, src + c);
}

// ---------------------------------------------------------------------------
// inv_rms[r] = 1 / sqrt(mean(x[r]^2) + eps)   (one warp per row)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rms_kernel(const T* __restrict__ x, float* __restrict__ inv_rms, int rows, int d,
                           float eps) {
  grid_launch_dependents();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const T* p = x + (size_t)warp * d;
  float acc = 0.0f;
  for (int c = lane * 8; c < d; c += 256) {
    float v[8];
    Storage<T>::load8(p + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = fmaf(v[i], v[i], acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) inv_rms[warp] = 1.0f / sqrtf(acc / (float)d + eps);
}

// ---------------------------------------------------------------------------
// Importance score per row (one warp per row; 16-byte streaming loads).
//  mode 0 (ES):  alpha*c + (1-alpha) * ||x-h||_1 / max(sqrt(d)*||h||_2, 1e-12)
//  mode 1 (COS): max(1 - x.h / sqrt(max(|x|^2 |h|^2, 1e-24)), 0) + lambda*(1-c)
// The COS sums use the same instruction sequence for x.h, x.x and h.h so that
// an unchanged row gives cos == 1 exactly.
// ---------------------------------------------------------------------------
template <typename T, int MODE>
__global__ void score_kernel(const T* __restrict__ x, const T* __restrict__ h,
                             const float* __restrict__ conf, float* __restrict__ score, int rows,
                             int d, float coef) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const T* px = x + (size_t)warp * d;
  const T* ph = h + (size_t)warp * d;
  float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f;
  for (int c = lane * 8; c < d; c += 256) {
    float vx[8], vh[8];
    load8_stream(px + c, vx);
    load8_stream(ph + c, vh);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (MODE == 0) {
        a0 += fabsf(vx[i] - vh[i]);
        a1 = fmaf(vh[i], vh[i], a1);
      } else {
        a0 = fmaf(vx[i], vh[i], a0);
        a1 = fmaf(vx[i], vx[i], a1);
        a2 = fmaf(vh[i], vh[i], a2);
      }
    }
  }
  a0 = warp_sum(a0);
  a1 = warp_sum(a1);
  if (MODE == 1) a2 = warp_sum(a2);
  if (lane == 0) {
    const float c = conf[warp];
    float s;
    if (MODE == 0) {
      const float den = fmaxf(sqrtf((float)d) * sqrtf(a1), 1e-12f);
      s = coef * c + (1.0f - coef) * (a0 / den);
    } else {
      const float cs = a0 / sqrtf(fmaxf(a1 * a2, 1e-24f));
      s = fmaxf(1.0f - cs, 0.0f) + coef * (1.0f - c);
    }
    score[warp] = s;
  }
}

// ---------------------------------------------------------------------------
// Per-sequence exact top-k (one CTA per sequence).
// Keys: score_key(score) (descending order of score; -0 == +0; NaN lowest).
// Pass 1: MSB-first radix select (4 x 8 bits) of the k-th largest key T.
// Pass 2: select key > T, plus the lowest-index (k - #greater) keys == T.
// Pass 3: write the selected indices in ascending order (block-wide scan).
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;

__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_sums[w] = inc;
  __syncthreads();
  if (w == 0) {
    int s = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += t;
    }
    if (lane < (int)(blockDim.x >> 5)) warp_sums[lane] = si - s;  // exclusive prefix of warps
    if (lane == 31) warp_sums[32] = si;
  }
  __syncthreads();
  int r = warp_sums[w] + inc - v;
  total = warp_sums[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ scores, int L, int k, int32_t* __restrict__ idx_out) {
  extern __shared__ uint32_t topk_keys[];  // [L]
  __shared__ int hist[256];
  __shared__ int warp_sums[33];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  const int b = blockIdx.x;
  const float* s = scores + (size_t)b * L;
  for (int i = threadIdx.x; i < L; i += blockDim.x) topk_keys[i] = score_key(s[i]);
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_need = k;
  }
  __syncthreads();
  // radix select of the k-th largest key
  uint32_t mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
      uint32_t key = topk_keys[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // the highest bin where the candidates counted from the top reach
      // `need`: lane l holds bins 255 - 8l .. 248 - 8l (descending), a warp
      // prefix over the lanes, the first lane that reaches it scans its 8
      const int lane = threadIdx.x;
      int c[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - (lane * 8 + j)];
        tot += c[j];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int need = s_need;
      const unsigned ball = __ballot_sync(0xffffffffu, incl >= need);
      if (lane == __ffs(ball) - 1) {
        int run = incl - tot, bin = 248 - lane * 8, nd = need - run;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + c[j] >= need) {
            bin = 255 - (lane * 8 + j);
            nd = need - run;
            break;
          }
          run += c[j];
        }
        s_prefix = prefix | ((uint32_t)bin << shift);
        s_need = nd;  // how many keys equal to the final threshold to take
      }
    }
    __syncthreads();
    mask |= 255u << shift;
  }
  const uint32_t T = s_prefix;
  const int take_eq = s_need;
  // contiguous chunk per thread so that the scans run in index order
  const int per = (L + blockDim.x - 1) / blockDim.x;
  const int i0 = threadIdx.x * per;
  const int i1 = min(L, i0 + per);
  int n_eq = 0;
  for (int i = i0; i < i1; ++i) n_eq += (topk_keys[i] == T);
  int tot;
  int eq_before = block_excl_scan(n_eq, warp_sums, tot);
  int n_sel = 0;
  {
    int e = eq_before;
    for (int i = i0; i < i1; ++i) {
      uint32_t key = topk_keys[i];
      if (key > T) ++n_sel;
      else if (key == T) { if (e < take_eq) ++n_sel; ++e; }
    }
  }
  int out_pos = block_excl_scan(n_sel, warp_sums, tot);
  int32_t* dst = idx_out + (size_t)b * k;
  int e = eq_before;
  for (int i = i0; i < i1; ++i) {
    uint32_t key = topk_keys[i];
    bool sel = false;
    if (key > T) sel = true;
    else if (key == T) { sel = (e < take_eq); ++e; }
    if (sel) dst[out_pos++] = i;
  }
}

// ---------------------------------------------------------------------------
// Context saliency ("DyLLM", technical summary sections 2.A and 2.B.1): one
// warp per row, s = cur.prev / sqrt(max(|cur|^2 |prev|^2, 1e-24)) with float32
// sums in the same instruction order for the three products (an unchanged row
// gives s == 1 exactly), then, one CTA per sequence, the rows with s < tau in
// ascending order (block-wide scan), -1 after the last, and their count.
// ---------------------------------------------------------------------------
// Rows whose values moved: flag[r] = 0 where row r of x differs bitwise from
// row r of prev in any element, else 1 (so compact_below_kernel with tau 0.5
// lists the moved rows). One warp per row, 16-byte loads.
template <typename T>
__global__ void row_changed_kernel(const T* __restrict__ x, const T* __restrict__ prev, int rows, int d,
                                   float* __restrict__ flag) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const uint4* a = reinterpret_cast<const uint4*>(x + (size_t)warp * d);
  const uint4* b = reinterpret_cast<const uint4*>(prev + (size_t)warp * d);
  const int n = (int)((size_t)d * sizeof(T) / 16);
  bool diff = false;
  for (int i = lane; i < n; i += 32) {
    const uint4 u = a[i], v = b[i];
    diff |= (u.x != v.x) | (u.y != v.y) | (u.z != v.z) | (u.w != v.w);
  }
  diff = __any_sync(0xffffffffu, diff);
  if (lane == 0) flag[warp] = diff ? 0.0f : 1.0f;
}

template <typename T>
__global__ void context_sim_kernel(const T* __restrict__ cur, const T* __restrict__ prev,
                                   float* __restrict__ sim, int rows, int d) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const T* pa = cur + (size_t)warp * d;
  const T* pb = prev + (size_t)warp * d;
  float dot = 0.0f, na = 0.0f, nb = 0.0f;
  for (int c = lane * 8; c < d; c += 256) {
    float va[8], vb[8];
    load8_stream(pa + c, va);
    load8_stream(pb + c, vb);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dot = fmaf(va[i], vb[i], dot);
      na = fmaf(va[i], va[i], na);
      nb = fmaf(vb[i], vb[i], nb);
    }
  }
  dot = warp_sum(dot);
  na = warp_sum(na);
  nb = warp_sum(nb);
  if (lane == 0) sim[warp] = dot / sqrtf(fmaxf(na * nb, 1e-24f));
}

constexpr int kCompactThreads = 1024;

// idx [B, L]: sequence b's rows with sim < tau, ascending, then -1; count [B].
__global__ void __launch_bounds__(kCompactThreads) compact_below_kernel(const float* __restrict__ sim, int L,
                                                                         float tau, int32_t* __restrict__ idx,
                                                                         int32_t* __restrict__ count) {
  __shared__ int warp_sums[33];
  const int b = blockIdx.x;
  const float* s = sim + (size_t)b * L;
  int32_t* out = idx + (size_t)b * L;
  const int per = (L + kCompactThreads - 1) / kCompactThreads;
  const int i0 = threadIdx.x * per, i1 = min(L, i0 + per);
  int n = 0;
  for (int i = i0; i < i1; ++i) n += s[i] < tau;
  int total;
  int pos = block_excl_scan(n, warp_sums, total);
  for (int i = i0; i < i1; ++i)
    if (s[i] < tau) out[pos++] = i;
  for (int i = total + threadIdx.x; i < L; i += kCompactThreads) out[i] = -1;
  if (threadIdx.x == 0) count[b] = total;
}

// Second skip point: the cached confidence of the k1 rows of each sequence
// that reached it (conf_sel[b*k1 + j] = conf[b*L + idx1[b*k1 + j]]), and the
// composition of the two selections: idx2[b*k2 + m] = idx1[b*k1 + j2[b*k2 + m]]
// (a position in [0, L)) and its global row b*L + idx2.
__global__ void gather_conf_kernel(const float* __restrict__ conf, const int32_t* __restrict__ idx1, int L,
                                   int k1, int rows, float* __restrict__ conf_sel) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows) return;
  conf_sel[i] = conf[(size_t)(i / k1) * L + idx1[i]];
}
__global__ void compose_idx_kernel(const int32_t* __restrict__ idx1, const int32_t* __restrict__ j2, int L,
                                   int k1, int k2, int rows, int32_t* __restrict__ idx2,
                                   int32_t* __restrict__ flat2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows) return;
  const int b = i / k2;
  const int p = idx1[(size_t)b * k1 + j2[i]];
  idx2[i] = p;
  flat2[i] = b * L + p;
}

// The rows of the current block [b0, b0 + R) of each sequence: positions
// pos[b*R + r] = b0 + r and tokens tok_blk[b*R + r] = tok[b*L + b0 + r].
__global__ void block_rows_kernel(const int32_t* __restrict__ tok, int L, int b0, int R, int rows,
                                  int32_t* __restrict__ pos, int32_t* __restrict__ tok_blk) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows) return;
  const int b = i / R, r = i - b * R;
  pos[i] = b0 + r;
  tok_blk[i] = tok[(size_t)b * L + b0 + r];
}

// Flat list of the salient rows of B sequences (one CTA per sequence):
// sequence b's count[b] positions idx[b*L ..] become rows b*L + i, stored at
// offset count[0] + ... + count[b-1].
__global__ void flatten_rows_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int L,
                                    int32_t* __restrict__ flat) {
  const int b = blockIdx.x;
  int off = 0;
  for (int j = 0; j < b; ++j) off += count[j];
  const int n = count[b];
  for (int i = threadIdx.x; i < n; i += blockDim.x) flat[off + i] = b * L + idx[(size_t)b * L + i];
}

// dst[dmap ? dmap[j] : j] = src[smap ? smap[j] : j] for n rows of d elements
// (one warp per row, 16-byte copies); with n_dev, only rows j < *n_dev (a
// count known on the device, at most n).
template <typename T>
__global__ void copy_rows_kernel(T* __restrict__ dst, const int32_t* __restrict__ dmap, const T* __restrict__ src,
                                 const int32_t* __restrict__ smap, int n, int d,
                                 const int32_t* __restrict__ n_dev = nullptr) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n || (n_dev && warp >= *n_dev)) return;
  const T* s = src + (size_t)(smap ? smap[warp] : warp) * d;
  T* o = dst + (size_t)(dmap ? dmap[warp] : warp) * d;
  for (int c = lane * 8; c < d; c += 256) copy8(o + c, s + c);
}

// Row capacities of the conditional bodies that take a count known only on
// the device (ascending; the last one is the largest count possible).
constexpr int kMaxBuckets = 48;
struct BucketCaps {
  int n;
  int cap[kMaxBuckets];
};

// The value of a switch node of a CUDA graph from the per-sequence counts
// count[0..B): with m their sum (use_max 0) or largest entry (use_max 1),
// base + the first k with caps.cap[k] >= m, or `none` when m is 0 (or above
// every capacity, which the capacities rule out). The sum also goes to *total
// when total is given. One warp.
__global__ void select_bucket_kernel(const int32_t* __restrict__ count, int B, int use_max, BucketCaps caps,
                                     unsigned base, unsigned none, cudaGraphConditionalHandle handle,
                                     int32_t* __restrict__ total) {
  int s = 0, m = 0;
  for (int b = threadIdx.x; b < B; b += 32) {
    const int v = count[b];
    s += v;
    m = max(m, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  }
  if (threadIdx.x != 0) return;
  if (total) *total = s;
  const int key = use_max ? m : s;
  unsigned v = none;
  if (key > 0)
    for (int k = 0; k < caps.n; ++k)
      if (caps.cap[k] >= key) {
        v = base + (unsigned)k;
        break;
      }
  cudaGraphSetConditional(handle, v);
}

__global__ void fill_i32_kernel(int32_t* __restrict__ p, int n, int v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

// ---------------------------------------------------------------------------
// x_sel[b*k + j] = x[b*L + idx[b,j]]; h_cache[b*L + idx[b,j]] = same (optional)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void gather_kernel(const T* __restrict__ x, const int32_t* __restrict__ idx, int L,
                              int k, int rows, int d, T* __restrict__ x_sel, T* __restrict__ hc,
                              int* flag) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const int b = warp / k;
  const int p = idx[warp];
  if (p < 0 || p >= L) {
    if (lane == 0) raise_flag(flag, kFlagCheck);
    return;
  }
  const size_t src_row = (size_t)b * L + p;
  const T* src = x + src_row * d;
  T* dst = x_sel + (size_t)warp * d;
  T* dh = hc ? hc + src_row * d : nullptr;
  for (int c = lane * 8; c < d; c += 256) {
    if constexpr (sizeof(T) == 2) {
      uint4 u = *reinterpret_cast<const uint4*>(src + c);
      *reinterpret_cast<uint4*>(dst + c) = u;
      if (dh) *reinterpret_cast<uint4*>(dh + c) = u;
    } else {
      float4 u0 = *reinterpret_cast<const float4*>(src + c);
      float4 u1 = *reinterpret_cast<const float4*>(src + c + 4);
      *reinterpret_cast<float4*>(dst + c) = u0;
      *reinterpret_cast<float4*>(dst + c + 4) = u1;
      if (dh) {
        *reinterpret_cast<float4*>(dh + c) = u0;
        *reinterpret_cast<float4*>(dh + c + 4) = u1;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Remask: per sequence, n_unmask rounds of a block-wide argmax over the masked
// positions of [b0, b1) by (conf desc, position asc). One CTA per sequence.
// When `params` is non-null the block range and n come from device memory
// (graph replays), otherwise from the arguments.
// ---------------------------------------------------------------------------
struct StepParams {
  int block_begin;
  int block_end;
  int n_unmask;
  int pad;
};

__global__ void remask_kernel(int32_t* __restrict__ tok, uint8_t* __restrict__ masked,
                              const float* __restrict__ conf, const int32_t* __restrict__ tok_c,
                              int L, int b0, int b1, int n, const StepParams* params) {
  __shared__ uint32_t s_key[32];
  __shared__ int s_pos[32];
  if (params) {
    b0 = params->block_begin;
    b1 = params->block_end;
    n = params->n_unmask;
  }
  const int b = blockIdx.x;
  int32_t* t = tok + (size_t)b * L;
  uint8_t* m = masked + (size_t)b * L;
  const float* c = conf + (size_t)b * L;
  const int32_t* tc = tok_c + (size_t)b * L;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int round = 0; round < n; ++round) {
    // best candidate of this thread: highest key, then lowest position
    uint32_t bk = 0u;
    int bp = INT_MAX;
    for (int i = b0 + threadIdx.x; i < b1; i += blockDim.x) {
      if (!m[i]) continue;
      uint32_t key = score_key(c[i]) + 1u;  // +1 so that any candidate beats "none" (0)
      if (key == 0u) key = 0xffffffffu;
      if (key > bk || (key == bk && i < bp)) { bk = key; bp = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      uint32_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
      int op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (ok > bk || (ok == bk && op < bp)) { bk = ok; bp = op; }
    }
    if (lane == 0) { s_key[w] = bk; s_pos[w] = bp; }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int j = 1; j < nw; ++j)
        if (s_key[j] > bk || (s_key[j] == bk && s_pos[j] < bp)) { bk = s_key[j]; bp = s_pos[j]; }
      if (bk != 0u && bp != INT_MAX) {
        t[bp] = tc[bp];
        m[bp] = 0;
      }
    }
    __syncthreads();
  }
}

__global__ void set_params_kernel(StepParams* p, int b0, int b1, int n) {
  p->block_begin = b0;
  p->block_end = b1;
  p->n_unmask = n;
}

// ---------------------------------------------------------------------------
// Head reduction: combine per-tile partials of each row into the confidence
// 1 / sum exp(l - l_max) and the argmax (lowest id on ties). Row r's result is
// written at r, or at b*L + idx[r] when idx is given (b = r / k).
// ---------------------------------------------------------------------------
__global__ void head_finalize_kernel(const HeadPartial* __restrict__ part, int rows, int n_tiles,
                                     const int32_t* __restrict__ idx, int L, int k,
                                     float* __restrict__ conf, int32_t* __restrict__ tok) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const HeadPartial* p = part + (size_t)warp * n_tiles;
  float m = 0.0f, s = 0.0f;
  int a = INT_MAX;
  for (int t = lane; t < n_tiles; t += 32) {
    HeadPartial q = p[t];
    head_merge(m, s, a, q.m, q.s, q.a);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    int a2 = __shfl_xor_sync(0xffffffffu, a, o);
    head_merge(m, s, a, m2, s2, a2);
  }
  if (lane == 0) {
    size_t dst = warp;
    if (idx) dst = (size_t)(warp / k) * L + idx[warp];
    conf[dst] = 1.0f / s;
    tok[dst] = a;
  }
}

// Partials of the head from a materialised float32 logits buffer [rows, V]
// (float32 models): one warp per (row, tile of `tile` columns).
__global__ void head_partials_from_logits(const float* __restrict__ logits, int rows, int V,
                                          int tile, int n_tiles, int mask_id,
                                          HeadPartial* __restrict__ part) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows * n_tiles) return;
  const int r = warp / n_tiles, t = warp % n_tiles;
  const float* l = logits + (size_t)r * V;
  const int c0 = t * tile, c1 = min(V, c0 + tile);
  float m = -INFINITY;
  int a = INT_MAX;
  for (int c = c0 + lane; c < c1; c += 32) {
    if (c == mask_id) continue;
    float v = l[c];
    if (v > m || (v == m && c < a)) { m = v; a = c; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    int a2 = __shfl_xor_sync(0xffffffffu, a, o);
    if (m2 > m || (m2 == m && a2 < a)) { m = m2; a = a2; }
  }
  float s = 0.0f;
  if (a != INT_MAX) {
    for (int c = c0 + lane; c < c1; c += 32) {
      if (c == mask_id) continue;
      s += expf(l[c] - m);
    }
  }
  s = warp_sum(s);
  if (lane == 0) part[warp] = HeadPartial{m, s, a};
}

// ---------------------------------------------------------------------------
// RoPE table: tab[p * half + j] = (cos, sin)(p * theta^(-2j/hd)), in float64
// then rounded to float32.
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float2* tab, int max_len, int half, double theta) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= max_len * half) return;
  const int p = i / half, j = i % half;
  const double freq = pow(theta, -2.0 * (double)j / (double)(2 * half));
  const double ang = (double)p * freq;
  tab[i] = make_float2((float)cos(ang), (float)sin(ang));
}

}  // namespace esd
