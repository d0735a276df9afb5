// Tensor-core GEMM for few gathered rows (M <= 256 tokens): C = A W^T with A
// the tokens [M, K] and W the weights [N, K], computed with the operand roles
// swapped: the MMA's M side is weight rows (output features) and its N side
// is the tokens, so D^T[feature, token] accumulates in TMEM (lanes = features,
// columns = tokens). A 192-token block is then one N = 192 MMA instead of a
// 128-row plus a half-used 64-row MMA, and no padded token rows are multiplied
// beyond the next multiple of 16.
//
// SM pairs (tcgen05 cta_group::2, a cluster of two CTAs): a pair-tile is 256
// weight rows; CTA r TMA-loads its own 128 weight rows and half r of the token
// block, and the leader's single thread issues M = 256, N = Mp MMAs. Each SM
// thus reads only half of the tokens per k-block: with 192 tokens the bytes an
// SM takes in per k-block are 16 KB of weights + 12 KB of tokens (the token
// re-reads of narrower tiles are the other half of the per-SM input budget,
// and that input path, not HBM, limits a one-SM version). No TMA load is
// multicast.
//
// Work is split over the W pairs in two phases: first floor(T / W) * W of the
// T pair-tiles go whole to the pairs, round robin; then the remaining tiles'
// (tile, 64-deep k-block) iterations are cut into W equal contiguous ranges,
// one per pair (stream-K), so every SM streams the same number of weight
// bytes whatever T is, and only the tiles of the second phase can be cut. A pair-tile
// that one pair covers whole is finished from TMEM by its epilogue; a cut
// tile's segments store fp32 partials (L2-resident workspace), and a second
// kernel, parallel over (tile half, 16-token chunk), adds them in k order and
// runs the same fused epilogue. No CTA waits for another; sums are in a fixed
// order, so results are deterministic.
//
// Warps: 0 TMA producer (both CTAs), 1 TMEM allocator + the leader's MMA
// issuer, 2..5 epilogue. Accumulators are double-buffered in TMEM (2 x 256
// columns), so a segment's epilogue overlaps the next segment's MMAs.
//
// The epilogue transposes each 16-token chunk through shared memory (fp32,
// [16 tokens][128 features], conflict-free padding) so that every fused
// operation is token-row local and every global access is a 16-byte vector,
// and it loads the next chunk's RoPE factors / residual rows while it finishes
// the current one:
//   QKV      : scale by the row's inverse RMS, rotate-half RoPE at the row's
//              position (pairs j, j + 64 of the head the CTA holds), store q
//              or scatter k / v into the layer's cache at the position;
//   SwiGLU   : the CTA's 128 rows = 64 gate + 64 up features:
//              act = silu(inv g) * inv u;
//   Residual : x = bf16(x + acc) for the O and down projections, and the sum
//              of squares of the 128 new x values per token, written as one
//              partial of the next RMS statistic (the consumer adds the d / 128
//              partials in tile order), so no separate statistics pass runs
//              between the layer's GEMMs.
// Every mbarrier wait is bounded; on expiry the kernel raises the error flag,
// stops issuing, drains what it issued and frees its TMEM; both CTAs of a pair
// always reach the final cluster barrier.
#pragma once

#include "tc_gemm2.cuh"

namespace esd {

constexpr int kSkThreads = 192;
constexpr int kSkMaxRows = 256;
constexpr int kSkStgStride = 132;           // floats per staged token row (128 + 4: conflict-free)
constexpr int kSkWBytes = 128 * 64 * 2;     // this CTA's weight rows of one stage
constexpr int kSkSmemFixed = 16 * kSkStgStride * 4 + 2 * kSkMaxRows * 4 + 4 * 16 * 4 + 512;
constexpr int kSkSmem = 232448 - 1024;      // dynamic shared memory requested (alignment slack inside)
constexpr int kSkTmemCols = 512;
constexpr int kSkMaxTiles = 1024;           // 128-row tiles of one GEMM the launcher accepts
constexpr size_t kSkPartFloats = (size_t)128 * kSkMaxRows;

__host__ __device__ constexpr int sk_stage_bytes(int mp) { return kSkWBytes + (mp / 2) * 128; }
__host__ __device__ constexpr int sk_stages(int mp) {
  return ((kSkSmem - 1024 - kSkSmemFixed) / sk_stage_bytes(mp)) > 8 ? 8
                                                                     : ((kSkSmem - 1024 - kSkSmemFixed) / sk_stage_bytes(mp));
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// the AND of `pred` over the 128 epilogue threads (named barrier 1)
__device__ __forceinline__ bool epi_all(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// A pair's segments: its whole tiles of the first phase (w, w + W, ... below
// p.sk_whole_tiles), then its range of the remaining tiles' k-blocks
// (stream-K over p.sk_total iterations). seg_no counts the second phase's
// segments only (0 = its first).
struct SkHyb {
  int W, kb, whole, next_whole;
  long long g, hi;
  int seg2;
  __device__ SkHyb(const GemmParams& p, int w, int kb_) : W(p.skw), kb(kb_), whole(p.sk_whole_tiles) {
    next_whole = w;
    g = sk_lo(p.sk_total, W, w);
    hi = sk_lo(p.sk_total, W, w + 1);
    seg2 = 0;
  }
  __device__ bool next(SkSeg& s) {
    if (next_whole < whole) {
      s.tile = next_whole;
      s.kb_a = 0;
      s.nkb = kb;
      s.full = true;
      s.seg_no = -1;
      next_whole += W;
      return true;
    }
    if (g >= hi) return false;
    const int t2 = (int)(g / kb);
    s.tile = whole + t2;
    s.kb_a = (int)(g - (long long)t2 * kb);
    const long long left = hi - g;
    s.nkb = (int)((long long)(kb - s.kb_a) < left ? (kb - s.kb_a) : left);
    s.full = (s.kb_a == 0 && s.nkb == kb);
    s.seg_no = seg2++;
    g += s.nkb;
    return true;
  }
};

// partial slot of a pair's segment (0: its first, 1: its last) for CTA rank
__host__ __device__ __forceinline__ size_t sk_slot(int pair, int which, int rank) {
  return ((size_t)pair * 2 + which) * 2 + rank;
}

// Global data one epilogue thread needs for a 16-token chunk, fetched one
// chunk ahead: thread e handles token t = e % 16 and feature group e / 16.
struct SkPre {
  float4 cs[4];  // QKV: (cos, sin) of 8 rotation pairs
  uint4 xu[2];   // residual: 16 bf16 of x
};

template <int KIND>
__device__ __forceinline__ void sk_prefetch(const GemmParams& p, int n128, int c0, int e, const int* pos_s,
                                            SkPre& pre) {
  const int t = e & 15, r = c0 + t;
  if (r >= p.M) return;
  if (KIND == kEpiQKV) {
    const int section = (n128 * 128) / p.d;
    if (section == 2 || pos_s[r] < 0) return;
    const float4* tab = reinterpret_cast<const float4*>(p.e.rope + (size_t)pos_s[r] * 64 + 8 * (e >> 4));
#pragma unroll
    for (int i = 0; i < 4; ++i) pre.cs[i] = tab[i];
  } else if (KIND == kEpiResidualO || KIND == kEpiResidualD) {
    const uint4* x = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.e.out) +
                                                    (size_t)r * p.d + n128 * 128 + 16 * (e >> 4));
    pre.xu[0] = x[0];
    pre.xu[1] = x[1];
  }
}

// Finish one 16-token chunk whose fp32 sums sit in stg [16][kSkStgStride]
// (row = token c0 + t, column = feature of the 128-row tile n128). All 128
// epilogue threads call it; it ends with the epilogue barrier.
template <int KIND>
__device__ __forceinline__ void sk_finish(const GemmParams& p, int n128, int c0, int e, const float* stg,
                                          const float* inv_s, const int* pos_s, float* red, const SkPre& pre) {
  const EpiArgs& ea = p.e;
  const int t = e & 15;
  const int r = c0 + t;
  // QKV: a negative position marks a padding row: nothing of it is written
  const bool live = r < p.M && (KIND != kEpiQKV || pos_s[r] >= 0);
  const int lane = e & 31, wq = e >> 5;
  if (KIND == kEpiQKV) {
    const int pg = e >> 4;  // dims 8pg..8pg+7 and their partners 64 further
    const int n0 = n128 * 128;
    const int section = n0 / p.d;
    const int h = (n0 - section * p.d) >> 7;
    if (live) {
      const float inv = inv_s[r];
      const float* row = stg + t * kSkStgStride;
      float lo[8], hi[8];
      *reinterpret_cast<float4*>(lo) = *reinterpret_cast<const float4*>(row + 8 * pg);
      *reinterpret_cast<float4*>(lo + 4) = *reinterpret_cast<const float4*>(row + 8 * pg + 4);
      *reinterpret_cast<float4*>(hi) = *reinterpret_cast<const float4*>(row + 64 + 8 * pg);
      *reinterpret_cast<float4*>(hi + 4) = *reinterpret_cast<const float4*>(row + 64 + 8 * pg + 4);
      const int pos = pos_s[r];
      const int b = r / ea.R;
      float o_lo[8], o_hi[8];
      if (section == 2) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o_lo[i] = lo[i] * inv;
          o_hi[i] = hi[i] * inv;
        }
      } else {
        const float2* cs = reinterpret_cast<const float2*>(pre.cs);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float a1 = lo[i] * inv, a2 = hi[i] * inv;
          o_lo[i] = a1 * cs[i].x - a2 * cs[i].y;
          o_hi[i] = a2 * cs[i].x + a1 * cs[i].y;
        }
      }
      __nv_bfloat16* dst = section == 0 ? reinterpret_cast<__nv_bfloat16*>(ea.out) + (size_t)r * p.d + h * 128
                                        : reinterpret_cast<__nv_bfloat16*>(section == 1 ? ea.k_dst : ea.v_dst) +
                                              ((size_t)b * ea.L + pos) * p.d + h * 128;
      uint4 u_lo, u_hi;
      __nv_bfloat162* hl = reinterpret_cast<__nv_bfloat162*>(&u_lo);
      __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&u_hi);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        hl[i] = __floats2bfloat162_rn(o_lo[2 * i], o_lo[2 * i + 1]);
        hh[i] = __floats2bfloat162_rn(o_hi[2 * i], o_hi[2 * i + 1]);
      }
      *reinterpret_cast<uint4*>(dst + 8 * pg) = u_lo;
      *reinterpret_cast<uint4*>(dst + 64 + 8 * pg) = u_hi;
    }
  } else if (KIND == kEpiSwiGLU) {
    const int pg = e >> 4;  // features 8pg..8pg+7 of the CTA's 64
    if (live) {
      const float inv = inv_s[r];
      const float* row = stg + t * kSkStgStride;
      float g[8], u[8];
      *reinterpret_cast<float4*>(g) = *reinterpret_cast<const float4*>(row + 8 * pg);
      *reinterpret_cast<float4*>(g + 4) = *reinterpret_cast<const float4*>(row + 8 * pg + 4);
      *reinterpret_cast<float4*>(u) = *reinterpret_cast<const float4*>(row + 64 + 8 * pg);
      *reinterpret_cast<float4*>(u + 4) = *reinterpret_cast<const float4*>(row + 64 + 8 * pg + 4);
      uint4 o4;
      __nv_bfloat162* ho = reinterpret_cast<__nv_bfloat162*>(&o4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float o2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float gg = g[2 * i + j] * inv;
          // silu with the fast exponential and divide (relative error ~1e-6,
          // far below the bf16 rounding of the product)
          o2[j] = __fdividef(gg, 1.0f + __expf(fminf(-gg, 80.0f))) * (u[2 * i + j] * inv);
        }
        ho[i] = __floats2bfloat162_rn(o2[0], o2[1]);
      }
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(ea.out) + (size_t)r * p.ffn + n128 * 64 + 8 * pg) = o4;
    }
  } else {  // residual
    const int gq = e >> 4;  // features 16gq..16gq+15 of the tile's 128
    float ss = 0.0f;
    if (live) {
      const float* row = stg + t * kSkStgStride + 16 * gq;
      __nv_bfloat16* x = reinterpret_cast<__nv_bfloat16*>(ea.out) + (size_t)r * p.d + n128 * 128 + 16 * gq;
      const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(pre.xu);
      uint4 ou[2];
      __nv_bfloat162* ho = reinterpret_cast<__nv_bfloat162*>(ou);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 xf = __bfloat1622float2(hx[i]);
        const float2 af = *reinterpret_cast<const float2*>(row + 2 * i);
        ho[i] = __floats2bfloat162_rn(xf.x + af.x, xf.y + af.y);
        const float2 of = __bfloat1622float2(ho[i]);
        ss = fmaf(of.x, of.x, ss);
        ss = fmaf(of.y, of.y, ss);
      }
      reinterpret_cast<uint4*>(x)[0] = ou[0];
      reinterpret_cast<uint4*>(x)[1] = ou[1];
    }
    if (ea.rms_part_out) {
      // the tile's sum of squares per token: lanes t and t + 16 of warp j of
      // the group hold feature groups 2j and 2j + 1 of token t
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);
      if (lane < 16) red[wq * 16 + lane] = ss;
      epi_bar();
      if (e < 16 && c0 + e < p.M)
        ea.rms_part_out[(size_t)n128 * kSkMaxRows + c0 + e] = ((red[e] + red[16 + e]) + red[32 + e]) + red[48 + e];
    }
  }
  epi_bar();
}

// The inverse RMS of rows [r0, r1) into inv_s (from the partial sums of
// squares, or copied from inv_rms), and for QKV each row's position into pos_s.
template <int KIND>
__device__ __forceinline__ void sk_row_setup(const GemmParams& p, int r0, int r1, int e, float* inv_s, int* pos_s) {
  const EpiArgs& ea = p.e;
  for (int r = r0 + e; r < r1 && r < p.M; r += 128) {
    if (KIND == kEpiQKV || KIND == kEpiSwiGLU) {
      if (ea.rms_parts > 0) {
        float s = 0.0f;
        for (int q = 0; q < ea.rms_parts; ++q) s += ea.rms_part_in[(size_t)q * kSkMaxRows + r];
        inv_s[r] = 1.0f / sqrtf(s / (float)p.d + ea.rms_eps);
      } else {
        inv_s[r] = ea.inv_rms[r];
      }
    }
    if (KIND == kEpiQKV) pos_s[r] = ea.idx ? ea.idx[r] : r % ea.R;
  }
}

// grid.x = 2 * pairs, cluster (2, 1, 1); rank in the cluster = CTA r of the pair.
template <int KIND>
__global__ void __launch_bounds__(kSkThreads, 1)
tc_skinny_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                 const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                 const GemmParams p) {
  const int mp = p.mp, stages = p.stages;
  const int stage_bytes = sk_stage_bytes(mp);
  extern __shared__ __align__(1024) uint8_t smem_raw_sk[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw_sk + 1023) & ~(uintptr_t)1023);
  float* stg = reinterpret_cast<float*>(smem + stages * stage_bytes);  // [16][kSkStgStride]
  float* inv_s = stg + 16 * kSkStgStride;                              // [256]
  int* pos_s = reinterpret_cast<int*>(inv_s + kSkMaxRows);             // [256]
  float* red = reinterpret_cast<float*>(pos_s + kSkMaxRows);           // [4][16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 64);
  uint64_t* full = bars;
  uint64_t* empty = bars + 8;
  uint64_t* tfull = bars + 16;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);   // leader: its own expect_tx arrive (+ both CTAs' bytes)
      mbar_init(smem_u32(&empty[i]), 1);  // both: the leader's multicast commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);   // both: multicast commit
      mbar_init(smem_u32(&tempty[i]), 8);  // leader: 4 epilogue warps x 2 CTAs
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), kSkTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer signals the leader's barriers from here on
  tc_fence_after();
  // the prologue above may overlap the previous kernel; the producers stream
  // the first weight stages before waiting for it, every other global access
  // of this kernel follows a grid-dependency wait
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const int kb_total = p.K / 64;
  const int pair = blockIdx.x >> 1;
  const int half_rows = mp / 2;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
      const uint32_t tx = 2u * (uint32_t)stage_bytes;
      int npre = 0;
      {
        SkHyb it0(p, pair, kb_total);
        SkSeg s0;
        if (it0.next(s0)) {
          int sel, row0, row1;
          b_rows<KIND, 128>(2 * s0.tile + (int)rank, p, sel, row0, row1);
          const CUtensorMap* mb0 = sel == 0 ? &tmB0 : (sel == 1 ? &tmB1 : &tmB2);
          const CUtensorMap* mb1 = (KIND == kEpiSwiGLU) ? &tmB1 : mb0;
          npre = s0.nkb < stages ? s0.nkb : stages;
          for (int i = 0; i < npre; ++i) {
            if (rank == 0) mbar_expect_tx(smem_u32(&full[i]), tx);
            const uint32_t fb = mapa_shared(smem_u32(&full[i]), 0);
            uint8_t* wb = smem + i * stage_bytes;
            const int k0 = (s0.kb_a + i) * 64;
            tma_load_2d_pair(smem_u32(wb), mb0, fb, k0, row0, pol_w);
            tma_load_2d_pair(smem_u32(wb + kSkWBytes / 2), mb1, fb, k0, row1, pol_w);
          }
        }
      }
      grid_dependency_wait();
      int stage = 0;
      uint32_t phase = 0;
      int gi = 0;
      uint32_t used = 0, last_phase = 0;  // per stage: loaded at least once / parity of its last load
      SkHyb it(p, pair, kb_total);
      SkSeg sg;
      while (!*abort_flag && it.next(sg)) {
        int sel, row0, row1;
        b_rows<KIND, 128>(2 * sg.tile + (int)rank, p, sel, row0, row1);
        const CUtensorMap* mb0 = sel == 0 ? &tmB0 : (sel == 1 ? &tmB1 : &tmB2);
        const CUtensorMap* mb1 = (KIND == kEpiSwiGLU) ? &tmB1 : mb0;
        bool ok = true;
        for (int i = 0; i < sg.nkb; ++i) {
          const int k0 = (sg.kb_a + i) * 64;
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* sbase = smem + stage * stage_bytes;
          if (gi >= npre) {  // (the first npre stages already hold their weights)
            if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.flag)) { ok = false; break; }
            if (rank == 0) mbar_expect_tx(smem_u32(&full[stage]), tx);
            tma_load_2d_pair(smem_u32(sbase), mb0, fb, k0, row0, pol_w);
            tma_load_2d_pair(smem_u32(sbase + kSkWBytes / 2), mb1, fb, k0, row1, pol_w);
          }
          tma_load_2d_pair(smem_u32(sbase + kSkWBytes), &tmA, fb, k0, (int)rank * half_rows, pol_a);
          ++gi;
          used |= 1u << stage;
          last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // drain: this CTA's loads have landed (the leader's full barriers count
      // both CTAs' bytes; the peer waits for its stages to be consumed)
      for (int i = 0; i < stages; ++i)
        if ((used >> i) & 1u) {
          const uint32_t bar = rank == 0 ? smem_u32(&full[i]) : smem_u32(&empty[i]);
          for (uint32_t k = 0; k < kWaitLimit; ++k)
            if (mbar_try_wait(bar, ((last_phase >> i) & 1u))) break;
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader CTA only)
      const uint32_t idesc = idesc_bf16(256, mp);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      SkHyb it(p, pair, kb_total);
      SkSeg sg;
      while (!*abort_flag && it.next(sg)) {
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.flag)) break;
        tc_fence_after();
        const uint32_t tacc = tmem + (uint32_t)(acc * 256);
        bool ok = true;
        for (int i = 0; i < sg.nkb; ++i) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.flag)) { ok = false; break; }
          const uint32_t wbase = smem_u32(smem + stage * stage_bytes);
          const uint32_t tbase = wbase + kSkWBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_pair(tacc, smem_desc_sw128(wbase + kk * 32), smem_desc_sw128(tbase + kk * 32), idesc,
                        (i | kk) != 0 ? 1u : 0u);
          issued = true;
          tc_commit_pair_both(smem_u32(&empty[stage]));
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_both(smem_u32(&tfull[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (issued) {
        tc_commit_pair_own(smem_u32(drain));
        for (uint32_t k = 0; k < kWaitLimit; ++k)
          if (mbar_try_wait(smem_u32(drain), 0u)) break;
      }
    }
  } else {
    // ---------------- epilogue warps 2..5 (both CTAs): this CTA's 128 rows
    grid_dependency_wait();
    const int e = threadIdx.x - 64;      // 0..127: the transposed work item
    const int quarter = warp & 3;        // TMEM lane quarter of this warp
    const int f = quarter * 32 + lane;   // feature row of the CTA's 128 this thread reads
    sk_row_setup<KIND>(p, 0, mp, e, inv_s, pos_s);
    if ((KIND == kEpiQKV || KIND == kEpiSwiGLU) && blockIdx.x == 0 && p.e.rms_parts > 0)
      for (int r = e; r < p.M; r += 128) p.e.inv_out[r] = inv_s[r];  // for the cut-tile kernel
    epi_bar();
    int acc = 0;
    uint32_t acc_phase = 0;
    SkHyb it(p, pair, kb_total);
    SkSeg sg;
    while (it.next(sg)) {
      // one decision for all four warps: they meet at named barriers below
      if (!epi_all(mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.flag))) break;
      tc_fence_after();
      const uint32_t tacc = tmem + (uint32_t)(acc * 256) + ((uint32_t)(quarter * 32) << 16);
      const int n128 = 2 * sg.tile + (int)rank;
      if (!sg.full) {
        // a cut tile: this segment's partial to its slot (the reduction
        // kernel finishes the tile)
        float* wt = p.ws + sk_slot(pair, sg.seg_no == 0 ? 0 : 1, (int)rank) * kSkPartFloats;
        for (int c = 0; c < mp; c += 32) {
          float v[2][16];
          tmem_ld16(tacc + (uint32_t)c, v[0]);
          if (c + 16 < mp) tmem_ld16(tacc + (uint32_t)(c + 16), v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (c + 16 * h >= mp) break;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              __stcg(reinterpret_cast<float4*>(wt + ws_index((c >> 4) + h, q, f, 128)),
                     make_float4(v[h][4 * q], v[h][4 * q + 1], v[h][4 * q + 2], v[h][4 * q + 3]));
          }
        }
      } else {
        SkPre cur{}, nxt{};
        sk_prefetch<KIND>(p, n128, 0, e, pos_s, cur);
        for (int c0 = 0; c0 < mp; c0 += 16) {
          float v[16];
          tmem_ld16(tacc + (uint32_t)c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) stg[i * kSkStgStride + f] = v[i];
          if (c0 + 16 < mp) sk_prefetch<KIND>(p, n128, c0 + 16, e, pos_s, nxt);
          epi_bar();
          sk_finish<KIND>(p, n128, c0, e, stg, inv_s, pos_s, red, cur);
          cur = nxt;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kSkTmemCols);
}

// Cut tiles: block = (pair-tile of the second phase, CTA half, 16-token
// chunk), 128 threads; adds the tile's segment partials in k order and runs
// the fused epilogue. A second-phase tile that one pair covered whole returns
// at once.
template <int KIND>
__global__ void __launch_bounds__(128)
tc_skinny_fixup_kernel(const GemmParams p) {
  __shared__ float stg[16 * kSkStgStride];
  __shared__ float inv_s[kSkMaxRows];
  __shared__ int pos_s[kSkMaxRows];
  __shared__ float red[64];
  grid_launch_dependents();  // the next kernel's prologue and weight loads may start
  grid_dependency_wait();
  const int nch = p.mp / 16;
  int bid = blockIdx.x;
  const int ch = bid % nch;
  bid /= nch;
  const int rank = bid & 1;
  const int tile = p.sk_whole_tiles + (bid >> 1);  // the grid covers the second phase's tiles only
  const int kb = p.K / 64;
  const long long T = p.sk_total;
  const long long g0 = (long long)(tile - p.sk_whole_tiles) * kb;
  const int w0 = sk_worker(T, p.skw, g0), w1 = sk_worker(T, p.skw, g0 + kb - 1);
  if (w0 == w1) return;
  const int e = threadIdx.x, f = threadIdx.x;
  const int c0 = ch * 16;
  const int n128 = 2 * tile + rank;
  // the first segments' partial loads go out before anything else (they
  // depend on nothing but the block), then the rows' inverse RMS, positions
  // and RoPE factors, then the adds in k order
  constexpr int kMaxSeg = 4;
  float4 x4[kMaxSeg][4];
#pragma unroll
  for (int j = 0; j < kMaxSeg; ++j) {
    const int ww = w0 + j;
    if (ww > w1) break;
    const int which = (ww == w0 && sk_lo(T, p.skw, ww) < g0) ? 1 : 0;
    const float* b = p.ws + sk_slot(ww, which, rank) * kSkPartFloats;
#pragma unroll
    for (int q = 0; q < 4; ++q) x4[j][q] = __ldcg(reinterpret_cast<const float4*>(b + ws_index(ch, q, f, 128)));
  }
  SkPre pre{};
  if (e < 16 && c0 + e < p.M) {
    const int r = c0 + e;
    if (KIND == kEpiQKV || KIND == kEpiSwiGLU) inv_s[r] = p.e.rms_parts > 0 ? p.e.inv_out[r] : p.e.inv_rms[r];
    if (KIND == kEpiQKV) pos_s[r] = p.e.idx ? p.e.idx[r] : r % p.e.R;
  }
  __syncthreads();
  sk_prefetch<KIND>(p, n128, c0, e, pos_s, pre);
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = 0.0f;
  for (int wb = w0; wb <= w1; wb += kMaxSeg) {
    if (wb != w0) {
#pragma unroll
      for (int j = 0; j < kMaxSeg; ++j) {
        const int ww = wb + j;
        if (ww > w1) break;
        const float* b = p.ws + sk_slot(ww, 0, rank) * kSkPartFloats;
#pragma unroll
        for (int q = 0; q < 4; ++q) x4[j][q] = __ldcg(reinterpret_cast<const float4*>(b + ws_index(ch, q, f, 128)));
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxSeg; ++j) {
      if (wb + j > w1) break;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[4 * q] += x4[j][q].x;
        v[4 * q + 1] += x4[j][q].y;
        v[4 * q + 2] += x4[j][q].z;
        v[4 * q + 3] += x4[j][q].w;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) stg[i * kSkStgStride + f] = v[i];
  epi_bar();
  sk_finish<KIND>(p, n128, c0, e, stg, inv_s, pos_s, red, pre);
}

// The RMS statistic of `rows` rows of x [rows, d] as the swapped-operand
// GEMMs consume it: per 128-feature tile n and row r, part[n][r] = the sum of
// squares of the 128 values, added in the residual epilogue's exact order
// (16 sequential fused multiply-adds per group of 16 features, then groups
// (0+1), (2+3), (4+5), (6+7), then those four left to right), so that a
// statistic from this kernel and one from a residual epilogue are the same
// bits. One thread per (row, tile).
__global__ void rms_part_kernel(const __nv_bfloat16* __restrict__ x, int rows, int d, float* __restrict__ part) {
  const int ntiles = d >> 7;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * ntiles) return;
  const int r = i / ntiles, n = i - r * ntiles;
  const uint4* px = reinterpret_cast<const uint4*>(x + (size_t)r * d + n * 128);
  float pr[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float s2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 u[2];
      u[0] = px[(2 * j + h) * 2];
      u[1] = px[(2 * j + h) * 2 + 1];
      const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(u);
      float ss = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 fv = __bfloat1622float2(hx[k]);
        ss = fmaf(fv.x, fv.x, ss);
        ss = fmaf(fv.y, fv.y, ss);
      }
      s2[h] = ss;
    }
    pr[j] = s2[0] + s2[1];
  }
  part[(size_t)n * kSkMaxRows + r] = ((pr[0] + pr[1]) + pr[2]) + pr[3];
}

template <int KIND>
inline void tc_skinny_set_attr() {
  cudaFuncSetAttribute(tc_skinny_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSkSmem);
}

inline void tc_skinny_set_attr_all() {
  tc_skinny_set_attr<kEpiQKV>();
  tc_skinny_set_attr<kEpiResidualO>();
  tc_skinny_set_attr<kEpiSwiGLU>();
  tc_skinny_set_attr<kEpiResidualD>();
}

// Whether the swapped-operand kernel takes a GEMM of M rows: the layer widths
// give an even number of 128-row tiles of every GEMM (pair-tiles of 256).
inline bool tc_skinny_ok(const TcPlan& pl, int M) {
  const int d = pl.w.d, f = pl.w.ffn;
  return M >= 1 && M <= kSkMaxRows && d % 256 == 0 && f % 128 == 0 && pl.ws && pl.num_sms >= 2 &&
         pl.ws_floats >= (size_t)4 * (pl.num_sms / 2) * kSkPartFloats && 3 * d / 128 <= kSkMaxTiles &&
         f / 64 <= kSkMaxTiles;
}

template <int KIND>
inline cudaError_t tc_skinny_launch(const TcPlan& pl, const void* A, const CUtensorMap& b0, const CUtensorMap& b1,
                                    const CUtensorMap& b2, GemmParams p, cudaStream_t st, uint64_t* launches) {
  const int mp = (p.M + 15) / 16 * 16;
  CUtensorMap a;
  if (!encode_2d(pl, &a, A, (uint64_t)p.M, (uint64_t)p.K, (uint32_t)(mp / 2))) return cudaErrorInvalidValue;
  int tiles128;
  if (KIND == kEpiQKV) tiles128 = 3 * p.d / 128;
  else if (KIND == kEpiSwiGLU) tiles128 = p.ffn / 64;
  else tiles128 = p.d / 128;
  const int tiles = tiles128 / 2;  // pair-tiles of 256 weight rows
  p.mp = mp;
  p.stages = sk_stages(mp);
  p.num_m = 1;
  p.num_n = tiles;
  p.num_tiles = tiles;
  p.splits = 1;
  p.num_units = tiles;
  p.ws = pl.ws;
  const int kb = p.K / 64;
  long long wk = (long long)tiles * kb / 4;  // at least 4 k-blocks per pair
  if (wk > pl.num_sms / 2) wk = pl.num_sms / 2;
  if (wk < 1) wk = 1;
  p.skw = (int)wk;
  p.sk_whole = 0;
  p.sk_whole_tiles = (tiles / p.skw) * p.skw;
  p.sk_total = (long long)(tiles - p.sk_whole_tiles) * kb;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.skw, 1, 1);
  cfg.blockDim = dim3(kSkThreads, 1, 1);
  cfg.dynamicSmemBytes = kSkSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the previous kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tc_skinny_kernel<KIND>, a, b0, b1, b2, p);
  (*launches)++;
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // cut tiles exist unless every second-phase range boundary falls on a tile boundary
  bool cut = false;
  for (int w = 1; w < p.skw && !cut && p.sk_total > 0; ++w) cut = (sk_lo(p.sk_total, p.skw, w) % kb) != 0;
  if (!cut) return cudaSuccess;
  cudaLaunchConfig_t c2 = {};
  c2.gridDim = dim3((tiles - p.sk_whole_tiles) * 2 * (mp / 16), 1, 1);
  c2.blockDim = dim3(128, 1, 1);
  c2.stream = st;
  cudaLaunchAttribute a2[1];
  a2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a2[0].val.programmaticStreamSerializationAllowed = 1;
  c2.attrs = a2;
  c2.numAttrs = 1;
  e = cudaLaunchKernelEx(&c2, tc_skinny_fixup_kernel<KIND>, p);
  (*launches)++;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace esd
