// Two-SM tensor-core GEMM (tcgen05 cta_group::2) for tiles of 256 activation
// rows x BN weight rows (BN 256, or 192 for the SwiGLU GEMM of few rows, where
// 96 gate + 96 up rows make 128 tiles for the 74 SM pairs instead of 96),
// used when a GEMM has more than 128 rows.
//
// A cluster of two CTAs on two SMs shares one tile: CTA r loads activation rows
// [128r, 128r + 128) and half r of the weight tile (the same halves as the
// one-SM kernel: two heads, gate|up, or two contiguous column blocks), both into
// its own shared memory, signalling the leader CTA's "full" barrier. The
// leader's single MMA thread issues tcgen05.mma.cta_group::2 with M = 256,
// N = 256: each SM multiplies its own 128 rows by the whole 256-column weight
// tile while reading only its half of it, which halves the shared-memory operand
// traffic per FLOP of the one-SM 256x128 tile. Commits are multicast to both
// CTAs' barriers; each CTA's epilogue reads its 128 rows x 256 columns of TMEM
// (double-buffered) and runs the same fused epilogues as the one-SM kernel.
//
// Work split: with at least half as many tiles as SM pairs, each pair takes a
// contiguous range of whole tiles. With fewer tiles (the N = d projections of
// the selected rows), stream-K: the T = tiles x k-blocks iterations are cut into
// W equal contiguous ranges, one per pair; a tile wholly inside one range is
// finished by that pair's epilogue, a tile cut by range boundaries is
// accumulated as fp32 partials (at most two per pair: its first and its last
// segment) that a reduction kernel sums in k order and finishes with the same
// epilogue. Both are deterministic. No TMA load is multicast.
#pragma once

#include "tc_gemm.cuh"

namespace esd {

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
// address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on a
// barrier of the leader CTA (cta_group::2 form, no multicast)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this offset in both CTAs once the issued MMAs finish
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair_own(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Stream-K: worker w covers global iterations [lo(w), lo(w+1)).
__host__ __device__ __forceinline__ long long sk_lo(long long T, int W, int w) {
  return (long long)w * T / W;
}
// the worker whose range holds global iteration g
__host__ __device__ __forceinline__ int sk_worker(long long T, int W, long long g) {
  return (int)(((g + 1) * W - 1) / T);
}

// One segment of a worker's range: k-blocks [kb_a, kb_a + nkb) of `tile`.
struct SkSeg {
  int tile, kb_a, nkb, seg_no;
  bool full;
};

struct SkIter {
  long long g, hi;
  int kb_total, seg_no;
  __device__ SkIter(const GemmParams& p, int w, int kb_total_) {
    if (p.sk_whole) {
      g = (long long)w * p.num_tiles / p.skw * kb_total_;
      hi = (long long)(w + 1) * p.num_tiles / p.skw * kb_total_;
    } else {
      g = sk_lo(p.sk_total, p.skw, w);
      hi = sk_lo(p.sk_total, p.skw, w + 1);
    }
    kb_total = kb_total_;
    seg_no = 0;
  }
  __device__ bool next(SkSeg& s) {
    if (g >= hi) return false;
    s.tile = (int)(g / kb_total);
    s.kb_a = (int)(g - (long long)s.tile * kb_total);
    const long long left = hi - g;
    s.nkb = (int)((long long)(kb_total - s.kb_a) < left ? (kb_total - s.kb_a) : left);
    s.full = (s.kb_a == 0 && s.nkb == kb_total);
    s.seg_no = seg_no++;
    g += s.nkb;
    return true;
  }
};

// partial slot of a worker's segment: 0 for its first, 1 for its last
__device__ __forceinline__ size_t sk_slot(int w, int seg_no) { return (size_t)w * 2 + (seg_no == 0 ? 0 : 1); }

template <int BN>
struct Tc2Cfg {
  static_assert(BN == 256 || BN == 192, "tile width");
  static constexpr int kBK = 64;
  static constexpr int kABytes = 128 * kBK * 2;       // this CTA's 128 activation rows
  static constexpr int kBBytes = (BN / 2) * kBK * 2;  // this CTA's half of the BN weight rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = ((232448 - 1280) / kStageBytes) > 8 ? 8 : ((232448 - 1280) / kStageBytes);
  static constexpr int kAcc = 2;
  static constexpr int kTmemCols = 512;  // 2 x BN fp32 columns
  static constexpr int kSmem = kStages * kStageBytes + 1024 + 256;
  static constexpr int kTileRows = 256;
};

// warps: 0 TMA, 1 TMEM + MMA (leader), 2..9 epilogue (two warps per TMEM lane
// quarter, each with half of the tile's columns)
constexpr int kTc2Threads = 320;

template <int KIND, int BN>
__global__ void __launch_bounds__(kTc2Threads, 1)
tc_gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                const GemmParams p) {
  using C = Tc2Cfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw2[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw2 + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tfull = bars + 2 * C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);   // leader: its own expect_tx arrive (+ both CTAs' bytes)
      mbar_init(smem_u32(&empty[i]), 1);  // both: the leader's multicast commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);   // both: multicast commit
      mbar_init(smem_u32(&tempty[i]), 16);  // leader: 8 epilogue warps x 2 CTAs
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer signals the leader's barriers from here on
  tc_fence_after();
  // the prologue above may overlap the previous kernel; the producers stream
  // the first weight stages before waiting for it, every other global access
  // of this kernel follows a grid-dependency wait
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const int kb_total = p.K / C::kBK;
  const int pair = blockIdx.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_phase = 0;  // per stage: loaded at least once / parity of its last load
      // the weights of the first stages of this pair's first segment do not
      // depend on the previous kernel: stream them while it finishes
      int npre = 0;
      {
        SkIter it0(p, pair, kb_total);
        SkSeg s0;
        if (it0.next(s0)) {
          const int koff0 = (int)(((unsigned)s0.tile * 7u + (unsigned)s0.kb_a) % (unsigned)s0.nkb);
          int sel, row0, row1;
          b_rows<KIND, BN>(s0.tile / p.num_m, p, sel, row0, row1);
          const CUtensorMap* mb = sel == 0 ? &tmB0 : (sel == 1 ? &tmB1 : &tmB2);
          if (KIND == kEpiSwiGLU && rank == 1) mb = &tmB1;
          npre = s0.nkb < C::kStages ? s0.nkb : C::kStages;
          for (int i = 0; i < npre; ++i) {
            int kb = koff0 + i;
            if (kb >= s0.nkb) kb -= s0.nkb;
            kb += s0.kb_a;
            if (rank == 0) mbar_expect_tx(smem_u32(&full[i]), 2u * C::kStageBytes);
            tma_load_2d_pair(smem_u32(smem + i * C::kStageBytes + C::kABytes), mb,
                             mapa_shared(smem_u32(&full[i]), 0), kb * C::kBK, rank ? row1 : row0, pol_w);
          }
        }
      }
      grid_dependency_wait();
      int gi = 0;  // iterations issued, over all segments
      SkIter it(p, pair, kb_total);
      SkSeg sg;
      while (!*abort_flag && it.next(sg)) {
        const int tile = sg.tile, kb0 = sg.kb_a, nkb = sg.nkb;
        const int koff = (int)(((unsigned)tile * 7u + (unsigned)kb0) % (unsigned)nkb);
        const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
        int sel, row0, row1;
        b_rows<KIND, BN>(n_blk, p, sel, row0, row1);
        const CUtensorMap* mb = sel == 0 ? &tmB0 : (sel == 1 ? &tmB1 : &tmB2);
        if (KIND == kEpiSwiGLU && rank == 1) mb = &tmB1;  // up rows
        const int my_row = rank ? row1 : row0;
        for (int i = 0; i < nkb; ++i) {
          int kb = koff + i;
          if (kb >= nkb) kb -= nkb;
          kb += kb0;
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* sbase = smem + stage * C::kStageBytes;
          const int k0 = kb * C::kBK;
          if (gi >= npre) {  // (the first npre stages already hold their weights)
            if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.flag)) break;
            if (rank == 0) mbar_expect_tx(smem_u32(&full[stage]), 2u * C::kStageBytes);
            tma_load_2d_pair(smem_u32(sbase + C::kABytes), mb, fb, k0, my_row, pol_w);
          }
          tma_load_2d_pair(smem_u32(sbase), &tmA, fb, k0, m_blk * C::kTileRows + (int)rank * 128, pol_a);
          ++gi;
          used |= 1u << stage;
          last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // drain: this CTA's loads have landed (the leader's full barriers count
      // both CTAs' bytes; the peer waits for its stages to be consumed)
      for (int i = 0; i < C::kStages; ++i)
        if ((used >> i) & 1u) {
          const uint32_t bar = rank == 0 ? smem_u32(&full[i]) : smem_u32(&empty[i]);
          const uint32_t par = (last_phase >> i) & 1u;
          for (uint32_t it = 0; it < kWaitLimit; ++it)
            if (mbar_try_wait(bar, par)) break;
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader CTA only)
      constexpr uint32_t idesc = idesc_bf16(256, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      SkIter it(p, pair, kb_total);
      SkSeg sg;
      while (!*abort_flag && it.next(sg)) {
        const int nkb = sg.nkb;
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.flag)) break;
        tc_fence_after();
        const uint32_t tacc = tmem + (uint32_t)(acc * BN);
        bool ok = true;
        for (int i = 0; i < nkb; ++i) {
          // the TMA bytes are ordered before the MMA's operand reads by the
          // barrier itself (both in the async proxy): no thread fence needed
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.flag)) { ok = false; break; }
          const uint32_t sbase = smem_u32(smem + stage * C::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < C::kBK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sbase + kk * 32);
            const uint64_t bdesc = smem_desc_sw128(sbase + C::kABytes + kk * 32);
            tc_mma_pair(tacc, adesc, bdesc, idesc, (i | kk) != 0 ? 1u : 0u);
          }
          issued = true;
          tc_commit_pair_both(smem_u32(&empty[stage]));
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_both(smem_u32(&tfull[acc]));
        if (++acc == C::kAcc) { acc = 0; acc_phase ^= 1u; }
      }
      if (issued) {
        tc_commit_pair_own(smem_u32(drain));
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(drain), 0u)) break;
      }
    }
  } else {
    // ---------------- epilogue warps 2..9 (both CTAs): this CTA's 128 rows
    grid_dependency_wait();
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // columns [half * BN / 2, (half + 1) * BN / 2)
    constexpr int G = epi_groups<KIND, BN>();
    int acc = 0;
    uint32_t acc_phase = 0;
    SkIter it(p, pair, kb_total);
    SkSeg sg;
    while (it.next(sg)) {
      const int tile = sg.tile;
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.flag)) break;
      tc_fence_after();
      const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
      const uint32_t tacc = tmem + (uint32_t)(acc * BN) + ((uint32_t)(quarter * 32) << 16);
      const int lr = (int)rank * 128 + quarter * 32 + lane;
      const int r = m_blk * C::kTileRows + lr;
      if (sg.full) {
        epilogue_rows<KIND, BN>(p, n_blk, r, r < p.M, TmemSrc{tacc}, half * G / 2, (half + 1) * G / 2);
      } else {
        const size_t split_stride = (size_t)C::kTileRows * BN;
        float* wt = p.ws + sk_slot(pair, sg.seg_no) * split_stride;
        const uint64_t pol_keep = policy_evict_last();
        const bool live = r < p.M;
#pragma unroll 4
        for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 16) {
          float v[16];
          tmem_ld16(tacc + (uint32_t)c, v);
          tmem_ld_wait();
          if (live) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_f4_keep(wt + ws_index(c >> 4, q, lr, C::kTileRows),
                         make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]), pol_keep);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (++acc == C::kAcc) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, C::kTmemCols);
}

template <int KIND, int BN>
inline void tc2_set_attr() {
  cudaFuncSetAttribute(tc_gemm2_kernel<KIND, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, Tc2Cfg<BN>::kSmem);
}

inline void tc2_set_attr_all() {
  tc2_set_attr<kEpiQKV, 256>();
  tc2_set_attr<kEpiResidualO, 256>();
  tc2_set_attr<kEpiSwiGLU, 256>();
  tc2_set_attr<kEpiSwiGLU, 192>();
  tc2_set_attr<kEpiResidualD, 256>();
}

// Partials of a stream-K tile cut by range boundaries, summed in k order:
// the first worker's segment (its first or its last slot), then the first slot
// of every later worker whose range starts inside the tile.
template <int BN>
struct SkSrc {
  const float* ws;
  int w0, w1;
  size_t slot0;  // slot of w0's segment
  int row;
  bool live;
  __device__ __forceinline__ void get(int col, float (&v)[16]) const {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    if (!live) return;
    constexpr size_t stride = (size_t)256 * BN;
    for (int w = w0; w <= w1; ++w) {
      const float* b = ws + (w == w0 ? slot0 : sk_slot(w, 0)) * stride;
      float4 f[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) f[q] = __ldcg(reinterpret_cast<const float4*>(b + ws_index(col >> 4, q, row, 256)));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[4 * q] += f[q].x;
        v[4 * q + 1] += f[q].y;
        v[4 * q + 2] += f[q].z;
        v[4 * q + 3] += f[q].w;
      }
    }
  }
  __device__ __forceinline__ void sync() const {}
};

// block = (tile, 128-row half, part of the column groups); tiles that one
// worker finished return at once
template <int KIND, int BN>
__global__ void __launch_bounds__(128)
tc2_streamk_epilogue_kernel(const GemmParams p, int n_parts) {
  constexpr int G = epi_groups<KIND, BN>();
  grid_launch_dependents();
  grid_dependency_wait();  // the GEMM's partials
  int bid = blockIdx.x;
  const int part = bid % n_parts;
  bid /= n_parts;
  const int t = bid % 2;
  const int tile = bid / 2;
  const int kb = p.K / 64;
  const long long g0 = (long long)tile * kb;
  const int w0 = sk_worker(p.sk_total, p.skw, g0);
  const int w1 = sk_worker(p.sk_total, p.skw, g0 + kb - 1);
  if (w0 == w1) return;
  const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
  if (m_blk * 256 + t * 128 >= p.M) return;
  const int lr = t * 128 + threadIdx.x;
  const int r = m_blk * 256 + lr;
  const size_t slot0 = sk_slot(w0, sk_lo(p.sk_total, p.skw, w0) >= g0 ? 0 : 1);
  SkSrc<BN> src{p.ws, w0, w1, slot0, lr, r < p.M};
  const int ga = (part * G) / n_parts, gb = ((part + 1) * G) / n_parts;
  epilogue_rows<KIND, BN>(p, n_blk, r, r < p.M, src, ga, gb);
}

// Launch one 2-SM GEMM (M > 128); weight maps with 128-row boxes.
template <int KIND, int BN>
inline cudaError_t tc2_launch(const TcPlan& pl, const void* A, const CUtensorMap& b0, const CUtensorMap& b1,
                              const CUtensorMap& b2, GemmParams p, cudaStream_t st, uint64_t* launches) {
  CUtensorMap a;
  if (!encode_2d(pl, &a, A, (uint64_t)p.M, (uint64_t)p.K, 128)) return cudaErrorInvalidValue;
  p.num_m = (p.M + 255) / 256;
  int num_n;
  if (KIND == kEpiQKV) num_n = 3 * p.d / BN;
  else if (KIND == kEpiSwiGLU) num_n = p.ffn / (BN / 2);
  else num_n = p.d / BN;
  p.num_n = num_n;
  p.num_tiles = p.num_m * num_n;
  const int pairs = pl.num_sms / 2;
  const int kb = p.K / 64;
  p.splits = 1;
  p.num_units = p.num_tiles;
  p.ws = pl.ws;
  p.sk_total = (long long)p.num_tiles * kb;
  // whole tiles unless the pairs their last round leaves idle lose more time
  // than the cut-tile epilogue kernel costs: measured on the 768-row layers,
  // a 256 x BN x 64 k-block step about 0.39 us per pair (BN 256), the cut-tile
  // kernel about 12 us; so the down projection (48 tiles of 192 k-blocks for
  // 74 pairs) goes stream-K and the O projection (64 k-blocks) stays whole
  const int rounds = (p.num_tiles + pairs - 1) / pairs;
  const double idle_kb = (rounds - (double)p.num_tiles / pairs) * kb * (BN / 256.0);
  const bool balanced = idle_kb * 0.39 <= 12.0;
  if (balanced || !pl.ws) {
    // whole tiles: contiguous ranges of tiles, one range per pair
    p.sk_whole = 1;
    p.skw = p.num_tiles < pairs ? p.num_tiles : pairs;
  } else {
    // stream-K over all pairs, at least 4 k-blocks per pair (no empty range)
    p.sk_whole = 0;
    long long w = p.sk_total / 4;
    if (w > pairs) w = pairs;
    if (w < 1) w = 1;
    p.skw = (int)w;
    if ((size_t)2 * p.skw * 256 * BN > pl.ws_floats) p.skw = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.skw, 1, 1);
  cfg.blockDim = dim3(kTc2Threads, 1, 1);
  cfg.dynamicSmemBytes = Tc2Cfg<BN>::kSmem;
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, tc_gemm2_kernel<KIND, BN>, a, b0, b1, b2, p);
  (*launches)++;
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  // every tile is whole within one range in whole-tile mode, or when the
  // workers divide the tiles
  if (e != cudaSuccess || p.sk_whole || p.num_tiles % p.skw == 0) return e;
  // one block per (tile half, column group) up to 16 blocks per SM: every
  // block is one round trip of partial loads, so more blocks keep more of
  // them in flight
  constexpr int G = epi_groups<KIND, BN>();
  int n_parts = (16 * pl.num_sms + p.num_tiles * 2 - 1) / (p.num_tiles * 2);
  if (n_parts > G) n_parts = G;
  if (n_parts < 1) n_parts = 1;
  cudaLaunchConfig_t c2 = {};
  c2.gridDim = dim3(p.num_tiles * 2 * n_parts, 1, 1);
  c2.blockDim = dim3(128, 1, 1);
  c2.stream = st;
  cudaLaunchAttribute a2[1];
  a2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a2[0].val.programmaticStreamSerializationAllowed = 1;
  c2.attrs = a2;
  c2.numAttrs = 1;
  e = cudaLaunchKernelEx(&c2, tc2_streamk_epilogue_kernel<KIND, BN>, p, n_parts);
  (*launches)++;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace esd
