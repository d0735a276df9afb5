// Split-K GEMM for few selected rows (M <= 192) with the reduction inside a
// thread-block cluster: the S CTAs of a cluster share one output tile
// [TM rows x BN columns] and each accumulates k-blocks [s*K/S, (s+1)*K/S) in its
// own TMEM. The tile's epilogue column groups are dealt out to the S CTAs
// (CTA o owns groups [o*G/S, (o+1)*G/S) of the G groups); each
// CTA sends the columns it does not own, as fp32 partials, into the shared
// memory of their owner (distributed shared memory), and the owner adds them
// to its own partial in a fixed order and runs the fused epilogue (the same
// epilogue code as the unsplit kernel). No partial reaches global memory and
// no second kernel runs. The receive buffer reuses the TMA ring, which every
// CTA declares free (all of its MMAs complete) to its peers before they write.
//
// Used for the gathered-row GEMMs of the sparse layers, whose weight matrix is
// streamed once per step ("ES-dLLM", method section: the skipped tokens bypass
// the later layers, so only the selected rows are projected). No TMA load is
// multicast. Every wait is bounded; every CTA reaches the final cluster
// barrier, so no CTA exits while a peer may still write into its memory.
#pragma once

#include "tc_gemm2.cuh"

namespace esd {

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  int* flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  raise_flag(flag, kFlagTimeout);
  return false;
}
__device__ __forceinline__ void st_cluster_f4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// The 16-column chunks of an epilogue group (epi_groups): QKV group = 16 dims
// of a head's first half and their rotation partners 64 further; SwiGLU group
// = 16 gate and the matching 16 up columns; residual group = 16 columns.
template <int KIND, int BN>
struct GroupCols {
  static constexpr int kChunks = (KIND == kEpiQKV || KIND == kEpiSwiGLU) ? 2 : 1;
  __device__ static int col(int gg, int w) {
    if (KIND == kEpiQKV) return (gg >> 2) * 128 + w * 64 + (gg & 3) * 16;
    if (KIND == kEpiSwiGLU) return w * (BN / 2) + gg * 16;
    return gg * 16;
  }
  __device__ static void locate(int c, int& gg, int& w) {
    if (KIND == kEpiQKV) {
      const int within = c & 127;
      w = within >> 6;
      gg = (c >> 7) * 4 + ((within & 63) >> 4);
    } else if (KIND == kEpiSwiGLU) {
      w = c >= BN / 2 ? 1 : 0;
      gg = (c - w * (BN / 2)) >> 4;
    } else {
      w = 0;
      gg = c >> 4;
    }
  }
};

// Receive buffer: for sender slot s (the S-1 peers in rank order), owned chunk
// j and 4-column quarter q, a plane of TM rows of float4 (a warp's 32 rows are
// 512 contiguous bytes: no bank conflicts on either side).
__host__ __device__ constexpr int cl_recv_index(int s, int j, int q, int row, int nchunks, int tm) {
  return ((s * nchunks + j) * 4 + q) * tm + row;
}

// Accumulator of an owned column: this CTA's TMEM partial plus the peers'.
template <int KIND, int BN>
struct ClusterSrc {
  uint32_t tbase;
  const float4* recv;
  int slots, nchunks, g0, row, tm;
  __device__ __forceinline__ void get(int c, float (&v)[16]) const {
    tmem_ld16(tbase + c, v);
    tmem_ld_wait();
    if (row < 0) return;
    int gg, w;
    GroupCols<KIND, BN>::locate(c, gg, w);
    const int j = (gg - g0) * GroupCols<KIND, BN>::kChunks + w;
    for (int s = 0; s < slots; ++s) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 f = recv[cl_recv_index(s, j, q, row, nchunks, tm)];
        v[4 * q] += f.x;
        v[4 * q + 1] += f.y;
        v[4 * q + 2] += f.z;
        v[4 * q + 3] += f.w;
      }
    }
  }
  __device__ __forceinline__ void sync() const {}
};

// Epilogue column groups [g0, g1) owned by cluster rank o of S.
__device__ __forceinline__ int cl_g0(int o, int S, int G) { return (o * G) / S; }

// grid.x = tiles * S, cluster (S, 1, 1); rank in the cluster = split index.
// Warps: 0 TMA, 1 TMEM + MMA, 2..9 epilogue (two warps per TMEM lane quarter,
// each with half of this CTA's columns).
constexpr int kClThreads = 320;

template <int KIND, int TM, int BN>
__global__ void __launch_bounds__(kClThreads, 1)
tc_gemm_cl_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                  const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                  const GemmParams p) {
  using C = TcCfg<TM, BN>;
  using GC = GroupCols<KIND, BN>;
  constexpr int MT = C::MT;
  constexpr int G = epi_groups<KIND, BN>();
  constexpr int kCols = MT * BN <= 256 ? 256 : 512;
  constexpr bool kResidual = KIND == kEpiResidualO || KIND == kEpiResidualD;
  constexpr int kPre = 4;  // residual rows prefetched when a CTA owns at most this many chunks
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tfull = bars + 2 * C::kStages;
  uint64_t* drain = tfull + 1;
  uint64_t* peer_ready = tfull + 2;  // every peer's ring is free (S-1 remote arrivals)
  uint64_t* parts_in = tfull + 3;    // every peer's partials are here (8 warps x (S-1))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int S = p.splits;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();
  const int tile = blockIdx.x / S;
  const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
  const int kb_total = p.K / C::kBK;
  const int kb0 = (int)(((long long)rank * kb_total) / S);
  const int nkb = (int)(((long long)(rank + 1) * kb_total) / S) - kb0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    mbar_init(smem_u32(tfull), 1);
    mbar_init(smem_u32(drain), 1);
    mbar_init(smem_u32(peer_ready), S > 1 ? S - 1 : 1);
    mbar_init(smem_u32(parts_in), S > 1 ? 8 * (S - 1) : 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // peers arrive on this CTA's barriers from here on
  // the prologue above may overlap the previous kernel; the producer streams
  // the first weight stages before waiting for it, every other global access
  // of this kernel follows a grid-dependency wait
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: k-blocks [kb0, kb0 + nkb) of the tile
      const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
      int sel, row0, row1;
      b_rows<KIND, BN>(n_blk, p, sel, row0, row1);
      const CUtensorMap* mb0 = sel == 0 ? &tmB0 : (sel == 1 ? &tmB1 : &tmB2);
      const CUtensorMap* mb1 = (KIND == kEpiSwiGLU) ? &tmB1 : mb0;
      // the weights of the first stages do not depend on the previous
      // kernel: stream them while it finishes, then its activations
      const int npre = nkb < C::kStages ? nkb : C::kStages;
      for (int i = 0; i < npre; ++i) {
        const uint32_t fb = smem_u32(&full[i]);
        mbar_expect_tx(fb, C::kTxBytes);
        uint8_t* bb = smem + i * C::kStageBytes + C::kABytes;
        const int k0 = (kb0 + i) * C::kBK;
        tma_load_2d(smem_u32(bb), mb0, fb, k0, row0, pol_w);
        tma_load_2d(smem_u32(bb + C::kBBytes / 2), mb1, fb, k0, row1, pol_w);
      }
      grid_dependency_wait();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const uint32_t fb = smem_u32(&full[stage]);
        uint8_t* sbase = smem + stage * C::kStageBytes;
        const int k0 = (kb0 + i) * C::kBK;
        if (i >= npre) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.flag)) break;
          mbar_expect_tx(fb, C::kTxBytes);
          uint8_t* bb = sbase + C::kABytes;
          tma_load_2d(smem_u32(bb), mb0, fb, k0, row0, pol_w);
          tma_load_2d(smem_u32(bb + C::kBBytes / 2), mb1, fb, k0, row1, pol_w);
        }
        tma_load_2d(smem_u32(sbase), &tmA, fb, k0, m_blk * C::kTileRows, pol_a);
        ++issued;
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
      }
      // drain: the last load of every stage used has landed
      for (int i = issued - C::kStages; i < issued; ++i) {
        if (i < 0) continue;
        const int st = i % C::kStages;
        const uint32_t ph = (uint32_t)((i / C::kStages) & 1);
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(&full[st]), ph)) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc0 = idesc_bf16(128, BN);
      constexpr uint32_t idesc1 = idesc_bf16(C::sub_rows(1), BN);
      int stage = 0;
      uint32_t phase = 0;
      bool issued = false, ok = true;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.flag)) { ok = false; break; }
        const uint32_t sbase = smem_u32(smem + stage * C::kStageBytes);
        const uint32_t bbase = sbase + C::kABytes;
#pragma unroll
        for (int kk = 0; kk < C::kBK / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(bbase + kk * 32);
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const uint64_t adesc = smem_desc_sw128(sbase + t * 128 * 128 + kk * 32);
            tc_mma(tmem + (uint32_t)(t * BN), adesc, bdesc, t == 0 ? idesc0 : idesc1, (i | kk) != 0 ? 1u : 0u);
          }
        }
        issued = true;
        tc_commit(smem_u32(&empty[stage]));
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
      }
      if (ok && issued) tc_commit(smem_u32(tfull));
      if (issued) {
        tc_commit(smem_u32(drain));
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(drain), 0u)) break;
      }
    }
  } else {
    // ---------------- epilogue warps 2..9
    grid_dependency_wait();
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t tacc = tmem + ((uint32_t)(quarter * 32) << 16);
    const int g0 = cl_g0(rank, S, G), g1 = cl_g0(rank + 1, S, G);
    const int nch = (g1 - g0) * GC::kChunks;
    // this warp's half of the owned groups
    const int hg0 = g0 + ((g1 - g0) * half) / 2, hg1 = g0 + ((g1 - g0) * (half + 1)) / 2;
    // residual rows of the owned columns, fetched while the MMAs run
    uint4 xv[MT][kPre][2];
    const bool pre = kResidual && hg1 - hg0 <= kPre;
    if (kResidual && pre) {
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int lr = C::row_of(t, quarter, lane);
        const int r = m_blk * C::kTileRows + lr;
        const bool live = lr >= 0 && r < p.M;
        const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(p.e.out) + (size_t)(live ? r : 0) * p.d +
                                 n_blk * BN;
#pragma unroll
        for (int j = 0; j < kPre; ++j) {
          if (live && j < hg1 - hg0) {
            const uint4* src = reinterpret_cast<const uint4*>(x + GC::col(hg0 + j, 0));
            xv[t][j][0] = src[0];
            xv[t][j][1] = src[1];
          }
        }
      }
    }
    bool ok = warp_wait(smem_u32(tfull), 0u, abort_flag, p.flag);
    tc_fence_after();
    const float4* recv = reinterpret_cast<const float4*>(smem);
    if (S > 1) {
      const uint32_t recv_u32 = smem_u32(smem);
      // 1. this CTA's ring is free: tell every peer
      if (warp == 2 && lane == 0)
        for (int o = 0; o < S; ++o)
          if (o != rank) mbar_arrive_cluster(mapa_shared(smem_u32(peer_ready), (uint32_t)o));
      // 2. every peer's ring is free
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(peer_ready), 0u, abort_flag, p.flag)) && ok;
      // 3. the columns of every peer's groups, into that peer's receive buffer
      //    (peers in rotated order, so that the CTAs do not all write to the
      //    same peer at once; two chunks per TMEM wait; this warp's half)
      for (int i = 1; i < S; ++i) {
        const int o = (rank + i) % S;
        const int og0 = cl_g0(o, S, G);
        const int onch = (cl_g0(o + 1, S, G) - og0) * GC::kChunks;
        const int slot = rank < o ? rank : rank - 1;
        const uint32_t dst = mapa_shared(recv_u32, (uint32_t)o);
        if (ok) {
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const int lr = C::row_of(t, quarter, lane);
            const int j_end = (onch * (half + 1)) / 2;
            for (int j = (onch * half) / 2; j < j_end; j += 2) {
              const int nh = j_end - j < 2 ? 1 : 2;
              float v[2][16];
#pragma unroll
              for (int h = 0; h < 2; ++h)
                if (h < nh) {
                  const int jj = j + h;
                  tmem_ld16(tacc + (uint32_t)(t * BN + GC::col(og0 + jj / GC::kChunks, jj % GC::kChunks)), v[h]);
                }
              tmem_ld_wait();
              if (lr >= 0) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
                  if (h < nh) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                      st_cluster_f4(dst + 16u * (uint32_t)cl_recv_index(slot, j + h, q, lr, onch, TM),
                                    v[h][4 * q], v[h][4 * q + 1], v[h][4 * q + 2], v[h][4 * q + 3]);
                  }
              }
            }
          }
        }
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(parts_in), (uint32_t)o));
      }
      // 4. every peer's partials of this CTA's groups have arrived
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(parts_in), 0u, abort_flag, p.flag)) && ok;
    }
    // 5. the fused epilogue of the owned groups
    if (ok) {
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int lr = C::row_of(t, quarter, lane);
        const int r = m_blk * C::kTileRows + lr;
        const bool live = lr >= 0 && r < p.M;
        ClusterSrc<KIND, BN> src{tacc + (uint32_t)(t * BN), recv, S - 1, nch, g0, lr, TM};
        if (kResidual && pre) {
          __nv_bfloat16* x = reinterpret_cast<__nv_bfloat16*>(p.e.out) + (size_t)(live ? r : 0) * p.d + n_blk * BN;
#pragma unroll
          for (int j = 0; j < kPre; ++j) {
            if (j >= hg1 - hg0) continue;
            const int c = GC::col(hg0 + j, 0);
            float v[16];
            src.get(c, v);
            if (!live) continue;
            const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(xv[t][j]);
            float o[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 f = __bfloat1622float2(hx[i]);
              o[2 * i] = f.x + v[2 * i];
              o[2 * i + 1] = f.y + v[2 * i + 1];
            }
            store16_bf16(x + c, o);
          }
        } else {
          epilogue_rows<KIND, BN>(p, n_blk, r, live, src, hg0, hg1);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kCols);
  cluster_sync_all();  // no CTA leaves while a peer may still write into its memory
}

// Shared memory the receive buffer needs, in bytes: S-1 slots sized for the
// largest owner.
template <int KIND, int TM, int BN>
constexpr size_t cl_recv_bytes(int S) {
  return (size_t)(S - 1) * ((epi_groups<KIND, BN>() + S - 1) / S) * GroupCols<KIND, BN>::kChunks * 4 * TM * 16;
}

template <int KIND, int TM, int BN>
inline void tc_cl_set_attr() {
  cudaFuncSetAttribute(tc_gemm_cl_kernel<KIND, TM, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       TcCfg<TM, BN>::kSmem);
}

// Clusters of S CTAs of this kernel that can be resident at once (0 if none).
template <int KIND, int TM, int BN>
inline int tc_cl_max_clusters(int S) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S * 64, 1, 1);
  cfg.blockDim = dim3(kClThreads, 1, 1);
  cfg.dynamicSmemBytes = TcCfg<TM, BN>::kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_cl_kernel<KIND, TM, BN>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int KIND, int TM, int BN>
inline cudaError_t tc_cl_launch(const TcPlan& pl, const void* A, const CUtensorMap& b0, const CUtensorMap& b1,
                                const CUtensorMap& b2, GemmParams p, int S, cudaStream_t st,
                                uint64_t* launches) {
  CUtensorMap a;
  if (!encode_2d(pl, &a, A, (uint64_t)p.M, (uint64_t)p.K, TM)) return cudaErrorInvalidValue;
  p.num_m = 1;
  int num_n;
  if (KIND == kEpiQKV) num_n = 3 * p.d / BN;
  else if (KIND == kEpiSwiGLU) num_n = p.ffn / (BN / 2);
  else num_n = p.d / BN;
  p.num_n = num_n;
  p.num_tiles = num_n;
  p.splits = S;
  p.num_units = p.num_tiles * S;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_units, 1, 1);
  cfg.blockDim = dim3(kClThreads, 1, 1);
  cfg.dynamicSmemBytes = TcCfg<TM, BN>::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the previous kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tc_gemm_cl_kernel<KIND, TM, BN>, a, b0, b1, b2, p);
  (*launches)++;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ choice
// Rough device times (microseconds) of one CTA: fixed start (barriers, TMEM,
// first loads), one 64-deep k-block of MMAs for the tile shape (measured
// tcgen05 rates: 128x256x16 in ~150 cycles, 64x256x16 in ~117, 128x128x16 in
// ~100; the 192-row tiles measured ~0.6 and ~0.45 us per k-block), and the
// partial exchange.
constexpr double kClStartUs = 3.0;
constexpr double kClExchangeBytesPerUs = 22e3;
inline double cl_kblock_us(int TM, int BN) {
  if (TM == 128) return BN == 256 ? 0.32 : 0.21;
  return BN == 256 ? 0.62 : 0.46;
}

constexpr int cl_kind_index(int KIND) {
  return KIND == kEpiQKV ? 0 : (KIND == kEpiResidualO ? 1 : (KIND == kEpiSwiGLU ? 2 : 3));
}

struct ClChoice {
  int bn = 0, S = 0;
  double us = 1e30;
};

template <int KIND, int TM, int BN>
inline void cl_consider(const TcPlan& pl, int M, int tiles, int kb_total, ClChoice* best) {
  constexpr int G = epi_groups<KIND, BN>();
  const size_t ring = (size_t)TcCfg<TM, BN>::kStages * TcCfg<TM, BN>::kStageBytes;
  const int* mc = pl.cl_max[cl_kind_index(KIND)][TM == 128 ? 0 : 1][BN == 128 ? 0 : 1];
  for (int S = 1; S <= 8 && S <= G; ++S) {
    if (kb_total / S < 2 || cl_recv_bytes<KIND, TM, BN>(S) > ring || mc[S] < 1) continue;
    const int waves = (tiles + mc[S] - 1) / mc[S];
    const int chunks = ((G + S - 1) / S) * GroupCols<KIND, BN>::kChunks;
    const double exch = (double)(S - 1) / S * TM * BN * 4 / kClExchangeBytesPerUs;
    const double epi = 0.3 * chunks * TcCfg<TM, BN>::MT;
    const double us =
        waves * (kClStartUs + ((kb_total + S - 1) / S) * cl_kblock_us(TM, BN) + exch + epi);
    if (us < best->us - 1e-9) {
      best->us = us;
      best->bn = BN;
      best->S = S;
    }
  }
  (void)M;
}

// Resident-cluster counts for every (kind, tile rows, tile width, S); after
// the kernels' shared-memory attributes are set.
inline void tc_cl_init(TcPlan& pl) {
#define ESD_CL_INIT1(KIND, TM, BN)                                                    \
  do {                                                                                \
    tc_cl_set_attr<KIND, TM, BN>();                                                   \
    for (int S = 1; S <= 8; ++S)                                                      \
      pl.cl_max[cl_kind_index(KIND)][TM == 128 ? 0 : 1][BN == 128 ? 0 : 1][S] =       \
          tc_cl_max_clusters<KIND, TM, BN>(S);                                        \
  } while (0)
#define ESD_CL_INIT(KIND)            \
  ESD_CL_INIT1(KIND, 128, 128);      \
  ESD_CL_INIT1(KIND, 128, 256);      \
  ESD_CL_INIT1(KIND, 192, 128);      \
  ESD_CL_INIT1(KIND, 192, 256)
  ESD_CL_INIT(kEpiQKV);
  ESD_CL_INIT(kEpiResidualO);
  ESD_CL_INIT(kEpiSwiGLU);
  ESD_CL_INIT(kEpiResidualD);
#undef ESD_CL_INIT
#undef ESD_CL_INIT1
}

// The cluster path for M <= 192 rows: the (tile width, S) with the lowest
// estimated time. The SwiGLU GEMM takes it only when that estimate beats the
// SM-pair kernel's (whole 256 x 256 tiles, ~0.32 us per k-block per pair).
// *done false leaves the GEMM to the other paths.
template <int KIND>
inline cudaError_t tc_cl_dispatch(const TcPlan& pl, int layer, const void* A, const GemmParams& p,
                                  cudaStream_t st, uint64_t* launches, bool* done) {
  *done = false;
  if (p.d % 256 != 0 || p.M > 192) return cudaSuccess;
  const int kb = p.K / 64;
  const int n_out = KIND == kEpiQKV ? 3 * p.d : (KIND == kEpiSwiGLU ? 2 * p.ffn : p.d);
  if (n_out % 256 != 0) return cudaSuccess;
  ClChoice best;
  if (p.M <= 128) {
    cl_consider<KIND, 128, 128>(pl, p.M, n_out / 128, kb, &best);
    cl_consider<KIND, 128, 256>(pl, p.M, n_out / 256, kb, &best);
  } else {
    cl_consider<KIND, 192, 128>(pl, p.M, n_out / 128, kb, &best);
    cl_consider<KIND, 192, 256>(pl, p.M, n_out / 256, kb, &best);
  }
  if (best.S < 1) return cudaSuccess;
  if (KIND == kEpiSwiGLU) {
    const int pairs = pl.num_sms / 2, tiles2 = n_out / 256;
    const double pair_us = ((tiles2 + pairs - 1) / pairs) * (kClStartUs + kb * 0.32);
    if (best.us >= pair_us) return cudaSuccess;
  }
  const bool wide = best.bn == 256;
  const CUtensorMap *b0, *b1, *b2;
  if (KIND == kEpiQKV) {
    b0 = wide ? &pl.q128[layer] : &pl.q64[layer];
    b1 = wide ? &pl.k128[layer] : &pl.k64[layer];
    b2 = wide ? &pl.v128[layer] : &pl.v64[layer];
  } else if (KIND == kEpiResidualO) {
    b0 = b1 = b2 = wide ? &pl.o128[layer] : &pl.o64[layer];
  } else if (KIND == kEpiSwiGLU) {
    b0 = wide ? &pl.g128[layer] : &pl.g64[layer];
    b1 = b2 = wide ? &pl.u128[layer] : &pl.u64[layer];
  } else {
    b0 = b1 = b2 = wide ? &pl.d128[layer] : &pl.d64[layer];
  }
  *done = true;
  if (p.M <= 128)
    return wide ? tc_cl_launch<KIND, 128, 256>(pl, A, *b0, *b1, *b2, p, best.S, st, launches)
                : tc_cl_launch<KIND, 128, 128>(pl, A, *b0, *b1, *b2, p, best.S, st, launches);
  return wide ? tc_cl_launch<KIND, 192, 256>(pl, A, *b0, *b1, *b2, p, best.S, st, launches)
              : tc_cl_launch<KIND, 192, 128>(pl, A, *b0, *b1, *b2, p, best.S, st, launches);
}

}  // namespace esd
