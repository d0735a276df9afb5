// Partial and dense attention on SM pairs (tcgen05 cta_group::2), bf16,
// head_dim 128: softmax(q K^T / sqrt(128)) V for the query rows of each
// sequence over all of its keys ("DyLLM", technical summary section 2.B.2:
// the salient rows of the attention matrix are recomputed exactly; with every
// row selected this is the dense bidirectional attention).
//
// A pair-tile is 256 query rows of one head of one sequence: CTA r of the pair
// holds query rows [128 r, 128 r + 128) (the MMA's M halves), and the keys are
// cut into chunks of 128. For a chunk, S = Q K^T (M 256, N 128 keys, K 128
// dims) takes K from both CTAs (CTA r loads keys [64 r, 64 r + 64) of the
// chunk), and O += P V (M 256, N 128 dims, K 128 keys) takes V from both
// (CTA r loads dims [64 r, 64 r + 64) of the chunk's 128 keys). So a pair reads
// every K/V byte of its chunks once, and each SM half of them.
//
// The chunks of a pair-tile are split over S pairs of one cluster (2 S CTAs,
// S <= 4) when the pair-tiles alone leave SMs idle; each pair walks its
// chunks, and the S partial results (row maximum, row sum and unnormalised O
// per query row) are merged through distributed shared memory: the CTA of
// split p owns rows [128 p / S, 128 (p + 1) / S) of the pair's half, every CTA
// stores its partial rows into the owners' shared memory, and each owner
// combines the S partials of its rows in split order and stores them. No CTA
// waits on a CTA outside its cluster.
//
// Warps (both CTAs): 0 TMA producer (Q once, K/V chunks through a three-stage
// ring, each load counted on the leader's barrier); 1 TMEM allocator and, in
// the leader CTA, the single MMA-issuing thread (S of a chunk as soon as its
// K/V has landed and an S buffer is free, P_j V_j as soon as P_j is written);
// in the peer CTA warp 1 relays the P-written signal to the leader; 2..9
// softmax, thread = one query row and one half of the chunk's keys (warps
// 2..5 keys 0-63, 6..9 keys 64-127 of every chunk): tcgen05.ld of its half of
// the row of S (three TMEM S buffers, so S of the next chunks is computed
// while chunk j's softmax runs), the row maximum from both halves through shared
// memory, base-2 softmax against a running maximum that only moves when a
// chunk's maximum exceeds it by more than 2^8 (then each half rescales its
// half of the O row in TMEM after the previous P V has landed), P rounded to
// bf16 into one of two shared P buffers (128-byte swizzle, the A operand of
// P V; P V of chunk j runs under chunk j + 1's exponentials). The result
// O / l is exact either way; only how often O is rescaled changes.
// Keys at or beyond the sequence's L are masked; query rows beyond its R rows
// are computed and not stored. Every mbarrier wait is bounded (error flag);
// every CTA reaches every cluster barrier.
#pragma once

#include "tc_gemm2.cuh"
#include "tc_gemm_cl.cuh"  // mbar_wait_cluster

namespace esd {

constexpr int kApQ = 256;                                  // query rows per pair
constexpr int kApK = 128;                                  // keys per chunk
constexpr int kApHd = 128;                                 // head dim
constexpr int kApStages = 3;                               // K/V ring
constexpr int kApMaxSplits = 4;                            // pairs per cluster
// softmax column groups (keys of a chunk): four groups (16 softmax warps, 32
// keys per thread) measured no faster than two (768 queries: 33.7 against
// 32.9 us; 192 queries: 16.9 against 16.6 us)
constexpr int kApGroups = 2;
constexpr int kApGK = kApK / kApGroups;                    // keys per group and chunk
constexpr int kApSoft = 128 * kApGroups;                   // softmax threads
constexpr int kApThreads = 64 + kApSoft;
constexpr int kApQBox = 128 * 64 * 2;                      // 128 query rows x 64 dims
constexpr int kApQBytes = 2 * kApQBox;                     // this CTA's Q rows, dims 0-63 | 64-127
constexpr int kApKBox = 64 * 64 * 2;                       // 64 keys x 64 dims
constexpr int kApVBox = 128 * 64 * 2;                      // 128 keys x this CTA's 64 dims
constexpr int kApStageBytes = 2 * kApKBox + kApVBox;       // K half (2 boxes) + V half
constexpr int kApPBox = 128 * 64 * 2;                      // 128 rows x 64 keys
constexpr int kApPBytes = 2 * kApPBox;                     // one chunk's P
constexpr int kApMergeStride = 132;                        // floats per staged output row
constexpr int kApMain = kApQBytes + kApStages * kApStageBytes + 2 * kApPBytes;
constexpr int kApStats = 3 * kApGroups * 128 * 4;          // row maxima and sums, merge statistics
static_assert(2 * kApGroups * 128 >= 2 * kApMaxSplits * 64, "merge statistics reuse the row maxima");
constexpr int kApSmem = kApMain + kApStats + 256 + 1024;   // + barriers, alignment slack
static_assert(kApMaxSplits * 64 * kApMergeStride * 4 <= kApStages * kApStageBytes + 2 * kApPBytes,
              "the merge slots reuse the K/V ring and the P buffers");

constexpr float kApLazy = 8.0f;  // log2 of the largest unnormalised P before the running maximum moves

// Shared-memory descriptor of an MN-major operand, 128-byte swizzle: rows of 64
// MN-elements (128 B), groups of 8 rows along K 1024 B apart (stride byte
// offset), the next 64 MN-elements `lbo` bytes further (leading byte offset).
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// kind::f16 instruction descriptor: D fp32, A and B bf16, A K-major, B K-major
// (b_mn 0) or MN-major (b_mn 1, bit 16)
__host__ __device__ constexpr uint32_t idesc_bf16_b(int M, int N, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16_tc(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void tc_commit_pair_mask(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
// 2^x with one MUFU operation, subnormal results flushed to zero (x <= 8 here;
// x = -inf gives 0)
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void st_dsmem_f4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_dsmem_f2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1,%2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 2, %0;" ::"n"(kApSoft) : "memory"); }
// the AND of `pred` over the softmax threads (named barrier 2)
__device__ __forceinline__ bool softmax_all(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 2, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(kApSoft)
      : "memory");
  return r != 0;
}

// Q [B*R, H*128] (the rows of the sequences back to back), K and V
// [B*L, H*128], O [B*R, H*128]. Grid (2 * splits, ceil(R / 256), H * B),
// cluster (2 * splits, 1, 1); split p covers chunks [p * cps, (p + 1) * cps)
// of the ceil(L / 128) chunks, every split at least one. K and V rows
// [0, B*L) finite.
__global__ void __launch_bounds__(kApThreads, 1)
attention_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O, int R, int L,
                      int H, int splits, int cps, float scale_log2, int* flag,
                      const int32_t* __restrict__ prow, float2* __restrict__ pstat,
                      const int32_t* __restrict__ rows_valid, int pld) {
  extern __shared__ __align__(1024) uint8_t smem_ap_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_ap_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + kApQBytes;                      // [stage][K0 K1 V]
  uint8_t* sP = sKV + kApStages * kApStageBytes;      // [buffer][keys 0-63 | 64-127]
  float* pm = reinterpret_cast<float*>(sP + 2 * kApPBytes);  // [S buffer][group][128] partial row maxima;
                                                             // merge: [split][64] (m, l)
  float* lsum = pm + 2 * kApGroups * 128;                     // [group][128] partial row sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(lsum + kApGroups * 128);
  uint64_t* qfull = bars;        // leader: Q of both CTAs landed
  uint64_t* kvfull = bars + 1;   // [3] leader: the chunk's K/V of both CTAs landed
  uint64_t* kvempty = bars + 4;  // [3] both: the chunk's S and P V are done with the stage
  uint64_t* sfull = bars + 7;    // [3] both: S of chunk j in S buffer j % 3
  uint64_t* pready = bars + 10;  // [2] both: P_j written (so S_j read, O rescaled) by this CTA's 8 warps
  uint64_t* pfull = bars + 12;   // [2] leader: the peer's P_j ready (its relay's arrive)
  uint64_t* ofull = bars + 14;   // [2] both: P_j V_j accumulated (P buffer j % 2 free)
  uint64_t* drain = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* mbuf = reinterpret_cast<float*>(sKV);  // [split][64][kApMergeStride] merge slots, after the last MMA

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const int pr = (int)(crank >> 1), r = (int)(crank & 1);
  const uint32_t lead = crank & ~1u;
  const uint16_t mask = (uint16_t)(3u << lead);
  const int t = blockIdx.y, b = blockIdx.z / H, h = blockIdx.z % H;
  const int nch = (L + kApK - 1) / kApK;
  const int c0 = pr * cps;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmQ) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmK) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmV) : "memory");
    mbar_init(smem_u32(qfull), 1);
    for (int i = 0; i < kApStages; ++i) {
      mbar_init(smem_u32(&kvfull[i]), 1);
      mbar_init(smem_u32(&kvempty[i]), 1);
    }
    for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&sfull[i]), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&pready[i]), kApSoft / 32);
      mbar_init(smem_u32(&pfull[i]), 1);
      mbar_init(smem_u32(&ofull[i]), 1);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer signals the leader's barriers from here on
  tc_fence_after();
  grid_launch_dependents();
  grid_dependency_wait();  // Q/K/V come from the previous kernel; O may still be read by an earlier one
  const uint32_t tmem = *tmem_slot;
  // query rows of this sequence that count (rows_valid, optional): a pair-tile
  // past them does no work (uniform over the cluster)
  const int nvalid = rows_valid ? min(R, max(0, rows_valid[b])) : R;
  const int n = t * kApQ < nvalid ? max(0, min(nch, c0 + cps) - c0) : 0;  // chunks of this pair

  // per query row of this CTA (softmax threads): the pair's running maximum and row sum
  float m_use = -INFINITY, lrow = 0.0f;
  const int grp = (warp - 2) >> 2;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;

  if (warp == 0) {
    if (lane == 0 && n > 0) {
      // ---------------- TMA producer (both CTAs)
      const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_last();
      const uint32_t qb = mapa_shared(smem_u32(qfull), lead);
      if (r == 0) mbar_expect_tx(smem_u32(qfull), 2u * kApQBytes);
      const int qrow = b * R + t * kApQ + r * 128;
      tma_load_2d_pair(smem_u32(sQ), &tmQ, qb, h * kApHd, qrow, pol_q);
      tma_load_2d_pair(smem_u32(sQ + kApQBox), &tmQ, qb, h * kApHd + 64, qrow, pol_q);
      int last = -1;
      for (int j = 0; j < n; ++j) {
        const int s = j % kApStages;
        if (j >= kApStages &&
            !mbar_wait(smem_u32(&kvempty[s]), (uint32_t)((j / kApStages - 1) & 1), abort_flag, flag))
          break;
        if (r == 0) mbar_expect_tx(smem_u32(&kvfull[s]), 2u * kApStageBytes);
        const uint32_t fb = mapa_shared(smem_u32(&kvfull[s]), lead);
        uint8_t* st = sKV + s * kApStageBytes;
        const int krow = b * L + (c0 + j) * kApK;
        tma_load_2d_pair(smem_u32(st), &tmK, fb, h * kApHd, krow + 64 * r, pol_kv);
        tma_load_2d_pair(smem_u32(st + kApKBox), &tmK, fb, h * kApHd + 64, krow + 64 * r, pol_kv);
        tma_load_2d_pair(smem_u32(st + 2 * kApKBox), &tmV, fb, h * kApHd + 64 * r, krow, pol_kv);
        last = j;
      }
      // drain: every load issued has landed before the CTA moves on (the
      // leader's barriers count both CTAs' bytes; the peer waits until its
      // stages have been consumed)
      if (r == 0)
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(qfull), 0u)) break;
      for (int j = max(0, last - kApStages + 1); j <= last; ++j) {
        const int s = j % kApStages;
        const uint32_t bar = r == 0 ? smem_u32(&kvfull[s]) : smem_u32(&kvempty[s]);
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(bar, (uint32_t)((j / kApStages) & 1))) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && r == 0 && n > 0) {
      // ---------------- MMA issuer (leader CTA). Two streams, each issued as
      // soon as it can go, neither waiting on the other: S_k = Q K_k^T into S
      // buffer k % 3 once chunk k's K/V has landed and P_{k-3} V_{k-3} has
      // been issued (so both CTAs have read S_{k-3}); P_k V_k once both CTAs
      // have written P_k.
      constexpr uint32_t id_s = idesc_bf16_b(256, 128, 0);
      constexpr uint32_t id_o = idesc_bf16_b(256, 128, 1);
      bool issued = false;
      const bool ok = mbar_wait(smem_u32(qfull), 0u, abort_flag, flag);
      int ns = 0, np = 0;
      uint32_t idle = 0;
      while (ok && np < n) {
        bool progress = false;
        if (ns < n && ns < np + 3 &&
            mbar_try_wait(smem_u32(&kvfull[ns % kApStages]), (uint32_t)((ns / kApStages) & 1))) {
          tc_fence_after();
          const uint32_t kb = smem_u32(sKV + (ns % kApStages) * kApStageBytes), qb = smem_u32(sQ);
          const uint32_t ts = tmem + (uint32_t)((ns % 3) * 128);
#pragma unroll
          for (int kk = 0; kk < kApHd / 16; ++kk) {
            const uint32_t qoff = (uint32_t)((kk >> 2) * kApQBox + (kk & 3) * 32);
            const uint32_t koff = (uint32_t)((kk >> 2) * kApKBox + (kk & 3) * 32);
            tc_mma_pair(ts, smem_desc_sw128(qb + qoff), smem_desc_sw128(kb + koff), id_s, kk != 0 ? 1u : 0u);
          }
          tc_commit_pair_mask(smem_u32(&sfull[ns % 3]), mask);
          issued = true;
          ++ns;
          progress = true;
        }
        if (np < ns) {
          const int sb = np & 1;
          const uint32_t par = (uint32_t)((np >> 1) & 1);
          if (mbar_try_wait(smem_u32(&pready[sb]), par) && mbar_try_wait_cluster(smem_u32(&pfull[sb]), par)) {
            tc_fence_after();
            const int s = np % kApStages;
            const uint32_t pb = smem_u32(sP + sb * kApPBytes);
            const uint32_t vb = smem_u32(sKV + s * kApStageBytes + 2 * kApKBox);
#pragma unroll
            for (int kk = 0; kk < kApK / 16; ++kk) {
              const uint32_t aoff = (uint32_t)((kk >> 2) * kApPBox + (kk & 3) * 32);  // P: 64 keys per box
              const uint32_t boff = (uint32_t)(kk * 16 * 128);                        // V: 16 key rows
              tc_mma_pair(tmem + 384u, smem_desc_sw128(pb + aoff), smem_desc_sw128_mn(vb + boff, kApVBox), id_o,
                          (np | kk) != 0 ? 1u : 0u);
            }
            tc_commit_pair_mask(smem_u32(&ofull[sb]), mask);
            tc_commit_pair_mask(smem_u32(&kvempty[s]), mask);
            ++np;
            progress = true;
          }
        }
        if (progress) {
          idle = 0;
        } else if (++idle >= kWaitLimit) {
          *abort_flag = 1;
          raise_flag(flag, kFlagTimeout);
          break;
        } else if ((idle & 255u) == 255u && *abort_flag) {
          break;
        }
      }
      if (issued) {
        tc_commit_pair_own(smem_u32(drain));
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(drain), 0u)) break;
      }
    } else if (lane == 0 && r == 1) {
      // ---------------- relay (the leader's peer): one cluster-scope arrive on
      // the leader's barrier per chunk, once this CTA's eight softmax warps
      // have written P_j (their own arrives stay CTA-local and cheap)
      for (int j = 0; j < n; ++j) {
        const int sb = j & 1;
        if (!mbar_wait(smem_u32(&pready[sb]), (uint32_t)((j >> 1) & 1), abort_flag, flag)) break;
        mbar_arrive_cluster(mapa_shared(smem_u32(&pfull[sb]), lead));
      }
    }
  } else {
    // ---------------- softmax (both CTAs): query row `row`, keys [64 grp, 64 grp + 64) of every chunk
    const uint32_t tS = tmem + lane_off + (uint32_t)(grp * kApGK);
    const uint32_t tO = tmem + lane_off + 384u + (uint32_t)(grp * kApGK);
    float l = 0.0f;  // this half's share of the row sum
    // row statistics out (optional): only for valid rows with a P row in [0, L)
    bool stat_out = false;
    if (pstat) {
      const int q = t * kApQ + r * 128 + row;
      const int pr_row = q < nvalid ? prow[(size_t)b * pld + q] : -1;
      stat_out = pr_row >= 0 && pr_row < L;
    }
    // A wait that gives up (error flag) ends the walk of all eight warps at
    // the same chunk: the decision is taken at the chunk's shared barrier.
    bool ok = true, ok_prev = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      const uint32_t par = (uint32_t)((j >> 1) & 1);
      const bool okw = warp_wait(smem_u32(&sfull[j % 3]), (uint32_t)((j / 3) & 1), abort_flag, flag);
      float sv[kApGK];
      if (okw) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kApGK; c += 16) {
          float v[16];
          tmem_ld16(tS + (uint32_t)((j % 3) * 128 + c), v);
#pragma unroll
          for (int i = 0; i < 16; ++i) sv[c + i] = v[i];
        }
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < kApGK; ++i) sv[i] = 0.0f;
      }
      const int kbase = (c0 + j) * kApK + grp * kApGK;
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (kbase + kApGK > L) {
#pragma unroll
        for (int i = 0; i < kApGK; ++i)
          if (kbase + i >= L) sv[i] = -INFINITY;
      }
#pragma unroll
      for (int i = 0; i < kApGK; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], sv[i]);
      // the row maximum over both halves, in base-2 units (the scale is
      // positive; the chunk's first key is < L, so it is finite)
      pm[(sb * kApGroups + grp) * 128 + row] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2;
      if (!softmax_all(okw && ok_prev)) {
        ok = false;
        break;
      }
      float mx = pm[sb * kApGroups * 128 + row];
#pragma unroll
      for (int g2 = 1; g2 < kApGroups; ++g2) mx = fmaxf(mx, pm[(sb * kApGroups + g2) * 128 + row]);
      bool okr = true;
      if (j == 0) {
        m_use = mx;
      } else {
        const bool need = mx > m_use + kApLazy;
        if (__any_sync(0xffffffffu, need)) {
          // O holds the products of chunks < j: wait for P_{j-1} V_{j-1}
          okr = warp_wait(smem_u32(&ofull[sb ^ 1]), (uint32_t)(((j - 1) >> 1) & 1), abort_flag, flag);
          if (okr) {
            tc_fence_after();
            const float f = need ? exp2f(m_use - mx) : 1.0f;
#pragma unroll 1
            for (int c = 0; c < kApGK; c += 16) {
              float v[16];
              tmem_ld16(tO + (uint32_t)c, v);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] *= f;
              tmem_st16(tO + (uint32_t)c, v);
            }
            tmem_st_wait();
            if (need) {
              l *= f;
              m_use = mx;
            }
          }
        }
      }
      // P_j into buffer sb once P_{j-2} V_{j-2} has read it
      const bool okp = j < 2 || warp_wait(smem_u32(&ofull[sb]), par ^ 1u, abort_flag, flag);
      ok_prev = okr && okp;
      uint8_t* pt = sP + sb * kApPBytes + ((grp * kApGK) / 64) * kApPBox;
      float rs4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int c = 0; c < kApGK / 8; ++c) {  // chunks of 8 keys (16 B)
        float pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pv[i] = ex2_ftz(fmaf(sv[c * 8 + i], scale_log2, -m_use));
          rs4[i & 3] += pv[i];
        }
        uint4 u;
        u.x = pack_bf16_tc(pv[0], pv[1]);
        u.y = pack_bf16_tc(pv[2], pv[3]);
        u.z = pack_bf16_tc(pv[4], pv[5]);
        u.w = pack_bf16_tc(pv[6], pv[7]);
        const int cb = ((grp * kApGK) % 64) / 8 + c;  // 16-byte chunk of the 64-key box row
        *reinterpret_cast<uint4*>(pt + row * 128 + ((cb ^ (row & 7)) << 4)) = u;
      }
      l += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P visible to the tensor cores
      tc_fence_before();                                             // and the O rescale
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&pready[sb]));
    }
    // O is final once the last P V has landed
    bool have = ok && ok_prev && n > 0;
    if (have) have = warp_wait(smem_u32(&ofull[(n - 1) & 1]), (uint32_t)(((n - 1) >> 1) & 1), abort_flag, flag);
    tc_fence_after();
    lsum[grp * 128 + row] = l;
    softmax_bar();
    lrow = 0.0f;
#pragma unroll
    for (int g2 = 0; g2 < kApGroups; ++g2) lrow += lsum[g2 * 128 + row];
    if (stat_out && grp == 0 && splits == 1)
      pstat[((size_t)b * pld + t * kApQ + r * 128 + row) * H + h] = make_float2(m_use, lrow);
    if (!have) m_use = -INFINITY;
    if (splits == 1) {
      // O / l for dims [kApGK grp, kApGK (grp + 1)) of this row
      const int q = t * kApQ + r * 128 + row;
      const float inv = 1.0f / lrow;
      __nv_bfloat16* dst = O + ((size_t)b * R + q) * ((size_t)H * kApHd) + h * kApHd + grp * kApGK;
#pragma unroll
      for (int c = 0; c < kApGK; c += 16) {
        float v[16];
        tmem_ld16(tO + (uint32_t)c, v);
        tmem_ld_wait();
        if (q < nvalid) {
          uint4 u0, u1;
          u0.x = pack_bf16_tc(v[0] * inv, v[1] * inv);
          u0.y = pack_bf16_tc(v[2] * inv, v[3] * inv);
          u0.z = pack_bf16_tc(v[4] * inv, v[5] * inv);
          u0.w = pack_bf16_tc(v[6] * inv, v[7] * inv);
          u1.x = pack_bf16_tc(v[8] * inv, v[9] * inv);
          u1.y = pack_bf16_tc(v[10] * inv, v[11] * inv);
          u1.z = pack_bf16_tc(v[12] * inv, v[13] * inv);
          u1.w = pack_bf16_tc(v[14] * inv, v[15] * inv);
          *reinterpret_cast<uint4*>(dst + c) = u0;
          *reinterpret_cast<uint4*>(dst + c + 8) = u1;
        }
      }
    }
  }

  if (splits > 1) {
    // ---------------- merge of the S pairs' partials (every thread of the cluster)
    // Row `row` of this CTA's 128 belongs to split p with 128 p / S <= row <
    // 128 (p + 1) / S; each CTA stores its unnormalised O half-rows and (m, l)
    // into the owner's shared memory, slot [source split][row - first owned
    // row] (rows of at most 64, stride kApMergeStride), and the owner combines
    // its rows locally. The first barrier says that every pair's MMAs are done
    // with the memory the slots reuse; the second that every slot is written.
    __syncwarp();
    cluster_arrive_release();
    cluster_wait_acquire();
    if (warp >= 2) {
      int own = 0;
      while (own + 1 < splits && (own + 1) * 128 / splits <= row) ++own;
      const int rr = row - own * 128 / splits;
      const uint32_t peer = (uint32_t)(2 * own + r);
      const uint32_t slot = (uint32_t)(pr * 64 + rr);
      const uint32_t dst = mapa_shared(smem_u32(mbuf + slot * kApMergeStride + grp * kApGK), peer);
#pragma unroll
      for (int c = 0; c < kApGK; c += 16) {
        float v[16];
        tmem_ld16(tmem + lane_off + 384u + (uint32_t)(grp * kApGK + c), v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          st_dsmem_f4(dst + (uint32_t)((c + i) * 4), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
      }
      if (grp == 0) st_dsmem_f2(mapa_shared(smem_u32(pm + 2 * slot), peer), m_use, lrow);
    }
    __syncwarp();
    cluster_arrive_release();
    cluster_wait_acquire();
    // this CTA's rows [128 p / S, 128 (p + 1) / S): O = sum over the source
    // splits (in split order) of 2^(m_q - M) O_q / sum_q 2^(m_q - M) l_q, the
    // weights of a row computed once into shared memory
    const int lo = pr * 128 / splits, hi = (pr + 1) * 128 / splits;
    float* wts = lsum;  // [64][4]
    if (threadIdx.x < hi - lo) {
      const int rr = threadIdx.x;
      float mstar = -INFINITY;
      for (int q = 0; q < splits; ++q) mstar = fmaxf(mstar, pm[2 * (q * 64 + rr)]);
      float w[kApMaxSplits], lstar = 0.0f;
#pragma unroll
      for (int q = 0; q < kApMaxSplits; ++q) {
        const float mq = q < splits ? pm[2 * (q * 64 + rr)] : -INFINITY;
        w[q] = mq == -INFINITY ? 0.0f : exp2f(mq - mstar);
        if (q < splits) lstar += w[q] * pm[2 * (q * 64 + rr) + 1];
      }
      const float inv = 1.0f / lstar;
#pragma unroll
      for (int q = 0; q < kApMaxSplits; ++q) wts[rr * 4 + q] = w[q] * inv;
      if (pstat) {
        const int qi = t * kApQ + r * 128 + lo + rr;
        if (qi < nvalid && prow[(size_t)b * pld + qi] >= 0 && prow[(size_t)b * pld + qi] < L)
          pstat[((size_t)b * pld + qi) * H + h] = make_float2(mstar, lstar);
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < (hi - lo) * 32; i += kApThreads) {
      const int rr = i >> 5, c4 = (i & 31) * 4;
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int q = 0; q < kApMaxSplits; ++q) {
        if (q < splits) {
          const float w = wts[rr * 4 + q];
          const float4 v = *reinterpret_cast<const float4*>(mbuf + (q * 64 + rr) * kApMergeStride + c4);
          acc.x += w * v.x;
          acc.y += w * v.y;
          acc.z += w * v.z;
          acc.w += w * v.w;
        }
      }
      const int qi = t * kApQ + r * 128 + lo + rr;
      if (qi < nvalid) {
        __nv_bfloat16* dst = O + ((size_t)b * R + qi) * ((size_t)H * kApHd) + h * kApHd + c4;
        uint2 u;
        u.x = pack_bf16_tc(acc.x, acc.y);
        u.y = pack_bf16_tc(acc.z, acc.w);
        *reinterpret_cast<uint2*>(dst) = u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while a peer may still read its memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

// Shared-memory opt-in, and how many clusters of 2 s CTAs can be resident at
// once (s = 1 .. 4), for the split choice. Non-zero on failure.
inline int attention_pair_setup(TcPlan* pl) {
  if (cudaFuncSetAttribute(attention_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kApSmem) !=
      cudaSuccess)
    return 1;
  for (int s = 1; s <= kApMaxSplits; ++s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * s, 1, 1);
    cfg.blockDim = dim3(kApThreads, 1, 1);
    cfg.dynamicSmemBytes = kApSmem;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = 2 * s;
    a[0].val.clusterDim.y = 1;
    a[0].val.clusterDim.z = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, attention_pair_kernel, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      nc = 0;
    }
    pl->ap_clusters[s] = nc;
  }
  return pl->ap_clusters[1] > 0 ? 0 : 1;
}

// Splits of a pair-tile's chunks: the most pairs per cluster (<= 4, at most
// one per chunk) for which every cluster of the launch is resident at once;
// one pair per pair-tile otherwise.
inline void attention_pair_plan(const TcPlan& pl, int B, int R, int L, int H, int* splits, int* cps) {
  const int nqt = (R + kApQ - 1) / kApQ, nch = (L + kApK - 1) / kApK;
  const long long tiles = (long long)nqt * H * B;  // clusters of the launch
  int s = 1;
  while (s < kApMaxSplits && s < nch && tiles <= pl.ap_clusters[s + 1] &&
         2LL * (s + 1) * tiles <= pl.num_sms)
    ++s;
  int c = (nch + s - 1) / s;
  s = (nch + c - 1) / c;  // every split non-empty
  *splits = s;
  *cps = c;
}

// Non-zero on failure (tensor-map encoding or launch).
// pstat (optional): for every valid query row q of sequence b with
// prow[b pld + q] in [0, L) (pld defaults to R), pstat[(b pld + q) H + h] =
// (row maximum, sum of 2^(score - maximum)) of the scores in base-2 units
// (q k / sqrt(128) log2 e): the row's probabilities are 2^(score - maximum) /
// sum. rows_valid (optional, device [B]): only query rows q < rows_valid[b]
// are valid; pair-tiles past them do no work, and their outputs and
// statistics are not written.
inline int attention_pair_launch(const TcPlan& pl, const void* Q, const void* K, const void* V, void* O, int B,
                                 int R, int L, int H, cudaStream_t st, uint64_t* launches,
                                 const int32_t* prow = nullptr, float2* pstat = nullptr,
                                 const int32_t* rows_valid = nullptr, int pld = 0) {
  if (R < 1 || L < 1) return 0;
  const uint64_t d = (uint64_t)H * kApHd;
  CUtensorMap mq, mk, mv;
  if (!encode_2d(pl, &mq, Q, (uint64_t)B * R, d, 128) || !encode_2d(pl, &mk, K, (uint64_t)B * L, d, 64) ||
      !encode_2d(pl, &mv, V, (uint64_t)B * L, d, 128))
    return 1;
  int splits, cps;
  attention_pair_plan(pl, B, R, L, H, &splits, &cps);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * splits, (R + kApQ - 1) / kApQ, H * B);
  cfg.blockDim = dim3(kApThreads, 1, 1);
  cfg.dynamicSmemBytes = kApSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2 * splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)kApHd);
  cudaError_t e = cudaLaunchKernelEx(&cfg, attention_pair_kernel, mq, mk, mv, (__nv_bfloat16*)O, R, L, H, splits,
                                     cps, scale_log2, pl.flag, prow, pstat, rows_valid, pld > 0 ? pld : R);
  (*launches)++;
  if (e != cudaSuccess) return 1;
  return cudaGetLastError() != cudaSuccess;
}

}  // namespace esd
