// Tensor-core GEMM for sm_100a: C = A W^T with A [M, K] bf16 activations and
// W [N, K] bf16 weights (both K-major), fp32 accumulation in tensor memory.
//
// Persistent, warp-specialised kernel (192 threads):
//   warp 0      TMA producer: A sub-tiles and two B half-tiles per k-block,
//               128-byte swizzled, into a STAGES-deep shared-memory ring;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//               (kind::f16, M = 128 per sub-tile, N = BN, K = 16 per MMA);
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulators (one TMEM lane
//               quarter per warp, one output row per thread), fused with the
//               layer's next operation.
// Accumulators are double-buffered in TMEM when 2*MT*BN <= 512 columns (MT =
// 128-row sub-tiles per tile), so the epilogue of one tile overlaps the main
// loop of the next. A tile has TM = 128, 192 or 256 rows; a 192-row tile is one
// M=128 and one M=64 MMA (no padded rows are multiplied), its second part
// occupying TMEM lanes 0-15 of each 32-lane quarter.
//
// Work units: a tile of TM rows x BN weight rows, optionally split along K
// into S parts (split-K) so that small-M GEMMs (the selected rows of a sparse
// step) keep every SM streaming weights. A split unit stores its fp32 partial
// to a workspace; a second kernel, parallel over (tile, sub-tile, column
// group), sums the S partials in split order (deterministic) and runs the same
// fused epilogue. No CTA waits for another. Each unit walks its k-blocks from
// a unit-dependent offset, so that concurrent CTAs do not all read the same
// activation k-block from the same L2 slices at once.
//
// The weight tile is fetched as two halves of BN/2 rows, which lets one tile
// hold both members of a RoPE pair (head-dim j and j + 64: a whole head for
// BN >= 128) or the gate and up rows of the same SwiGLU column, so that every
// epilogue is row-local:
//   QKV     : scale by inv_rms, rotate-half RoPE at the row's position, store q
//             (compact) or scatter k / v into the K/V destination at the
//             position (the partial-cache update);
//   Residual: x = bf16(x + acc)   (O projection and FFN down projection);
//   SwiGLU  : act = bf16(silu(inv*g) * inv*u);
//   Head    : per (row, BN-column tile): max, argmax and sum exp(l - max) of
//             the logits l = inv*acc with the mask id excluded (logits never
//             reach memory);
//   Logits  : float32 logits to memory (test helper).
// Every mbarrier wait is bounded; on expiry the kernel raises the context's
// error flag, stops issuing work, drains what it issued and frees its TMEM.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <string>
#include <vector>

#include "common.cuh"
#include "esd.h"

namespace esd {

enum EpiKind { kEpiQKV = 0, kEpiResidualO = 1, kEpiSwiGLU = 2, kEpiResidualD = 3, kEpiHead = 4, kEpiLogits = 5 };

struct EpiArgs {
  const float* inv_rms = nullptr;
  const int32_t* idx = nullptr;  // positions of the rows (QKV), nullptr = r % R
  const float2* rope = nullptr;  // [max_len, 64] (cos, sin)
  int R = 0;                     // rows per sequence
  int L = 0;                     // sequence length (K/V destination rows per sequence)
  void* out = nullptr;           // q / x / act / logits
  void* k_dst = nullptr;
  void* v_dst = nullptr;
  HeadPartial* part = nullptr;
  int n_tiles = 0;
  // RMS statistic as partial sums of squares ([parts][256] floats, summed in
  // part order by the consumer; rms_parts == 0: use inv_rms), and the partials
  // a residual epilogue writes for the next consumer (nullable)
  const float* rms_part_in = nullptr;
  int rms_parts = 0;
  float rms_eps = 0.0f;
  float* rms_part_out = nullptr;
  float* inv_out = nullptr;  // the inverse RMS computed from rms_part_in, [M] (swapped-operand GEMMs)
};

struct GemmParams {
  int M, K;
  int num_m, num_n, num_tiles;
  int splits, num_units;
  int d, n_heads, ffn, vocab, mask_id;
  EpiArgs e;
  float* ws;      // split-K partials [tile][split][TM x BN, see ws_index]
  int skw;        // workers of the two-SM kernel (SM pairs)
  int sk_whole;   // 1: each worker takes a contiguous range of whole tiles
  long long sk_total;  // iterations: tiles x k-blocks
  int* flag;
  int mp, stages;      // swapped-operand kernel: token rows padded to 16, ring stages
  int sk_whole_tiles;  // swapped-operand kernel: tiles [0, this) go whole to the pairs, round robin
};

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: about a second or more of polling before giving up.
constexpr uint32_t kWaitLimit = 1u << 24;
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* flag, uint32_t limit = kWaitLimit) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  raise_flag(flag, kFlagTimeout);
  return false;
}
// the same decision in every lane of the warp
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag, flag);
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
// L2 eviction policies: weights stream through once (evict first); activations
// are re-read by every weight tile and split-K partials by the reduction, so
// they should stay (evict last).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void st_f4_keep(float* ptr, float4 v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(ptr), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 lanes x 32 bit, 16 consecutive columns per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  __syncwarp();
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15},"
      " [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes grouped by 8 (stride 1024 B between groups), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;           // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32; // stride byte offset
  d |= (uint64_t)1u << 46;           // version
  d |= (uint64_t)2u << 61;           // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16: D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int TM, int BN>
struct TcCfg {
  static_assert(TM == 128 || TM == 192 || TM == 256, "tile rows");
  static constexpr int kBK = 64;
  static constexpr int MT = (TM + 127) / 128;           // MMAs (sub-tiles) per k-step
  static constexpr int kABytes = TM * kBK * 2;            // the activation tile of a stage
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // 227 KB of dynamic shared memory, less alignment slack and barriers
  static constexpr int kStages = ((232448 - 1280) / kStageBytes) > 8 ? 8 : ((232448 - 1280) / kStageBytes);
  static constexpr int kAcc = (2 * MT * BN <= 512) ? 2 : 1;
  static constexpr int kTmemCols = kAcc * MT * BN <= 32 ? 32
                                 : kAcc * MT * BN <= 64 ? 64
                                 : kAcc * MT * BN <= 128 ? 128
                                 : kAcc * MT * BN <= 256 ? 256 : 512;
  static constexpr int kSmem = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr uint32_t kTxBytes = (uint32_t)kStageBytes;
  static constexpr int kTileRows = TM;
  // rows of sub-tile t, and the tile row held by TMEM lane (32*quarter + lane)
  __host__ __device__ static constexpr int sub_rows(int t) { return (TM == 192 && t == 1) ? 64 : 128; }
  __device__ static int row_of(int t, int quarter, int lane) {
    return (TM == 192 && t == 1) ? (lane < 16 ? 128 + quarter * 16 + lane : -1)
                                 : t * 128 + quarter * 32 + lane;
  }
};

// ------------------------------------------------------------------ epilogues
__device__ __forceinline__ void store16_bf16(__nv_bfloat16* p, const float (&v)[16]) {
  uint4 u[2];
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(u);
#pragma unroll
  for (int i = 0; i < 8; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  reinterpret_cast<uint4*>(p)[0] = u[0];
  reinterpret_cast<uint4*>(p)[1] = u[1];
}

// Tile column block n_blk -> which weight map and the rows of the two B halves.
// QKV: BN/128 whole heads, contiguous rows within one of wq/wk/wv (d % BN == 0).
// SwiGLU: half 0 = gate rows [f0, f0+BN/2), half 1 = up rows [f0, f0+BN/2).
// Others: contiguous rows [n0, n0+BN).
template <int KIND, int BN>
__device__ __forceinline__ void b_rows(int n_blk, const GemmParams& p, int& map_sel, int& row0,
                                       int& row1) {
  if (KIND == kEpiQKV) {
    const int n0 = n_blk * BN;
    map_sel = n0 / p.d;
    row0 = n0 - map_sel * p.d;
    row1 = row0 + BN / 2;
  } else if (KIND == kEpiSwiGLU) {
    map_sel = 0;
    row0 = n_blk * (BN / 2);
    row1 = row0;
  } else {
    map_sel = 0;
    row0 = n_blk * BN;
    row1 = row0 + BN / 2;
  }
}

// Accumulator sources for the epilogue: TMEM (the unit's own accumulator) or
// the sum of a tile's split-K partials in split order.
struct TmemSrc {
  uint32_t tbase;
  __device__ __forceinline__ void get(int col, float (&v)[16]) const { tmem_ld16(tbase + col, v); }
  __device__ __forceinline__ void sync() const { tmem_ld_wait(); }
};

// Split-K partial of one unit: for each 16-column chunk c and quarter q
// (columns 4q..4q+3 of the chunk), a plane of [tile rows] float4, so that the
// 32 lanes of a warp (32 consecutive rows) touch 512 contiguous bytes.
__device__ __forceinline__ size_t ws_index(int chunk, int q, int row, int tile_rows) {
  return ((size_t)(chunk * 4 + q) * tile_rows + row) * 4;
}

template <int BN>
struct WsSrc {
  const float* base;  // partial of split 0 of this tile
  size_t split_stride;
  int splits;
  int row;            // row within the tile
  int tile_rows;
  bool live;
  __device__ __forceinline__ void get(int col, float (&v)[16]) const {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    if (!live) return;
    for (int s = 0; s < splits; ++s) {
      const float* b = base + s * split_stride;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 f = __ldcg(reinterpret_cast<const float4*>(b + ws_index(col >> 4, q, row, tile_rows)));
        v[4 * q] += f.x;
        v[4 * q + 1] += f.y;
        v[4 * q + 2] += f.z;
        v[4 * q + 3] += f.w;
      }
    }
  }
  __device__ __forceinline__ void sync() const {}
};

// Column groups of a tile's epilogue (the split-K reduction kernel spreads them
// over blocks): QKV: (head, 16-dim chunk of the first half) pairs; SwiGLU: 16
// columns of gate and up; residual: 16 columns. Head and logits never split.
template <int KIND, int BN>
__host__ __device__ constexpr int epi_groups() {
  return KIND == kEpiQKV ? BN / 32 : (KIND == kEpiSwiGLU ? BN / 32 : BN / 16);
}

// Epilogue of output row r (live = r < M) for column groups [g0, g1).
template <int KIND, int BN, class Src>
__device__ __forceinline__ void epilogue_rows(const GemmParams& p, int n_blk, int r, bool live,
                                              const Src& src, int g0 = 0,
                                              int g1 = epi_groups<KIND, BN>()) {
  const EpiArgs& e = p.e;
  if (KIND == kEpiQKV) {
    // a negative position marks a padding row: nothing of it is written
    const int pos_r = live ? (e.idx ? e.idx[r] : r % e.R) : 0;
    live = live && pos_r >= 0;
    const float inv = live ? e.inv_rms[r] : 0.0f;
    const int b = live ? r / e.R : 0;
    const int pos = live ? pos_r : 0;
    const int n0 = n_blk * BN;
    const int section = n0 / p.d;
    const bool rot = section != 2 && live;
    // the rotation factors of group gg + 1 are loaded while group gg is finished
    float4 cs_next[8];
    if (rot && g0 < g1) {
      const float4* tab = reinterpret_cast<const float4*>(e.rope + (size_t)pos * 64 + (g0 & 3) * 16);
#pragma unroll
      for (int i = 0; i < 8; ++i) cs_next[i] = tab[i];
    }
    for (int gg = g0; gg < g1; ++gg) {
      const int g = gg >> 2;         // head within the tile
      const int c = (gg & 3) * 16;   // first-half dims c..c+15, partners c+64..
      const int h = (n0 - section * p.d) / 128 + g;
      float4 cs[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) cs[i] = cs_next[i];
      if (rot && gg + 1 < g1) {
        const float4* tab = reinterpret_cast<const float4*>(e.rope + (size_t)pos * 64 + ((gg + 1) & 3) * 16);
#pragma unroll
        for (int i = 0; i < 8; ++i) cs_next[i] = tab[i];
      }
      __nv_bfloat16* dst;
      if (section == 0)
        dst = reinterpret_cast<__nv_bfloat16*>(e.out) + (size_t)r * p.d + h * 128;
      else
        dst = reinterpret_cast<__nv_bfloat16*>(section == 1 ? e.k_dst : e.v_dst) +
              ((size_t)b * e.L + pos) * p.d + h * 128;
      {
        float lo[16], hi[16];
        src.get(g * 128 + c, lo);
        src.get(g * 128 + 64 + c, hi);
        src.sync();
        if (!live) continue;
        float o_lo[16], o_hi[16];
        if (section == 2) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            o_lo[i] = lo[i] * inv;
            o_hi[i] = hi[i] * inv;
          }
        } else {
          const float2* cs2 = reinterpret_cast<const float2*>(cs);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a1 = lo[i] * inv, a2 = hi[i] * inv;
            o_lo[i] = a1 * cs2[i].x - a2 * cs2[i].y;
            o_hi[i] = a2 * cs2[i].x + a1 * cs2[i].y;
          }
        }
        store16_bf16(dst + c, o_lo);
        store16_bf16(dst + c + 64, o_hi);
      }
    }
  } else if (KIND == kEpiResidualO || KIND == kEpiResidualD) {
    __nv_bfloat16* x = reinterpret_cast<__nv_bfloat16*>(e.out) + (size_t)r * p.d + n_blk * BN;
#pragma unroll 4
    for (int c = g0 * 16; c < g1 * 16; c += 16) {
      float v[16];
      src.get(c, v);
      src.sync();
      if (!live) continue;
      uint4 u[2];
      u[0] = reinterpret_cast<const uint4*>(x + c)[0];
      u[1] = reinterpret_cast<const uint4*>(x + c)[1];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(u);
      float o[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        o[2 * i] = f.x + v[2 * i];
        o[2 * i + 1] = f.y + v[2 * i + 1];
      }
      store16_bf16(x + c, o);
    }
  } else if (KIND == kEpiSwiGLU) {
    const float inv = live ? e.inv_rms[r] : 0.0f;
    __nv_bfloat16* a = reinterpret_cast<__nv_bfloat16*>(e.out) + (size_t)r * p.ffn + n_blk * (BN / 2);
#pragma unroll 2
    for (int c = g0 * 16; c < g1 * 16; c += 16) {
      float g[16], u[16];
      src.get(c, g);
      src.get(BN / 2 + c, u);
      src.sync();
      if (!live) continue;
      float o[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float gg = g[i] * inv;
        // silu with the fast exponential and divide (relative error ~1e-6,
        // far below the bf16 rounding of the product)
        o[i] = __fdividef(gg, 1.0f + __expf(fminf(-gg, 80.0f))) * (u[i] * inv);
      }
      store16_bf16(a + c, o);
    }
  } else if (KIND == kEpiHead) {
    const float inv = live ? e.inv_rms[r] : 0.0f;
    const int n0 = n_blk * BN;
    float m = -INFINITY, s = 0.0f;
    int a = INT_MAX;
#pragma unroll 2
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      src.get(c, v);
      src.sync();
      float cm = -INFINITY;
      int ca = INT_MAX;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int col = n0 + c + i;
        const bool ok = col < p.vocab && col != p.mask_id;
        v[i] = ok ? v[i] * inv : -INFINITY;
        if (v[i] > cm) { cm = v[i]; ca = col; }
      }
      if (cm == -INFINITY) continue;
      if (cm > m) {
        s = (s == 0.0f) ? 0.0f : s * __expf(m - cm);
        m = cm;
        a = ca;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) s += __expf(v[i] - m);  // exp(-inf) = 0
    }
    if (live) e.part[(size_t)r * e.n_tiles + n_blk] = HeadPartial{m, s, a};
  } else {  // kEpiLogits
    const float inv = live ? e.inv_rms[r] : 0.0f;
    const int n0 = n_blk * BN;
    float* out = reinterpret_cast<float*>(e.out) + (size_t)r * p.vocab;
#pragma unroll 2
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      src.get(c, v);
      src.sync();
      if (!live) continue;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int col = n0 + c + i;
        if (col < p.vocab) out[col] = (col == p.mask_id) ? -INFINITY : v[i] * inv;
      }
    }
  }
}

// k-blocks [kb0, kb1) of unit u, walked from a unit-dependent offset
__device__ __forceinline__ void unit_range(const GemmParams& p, int u, int kb_total, int& tile,
                                           int& split, int& kb0, int& nkb, int& koff) {
  tile = u / p.splits;
  split = u - tile * p.splits;
  kb0 = (int)(((long long)split * kb_total) / p.splits);
  const int kb1 = (int)(((long long)(split + 1) * kb_total) / p.splits);
  nkb = kb1 - kb0;
  koff = nkb > 0 ? (int)(((unsigned)u * 7u) % (unsigned)nkb) : 0;
}

// ------------------------------------------------------------------ kernel
template <int KIND, int TM, int BN>
__global__ void __launch_bounds__(192, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
               const GemmParams p) {
  using C = TcCfg<TM, BN>;
  constexpr int MT = C::MT;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain; then tmem base, abort flag, ticket flag
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tfull = bars + 2 * C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 4);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int kb_total = p.K / C::kBK;
  // the prologue above may overlap the previous kernel; its outputs are read
  // from here on
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_phase = 0;  // per stage: loaded at least once / parity of its last load
      for (int u = blockIdx.x; u < p.num_units && !*abort_flag; u += gridDim.x) {
        int tile, split, kb0, nkb, koff;
        unit_range(p, u, kb_total, tile, split, kb0, nkb, koff);
        const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
        int sel, row0, row1;
        b_rows<KIND, BN>(n_blk, p, sel, row0, row1);
        const CUtensorMap* mb0 = sel == 0 ? &tmB0 : (sel == 1 ? &tmB1 : &tmB2);
        const CUtensorMap* mb1 = (KIND == kEpiSwiGLU) ? &tmB1 : mb0;
        for (int i = 0; i < nkb; ++i) {
          int kb = koff + i;
          if (kb >= nkb) kb -= nkb;
          kb += kb0;
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.flag)) break;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, C::kTxBytes);
          uint8_t* sbase = smem + stage * C::kStageBytes;
          const int k0 = kb * C::kBK;
          tma_load_2d(smem_u32(sbase), &tmA, fb, k0, m_blk * C::kTileRows, pol_a);
          uint8_t* bb = sbase + C::kABytes;
          tma_load_2d(smem_u32(bb), mb0, fb, k0, row0, pol_w);
          tma_load_2d(smem_u32(bb + C::kBBytes / 2), mb1, fb, k0, row1, pol_w);
          used |= 1u << stage;
          last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // drain: every stage this thread filled has landed before the CTA exits
      for (int i = 0; i < C::kStages; ++i)
        if ((used >> i) & 1u) {
          for (uint32_t it = 0; it < kWaitLimit; ++it)
            if (mbar_try_wait(smem_u32(&full[i]), ((last_phase >> i) & 1u))) break;
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc0 = idesc_bf16(128, BN);
      constexpr uint32_t idesc1 = idesc_bf16(C::sub_rows(1), BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int u = blockIdx.x; u < p.num_units && !*abort_flag; u += gridDim.x) {
        int tile, split, kb0, nkb, koff;
        unit_range(p, u, kb_total, tile, split, kb0, nkb, koff);
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.flag)) break;
        tc_fence_after();
        const uint32_t tacc = tmem + (uint32_t)(acc * MT * BN);
        bool ok = true;
        for (int i = 0; i < nkb; ++i) {
          // the TMA bytes are ordered before the MMA's operand reads by the
          // barrier itself (both in the async proxy): no thread fence needed
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.flag)) { ok = false; break; }
          const uint32_t sbase = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t bbase = sbase + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < C::kBK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(bbase + kk * 32);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              const uint64_t adesc = smem_desc_sw128(sbase + t * 128 * 128 + kk * 32);
              tc_mma(tacc + (uint32_t)(t * BN), adesc, bdesc, t == 0 ? idesc0 : idesc1,
                     (i | kk) != 0 ? 1u : 0u);
            }
          }
          issued = true;
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull[acc]));
        if (++acc == C::kAcc) { acc = 0; acc_phase ^= 1u; }
      }
      if (issued) {
        // all MMAs this thread issued have completed before TMEM is freed
        tc_commit(smem_u32(drain));
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(drain), 0u)) break;
      }
    }
  } else {
    // ---------------- epilogue warps 2..5
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
      int tile, split, kb0, nkb, koff;
      unit_range(p, u, kb_total, tile, split, kb0, nkb, koff);
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.flag)) break;
      tc_fence_after();
      const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
      const uint32_t tacc = tmem + (uint32_t)(acc * MT * BN) + ((uint32_t)(quarter * 32) << 16);
      if (p.splits == 1) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const int lr = C::row_of(t, quarter, lane);
          const int r = m_blk * C::kTileRows + lr;
          epilogue_rows<KIND, BN>(p, n_blk, r, lr >= 0 && r < p.M, TmemSrc{tacc + (uint32_t)(t * BN)});
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      } else {
        // store this split's partial (the reduction kernel finishes the tile)
        const size_t split_stride = (size_t)C::kTileRows * BN;
        float* wt = p.ws + ((size_t)tile * p.splits + split) * split_stride;
        const uint64_t pol_keep = policy_evict_last();
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const int lr = C::row_of(t, quarter, lane);
          const bool live = lr >= 0 && m_blk * C::kTileRows + lr < p.M;
#pragma unroll 4
          for (int c = 0; c < BN; c += 16) {
            float v[16];
            tmem_ld16(tacc + (uint32_t)(t * BN + c), v);
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
        if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      }
      if (++acc == C::kAcc) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// Split-K reduction + fused epilogue: block = (tile, 128-row sub-tile, part of
// the tile's column groups), one thread per row; sums the S partials in split
// order and applies the same epilogue as the unsplit kernel.
template <int KIND, int TM, int BN>
__global__ void __launch_bounds__(128)
tc_splitk_epilogue_kernel(const GemmParams p, int n_parts) {
  grid_launch_dependents();
  grid_dependency_wait();  // the GEMM's partials
  constexpr int kTileRows = TM;
  constexpr int MT = TcCfg<TM, BN>::MT;
  constexpr int G = epi_groups<KIND, BN>();
  int bid = blockIdx.x;
  const int part = bid % n_parts;
  bid /= n_parts;
  const int t = bid % MT;
  const int tile = bid / MT;
  const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
  const int lr = t * 128 + threadIdx.x;
  const int r = m_blk * kTileRows + lr;
  const bool live = r < p.M && lr < kTileRows;
  if (m_blk * kTileRows + t * 128 >= p.M) return;  // a sub-tile of padding rows only
  const size_t split_stride = (size_t)kTileRows * BN;
  WsSrc<BN> src{p.ws + (size_t)tile * p.splits * split_stride, split_stride, p.splits, lr, kTileRows, live};
  const int g0 = (part * G) / n_parts, g1 = ((part + 1) * G) / n_parts;
  epilogue_rows<KIND, BN>(p, n_blk, r, live, src, g0, g1);
}

// ------------------------------------------------------------------ host side
struct TcWeights {
  int d, ffn, vocab, mask_id, n_heads, n_layers;
  const void* w_out;
  const void* const* wq;
  const void* const* wk;
  const void* const* wv;
  const void* const* wo;
  const void* const* wg;
  const void* const* wu;
  const void* const* wd;
};

struct TcPlan {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  TcWeights w{};
  int num_sms = 148;
  int* flag = nullptr;
  float* ws = nullptr;      // split-K partials
  size_t ws_floats = 0;
  int max_tiles = 0;
  // resident clusters of the cluster split-K kernel: [QKV, O, SwiGLU, down][TM 128, 192][BN 128, 256][S]
  int cl_max[4][2][2][9] = {};
  // weight maps per layer, for half-tile heights 64 (BN 128) and 128 (BN 256)
  std::vector<CUtensorMap> q64, k64, v64, o64, g64, u64, d64;
  std::vector<CUtensorMap> q128, k128, v128, o128, g128, u128, d128;
  std::vector<CUtensorMap> g96, u96;  // SwiGLU halves of the 192-wide SM-pair tiles
  int ap_clusters[5] = {};  // co-resident clusters of the pair attention kernel with 2 s CTAs (index s)
  CUtensorMap out64{};
};

inline bool encode_2d(const TcPlan& pl, CUtensorMap* m, const void* base, uint64_t rows,
                      uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = pl.encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                         strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int KIND, int TM, int BN>
inline void tc_set_attr() {
  cudaFuncSetAttribute(tc_gemm_kernel<KIND, TM, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       TcCfg<TM, BN>::kSmem);
}

template <int TM, int BN>
inline void tc_set_attr_layers() {
  tc_set_attr<kEpiQKV, TM, BN>();
  tc_set_attr<kEpiResidualO, TM, BN>();
  tc_set_attr<kEpiSwiGLU, TM, BN>();
  tc_set_attr<kEpiResidualD, TM, BN>();
}

// Largest number of work units a split GEMM may use: two per SM.
inline int tc_max_units(int num_sms) { return 2 * num_sms; }

// ws is a device buffer owned by the caller (the context), sized with
// tc_workspace_floats.
inline size_t tc_workspace_floats(int num_sms) { return (size_t)tc_max_units(num_sms) * 256 * 256; }

inline esd_status tc_plan_create(TcPlan* pl, const TcWeights& w, std::string* err, int* flag) {
  pl->w = w;
  pl->flag = flag;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn) {
    *err = "cuTensorMapEncodeTiled not available";
    return ESD_ERR_UNSUPPORTED;
  }
  pl->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&pl->num_sms, cudaDevAttrMultiProcessorCount, dev);
  const int L = w.n_layers;
  auto mk = [&](std::vector<CUtensorMap>& v, const void* const* ptrs, uint64_t rows, uint64_t cols,
                uint32_t box) {
    v.resize(L);
    for (int l = 0; l < L; ++l)
      if (!encode_2d(*pl, &v[l], ptrs[l], rows, cols, box)) return false;
    return true;
  };
  const uint64_t d = w.d, f = w.ffn;
  bool ok = mk(pl->q64, w.wq, d, d, 64) && mk(pl->k64, w.wk, d, d, 64) && mk(pl->v64, w.wv, d, d, 64) &&
            mk(pl->o64, w.wo, d, d, 64) && mk(pl->g64, w.wg, f, d, 64) && mk(pl->u64, w.wu, f, d, 64) &&
            mk(pl->d64, w.wd, d, f, 64) && mk(pl->q128, w.wq, d, d, 128) &&
            mk(pl->k128, w.wk, d, d, 128) && mk(pl->v128, w.wv, d, d, 128) &&
            mk(pl->o128, w.wo, d, d, 128) && mk(pl->g128, w.wg, f, d, 128) &&
            mk(pl->u128, w.wu, f, d, 128) && mk(pl->d128, w.wd, d, f, 128) &&
            mk(pl->g96, w.wg, f, d, 96) && mk(pl->u96, w.wu, f, d, 96) &&
            encode_2d(*pl, &pl->out64, w.w_out, (uint64_t)w.vocab, d, 64);
  if (!ok) {
    *err = "cuTensorMapEncodeTiled failed for a weight matrix";
    return ESD_ERR_CUDA;
  }
  tc_set_attr_layers<128, 256>();
  tc_set_attr_layers<256, 128>();
  tc_set_attr<kEpiHead, 128, 128>();
  tc_set_attr<kEpiHead, 192, 128>();
  tc_set_attr<kEpiHead, 256, 128>();
  tc_set_attr<kEpiLogits, 128, 128>();
  tc_set_attr<kEpiLogits, 256, 128>();
  if (cudaGetLastError() != cudaSuccess) {
    *err = "cudaFuncSetAttribute failed for the tensor-core GEMM";
    return ESD_ERR_CUDA;
  }
  return ESD_OK;
}

// Split count for `tiles` tiles of `kb_total` k-blocks: minimise the number of
// whole-tile times the busiest SM needs (ceil(tiles*S / SMs) / S), preferring
// fewer splits on ties, with at least 4 k-blocks per split.
inline int choose_splits(int tiles, int kb_total, int num_sms) {
  int best = 1;
  double best_t = (double)((tiles + num_sms - 1) / num_sms);
  for (int s = 2; s <= 16; ++s) {
    if (kb_total / s < 4 || tiles * s > tc_max_units(num_sms)) break;
    const double t = (double)((tiles * s + num_sms - 1) / num_sms) / s;
    if (t < best_t - 1e-9) {
      best_t = t;
      best = s;
    }
  }
  return best;
}

// Split count for `tiles` tiles of `kb_total` k-blocks: split only when the
// tiles leave more than half of the SMs idle; then minimise the number of
// whole-tile times the busiest SM needs (ceil(tiles*S / SMs) / S), preferring
// fewer splits on ties, with at least 4 k-blocks per split.
inline int choose_splits_sparse(int tiles, int kb_total, int num_sms) {
  if (2 * tiles >= num_sms) return 1;
  return choose_splits(tiles, kb_total, num_sms);
}

template <int KIND, int TM, int BN>
inline cudaError_t tc_launch_cfg(const TcPlan& pl, const void* A, const CUtensorMap& b0,
                                 const CUtensorMap& b1, const CUtensorMap& b2, GemmParams p,
                                 bool allow_split, cudaStream_t st, uint64_t* launches) {
  constexpr int MT = TcCfg<TM, BN>::MT;
  CUtensorMap a;
  if (!encode_2d(pl, &a, A, (uint64_t)p.M, (uint64_t)p.K, TM)) return cudaErrorInvalidValue;
  p.num_m = (p.M + TM - 1) / TM;
  int num_n;
  if (KIND == kEpiQKV) num_n = 3 * p.d / BN;
  else if (KIND == kEpiSwiGLU) num_n = p.ffn / (BN / 2);
  else if (KIND == kEpiHead || KIND == kEpiLogits) num_n = (p.vocab + BN - 1) / BN;
  else num_n = p.d / BN;
  p.num_n = num_n;
  p.num_tiles = p.num_m * num_n;
  p.splits = 1;
  if (KIND != kEpiHead && KIND != kEpiLogits && allow_split && pl.ws && p.num_tiles <= pl.max_tiles)
    p.splits = choose_splits_sparse(p.num_tiles, p.K / 64, pl.num_sms);
  p.num_units = p.num_tiles * p.splits;
  p.ws = pl.ws;
  const int grid = p.num_units < pl.num_sms ? p.num_units : pl.num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = TcCfg<TM, BN>::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tc_gemm_kernel<KIND, TM, BN>, a, b0, b1, b2, p);
  (*launches)++;
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  if constexpr (KIND != kEpiHead && KIND != kEpiLogits) {
    // enough blocks to cover every SM twice
    constexpr int G = epi_groups<KIND, BN>();
    int n_parts = (2 * pl.num_sms + p.num_tiles * MT - 1) / (p.num_tiles * MT);
    if (n_parts > G) n_parts = G;
    if (n_parts < 1) n_parts = 1;
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3(p.num_tiles * MT * n_parts, 1, 1);
    c2.blockDim = dim3(128, 1, 1);
    c2.stream = st;
    cudaLaunchAttribute a2[1];
    a2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a2[0].val.programmaticStreamSerializationAllowed = 1;
    c2.attrs = a2;
    c2.numAttrs = 1;
    e = cudaLaunchKernelEx(&c2, tc_splitk_epilogue_kernel<KIND, TM, BN>, p, n_parts);
    (*launches)++;
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  return e;
}

template <int KIND, int BN>
inline cudaError_t tc2_launch(const TcPlan& pl, const void* A, const CUtensorMap& b0, const CUtensorMap& b1,
                              const CUtensorMap& b2, GemmParams p, cudaStream_t st, uint64_t* launches);

// SM-pair tile width of the SwiGLU GEMM on M rows: 192 (96 gate + 96 up) when
// its rounds of tiles over the SM pairs, weighted by the narrower tile's cost
// (~0.83 of a 256-wide tile), take less time.
inline int tc2_swiglu_bn(int M, int ffn, int num_sms) {
  if (ffn % 96 != 0) return 256;
  const int pairs = num_sms / 2, m_blks = (M + 255) / 256;
  const int r256 = (m_blks * (ffn / 128) + pairs - 1) / pairs, r192 = (m_blks * (ffn / 96) + pairs - 1) / pairs;
  return 0.83 * r192 < r256 ? 192 : 256;
}

template <int KIND>
inline cudaError_t tc_cl_dispatch(const TcPlan& pl, int layer, const void* A, const GemmParams& p,
                                  cudaStream_t st, uint64_t* launches, bool* done);

template <int KIND>
inline cudaError_t tc_skinny_launch(const TcPlan& pl, const void* A, const CUtensorMap& b0, const CUtensorMap& b1,
                                    const CUtensorMap& b2, GemmParams p, cudaStream_t st, uint64_t* launches);
inline bool tc_skinny_ok(const TcPlan& pl, int M);

// Dispatch one GEMM of the layer (or the head) on A [M, K].
inline esd_status tc_gemm(TcPlan& pl, int kind, int layer, const void* A, int M, const EpiArgs& e,
                          cudaStream_t st, uint64_t* launches, std::string* err) {
  const TcWeights& w = pl.w;
  GemmParams p{};
  p.M = M;
  p.d = w.d;
  p.n_heads = w.n_heads;
  p.ffn = w.ffn;
  p.vocab = w.vocab;
  p.mask_id = w.mask_id;
  p.e = e;
  p.flag = pl.flag;
  p.K = (kind == kEpiResidualD) ? w.ffn : w.d;
  cudaError_t r = cudaSuccess;
  if (kind == kEpiHead || kind == kEpiLogits) {
    const CUtensorMap& o = pl.out64;
    if (kind == kEpiHead) {
      if (M <= 128) r = tc_launch_cfg<kEpiHead, 128, 128>(pl, A, o, o, o, p, false, st, launches);
      else if (M <= 192) r = tc_launch_cfg<kEpiHead, 192, 128>(pl, A, o, o, o, p, false, st, launches);
      else r = tc_launch_cfg<kEpiHead, 256, 128>(pl, A, o, o, o, p, false, st, launches);
    } else {
      if (M <= 128) r = tc_launch_cfg<kEpiLogits, 128, 128>(pl, A, o, o, o, p, false, st, launches);
      else r = tc_launch_cfg<kEpiLogits, 256, 128>(pl, A, o, o, o, p, false, st, launches);
    }
  } else {
    // up to 128 rows (few selected rows): one SM per 128 x 256 tile; more rows:
    // SM pairs on 256 x 256 tiles (tc_gemm2.cuh); 256 x 128 tiles when d is
    // not a multiple of 256
    const int cfg = (w.d % 256 != 0) ? 3 : (M <= 128 ? 0 : 1);
#define ESD_TC_KIND(KIND, B0, B1, B2)                                                                \
  do {                                                                                               \
    bool done = false;                                                                               \
    if (tc_skinny_ok(pl, M)) {                                                                       \
      r = tc_skinny_launch<KIND>(pl, A, B0##64[layer], B1##64[layer], B2##64[layer], p, st, launches); \
      break;                                                                                         \
    }                                                                                                \
    if (cfg != 3 && M <= 192) {                                                                      \
      r = tc_cl_dispatch<KIND>(pl, layer, A, p, st, launches, &done);                                \
      if (done || r != cudaSuccess) break;                                                           \
    }                                                                                                \
    if (cfg == 0) r = tc_launch_cfg<KIND, 128, 256>(pl, A, B0##128[layer], B1##128[layer], B2##128[layer], p, true, st, launches); \
    else if (cfg == 1 && KIND == kEpiSwiGLU && tc2_swiglu_bn(M, w.ffn, pl.num_sms) == 192)        \
      r = tc2_launch<kEpiSwiGLU, 192>(pl, A, pl.g96[layer], pl.u96[layer], pl.u96[layer], p, st, launches); \
    else if (cfg == 1) r = tc2_launch<KIND, 256>(pl, A, B0##128[layer], B1##128[layer], B2##128[layer], p, st, launches); \
    else r = tc_launch_cfg<KIND, 256, 128>(pl, A, B0##64[layer], B1##64[layer], B2##64[layer], p, true, st, launches); \
  } while (0)
    switch (kind) {
      case kEpiQKV: ESD_TC_KIND(kEpiQKV, pl.q, pl.k, pl.v); break;
      case kEpiResidualO: ESD_TC_KIND(kEpiResidualO, pl.o, pl.o, pl.o); break;
      case kEpiSwiGLU: ESD_TC_KIND(kEpiSwiGLU, pl.g, pl.u, pl.u); break;
      case kEpiResidualD: ESD_TC_KIND(kEpiResidualD, pl.d, pl.d, pl.d); break;
      default: *err = "unknown GEMM kind"; return ESD_ERR_INVALID_ARG;
    }
#undef ESD_TC_KIND
  }
  if (r != cudaSuccess) {
    *err = std::string("tensor-core GEMM launch failed: ") + cudaGetErrorString(r);
    return ESD_ERR_CUDA;
  }
  return ESD_OK;
}

}  // namespace esd
