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
// Accumulators are double-buffered in TMEM when 2*MT*BN <= 512 columns, so the
// epilogue of one tile overlaps the main loop of the next.
//
// Each CTA tile covers MT*128 rows and BN weight rows, the latter fetched as two
// halves of BN/2 rows. The halves let one tile hold both members of a RoPE
// pair (head-dim j and j + 64) or the gate and up rows of the same SwiGLU
// column, so that every epilogue is row-local:
//   QKV     : scale by inv_rms, rotate-half RoPE at the row's position, store q
//             (compact) or scatter k / v into the K/V destination at the
//             position (the partial-cache update);
//   Residual: x = bf16(x + acc)   (O projection and FFN down projection);
//   SwiGLU  : act = bf16(silu(inv*g) * inv*u);
//   Head    : per (row, 128-column tile): max, argmax and sum exp(l - max) of
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
};

struct GemmParams {
  int M, K;
  int num_m, num_n, num_tiles;
  int d, n_heads, ffn, vocab, mask_id;
  EpiArgs e;
  int* flag;
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
                                          int* flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  raise_flag(flag, kFlagTimeout);
  return false;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
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

template <int MT, int BN>
struct TcCfg {
  static constexpr int kBK = 64;
  static constexpr int kABytes = 128 * kBK * 2;          // one 128-row A sub-tile
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = MT * kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024 / kStageBytes) > 8 ? 8 : (200 * 1024 / kStageBytes);
  static constexpr int kAcc = (2 * MT * BN <= 512) ? 2 : 1;
  static constexpr int kTmemCols = kAcc * MT * BN <= 32 ? 32
                                 : kAcc * MT * BN <= 64 ? 64
                                 : kAcc * MT * BN <= 128 ? 128
                                 : kAcc * MT * BN <= 256 ? 256 : 512;
  static constexpr int kSmem = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr uint32_t kTxBytes = (uint32_t)kStageBytes;
};

// ------------------------------------------------------------------ epilogues
template <int BN>
__device__ __forceinline__ void epi_store16_bf16(__nv_bfloat16* p, const float (&v)[16]) {
  uint4 u[2];
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(u);
#pragma unroll
  for (int i = 0; i < 8; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  reinterpret_cast<uint4*>(p)[0] = u[0];
  reinterpret_cast<uint4*>(p)[1] = u[1];
}

// Tile (m_blk, n_blk) -> B half-tile row coordinates for each epilogue kind.
// QKV: 3*H heads, each split into 128/BN tiles; half 0 = dims [j0, j0+BN/2),
// half 1 = dims [j0+64, j0+64+BN/2) of the same head (wq/wk/wv by section).
// SwiGLU: half 0 = gate rows [f0, f0+BN/2), half 1 = up rows [f0, f0+BN/2).
// Others: contiguous rows [n0, n0+BN).
template <int KIND, int BN>
__device__ __forceinline__ void b_rows(int n_blk, const GemmParams& p, int& map_sel, int& row0,
                                       int& row1) {
  if (KIND == kEpiQKV) {
    constexpr int per_head = 128 / BN;
    const int hh = n_blk / per_head, sub = n_blk % per_head;
    map_sel = hh / p.n_heads;
    const int h = hh % p.n_heads;
    row0 = h * 128 + sub * (BN / 2);
    row1 = row0 + 64;
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

template <int KIND, int MT, int BN>
__device__ __forceinline__ void run_epilogue(const GemmParams& p, int m_blk, int n_blk, int sub,
                                             uint32_t tmem_tile, int quarter, int lane) {
  const int r = m_blk * (MT * 128) + sub * 128 + quarter * 32 + lane;  // output row
  const bool live = r < p.M;
  const uint32_t tbase = tmem_tile + ((uint32_t)(quarter * 32) << 16);
  const EpiArgs& e = p.e;
  if (KIND == kEpiQKV) {
    constexpr int per_head = 128 / BN;
    const int hh = n_blk / per_head, s = n_blk % per_head;
    const int section = hh / p.n_heads, h = hh % p.n_heads;
    const float inv = live ? e.inv_rms[r] : 0.0f;
    const int R = e.R;
    const int b = live ? r / R : 0;
    const int pos = live ? (e.idx ? e.idx[r] : r % R) : 0;
    __nv_bfloat16* dst;
    if (section == 0)
      dst = reinterpret_cast<__nv_bfloat16*>(e.out) + (size_t)r * p.d + h * 128;
    else
      dst = reinterpret_cast<__nv_bfloat16*>(section == 1 ? e.k_dst : e.v_dst) +
            ((size_t)b * e.L + pos) * p.d + h * 128;
#pragma unroll
    for (int c = 0; c < BN / 2; c += 16) {
      float lo[16], hi[16];
      tmem_ld16(tbase + c, lo);
      tmem_ld16(tbase + BN / 2 + c, hi);
      tmem_ld_wait();
      if (!live) continue;
      const int j0 = s * (BN / 2) + c;  // head-dim index of lo[0]; partner j0 + 64
      float o_lo[16], o_hi[16];
      if (section == 2) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          o_lo[i] = lo[i] * inv;
          o_hi[i] = hi[i] * inv;
        }
      } else {
        const float2* tab = e.rope + (size_t)pos * 64 + j0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 cs = tab[i];
          const float a1 = lo[i] * inv, a2 = hi[i] * inv;
          o_lo[i] = a1 * cs.x - a2 * cs.y;
          o_hi[i] = a2 * cs.x + a1 * cs.y;
        }
      }
      epi_store16_bf16<BN>(dst + j0, o_lo);
      epi_store16_bf16<BN>(dst + j0 + 64, o_hi);
    }
  } else if (KIND == kEpiResidualO || KIND == kEpiResidualD) {
    __nv_bfloat16* x = reinterpret_cast<__nv_bfloat16*>(e.out) + (size_t)r * p.d + n_blk * BN;
#pragma unroll
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(tbase + c, v);
      tmem_ld_wait();
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
      epi_store16_bf16<BN>(x + c, o);
    }
  } else if (KIND == kEpiSwiGLU) {
    const float inv = live ? e.inv_rms[r] : 0.0f;
    __nv_bfloat16* a = reinterpret_cast<__nv_bfloat16*>(e.out) + (size_t)r * p.ffn + n_blk * (BN / 2);
#pragma unroll
    for (int c = 0; c < BN / 2; c += 16) {
      float g[16], u[16];
      tmem_ld16(tbase + c, g);
      tmem_ld16(tbase + BN / 2 + c, u);
      tmem_ld_wait();
      if (!live) continue;
      float o[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float gg = g[i] * inv;
        o[i] = gg / (1.0f + expf(-gg)) * (u[i] * inv);
      }
      epi_store16_bf16<BN>(a + c, o);
    }
  } else if (KIND == kEpiHead) {
    const float inv = live ? e.inv_rms[r] : 0.0f;
    const int n0 = n_blk * BN;
    float m = -INFINITY, s = 0.0f;
    int a = INT_MAX;
#pragma unroll
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(tbase + c, v);
      tmem_ld_wait();
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
        s = (s == 0.0f) ? 0.0f : s * expf(m - cm);
        m = cm;
        a = ca;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) s += expf(v[i] - m);  // exp(-inf) = 0
    }
    if (live) e.part[(size_t)r * e.n_tiles + n_blk] = HeadPartial{m, s, a};
  } else {  // kEpiLogits
    const float inv = live ? e.inv_rms[r] : 0.0f;
    const int n0 = n_blk * BN;
    float* out = reinterpret_cast<float*>(e.out) + (size_t)r * p.vocab;
#pragma unroll
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(tbase + c, v);
      tmem_ld_wait();
      if (!live) continue;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int col = n0 + c + i;
        if (col < p.vocab) out[col] = (col == p.mask_id) ? -INFINITY : v[i] * inv;
      }
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int KIND, int MT, int BN>
__global__ void __launch_bounds__(192, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
               const GemmParams p) {
  using C = TcCfg<MT, BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain; then tmem base and abort flag
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
  const int kb_count = p.K / C::kBK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int last_phase[8];
      bool used[8];
      for (int i = 0; i < 8; ++i) { used[i] = false; last_phase[i] = 0; }
      for (int t = blockIdx.x; t < p.num_tiles && !*abort_flag; t += gridDim.x) {
        const int m_blk = t % p.num_m, n_blk = t / p.num_m;
        int sel, row0, row1;
        b_rows<KIND, BN>(n_blk, p, sel, row0, row1);
        const CUtensorMap* mb0 = sel == 0 ? &tmB0 : (sel == 1 ? &tmB1 : &tmB2);
        const CUtensorMap* mb1 = (KIND == kEpiSwiGLU) ? &tmB1 : mb0;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.flag)) break;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, C::kTxBytes);
          uint8_t* sbase = smem + stage * C::kStageBytes;
          const int k0 = kb * C::kBK;
#pragma unroll
          for (int i = 0; i < MT; ++i)
            tma_load_2d(smem_u32(sbase + i * C::kABytes), &tmA, fb, k0, m_blk * (MT * 128) + i * 128);
          uint8_t* bb = sbase + MT * C::kABytes;
          tma_load_2d(smem_u32(bb), mb0, fb, k0, row0);
          tma_load_2d(smem_u32(bb + C::kBBytes / 2), mb1, fb, k0, row1);
          used[stage] = true;
          last_phase[stage] = (int)phase;
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // drain: every stage this thread filled has landed before the CTA exits
      for (int i = 0; i < C::kStages; ++i)
        if (used[i]) {
          for (uint32_t it = 0; it < kWaitLimit; ++it)
            if (mbar_try_wait(smem_u32(&full[i]), (uint32_t)last_phase[i])) break;
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16(128, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < p.num_tiles && !*abort_flag; t += gridDim.x) {
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.flag)) break;
        tc_fence_after();
        const uint32_t tacc = tmem + (uint32_t)(acc * MT * BN);
        bool ok = true;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sbase = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t bbase = sbase + MT * C::kABytes;
#pragma unroll
          for (int kk = 0; kk < C::kBK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(bbase + kk * 32);
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              const uint64_t adesc = smem_desc_sw128(sbase + i * C::kABytes + kk * 32);
              tc_mma(tacc + (uint32_t)(i * BN), adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
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
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.flag)) break;
      tc_fence_after();
      const int m_blk = t % p.num_m, n_blk = t / p.num_m;
#pragma unroll
      for (int i = 0; i < MT; ++i)
        run_epilogue<KIND, MT, BN>(p, m_blk, n_blk, i, tmem + (uint32_t)(acc * MT * BN + i * BN),
                                   quarter, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      if (++acc == C::kAcc) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
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
  // weight maps per layer, for half-tile heights 32 (BN 64) and 64 (BN 128)
  std::vector<CUtensorMap> q32, k32, v32, o32, g32, u32, d32;
  std::vector<CUtensorMap> q64, k64, v64, o64, g64, u64, d64;
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

template <int KIND, int MT, int BN>
inline void tc_set_attr() {
  cudaFuncSetAttribute(tc_gemm_kernel<KIND, MT, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       TcCfg<MT, BN>::kSmem);
}

template <int MT, int BN>
inline void tc_set_attr_all() {
  tc_set_attr<kEpiQKV, MT, BN>();
  tc_set_attr<kEpiResidualO, MT, BN>();
  tc_set_attr<kEpiSwiGLU, MT, BN>();
  tc_set_attr<kEpiResidualD, MT, BN>();
  tc_set_attr<kEpiHead, MT, BN>();
  tc_set_attr<kEpiLogits, MT, BN>();
}

inline esd_status tc_plan_create(TcPlan* pl, const TcWeights& w, int max_rows, std::string* err,
                                 int* flag) {
  (void)max_rows;
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
  bool ok = mk(pl->q32, w.wq, d, d, 32) && mk(pl->k32, w.wk, d, d, 32) && mk(pl->v32, w.wv, d, d, 32) &&
            mk(pl->o32, w.wo, d, d, 32) && mk(pl->g32, w.wg, f, d, 32) && mk(pl->u32, w.wu, f, d, 32) &&
            mk(pl->d32, w.wd, d, f, 32) && mk(pl->q64, w.wq, d, d, 64) && mk(pl->k64, w.wk, d, d, 64) &&
            mk(pl->v64, w.wv, d, d, 64) && mk(pl->o64, w.wo, d, d, 64) && mk(pl->g64, w.wg, f, d, 64) &&
            mk(pl->u64, w.wu, f, d, 64) && mk(pl->d64, w.wd, d, f, 64) &&
            encode_2d(*pl, &pl->out64, w.w_out, (uint64_t)w.vocab, d, 64);
  if (!ok) {
    *err = "cuTensorMapEncodeTiled failed for a weight matrix";
    return ESD_ERR_CUDA;
  }
  tc_set_attr_all<1, 64>();
  tc_set_attr_all<2, 64>();
  tc_set_attr_all<2, 128>();
  tc_set_attr<kEpiHead, 1, 128>();
  tc_set_attr<kEpiLogits, 1, 128>();
  if (cudaGetLastError() != cudaSuccess) {
    *err = "cudaFuncSetAttribute failed for the tensor-core GEMM";
    return ESD_ERR_CUDA;
  }
  return ESD_OK;
}

template <int KIND, int MT, int BN>
inline cudaError_t tc_launch_cfg(const TcPlan& pl, const CUtensorMap& a, const CUtensorMap& b0,
                                 const CUtensorMap& b1, const CUtensorMap& b2, GemmParams p,
                                 cudaStream_t st) {
  p.num_m = (p.M + MT * 128 - 1) / (MT * 128);
  int num_n;
  if (KIND == kEpiQKV) num_n = 3 * p.n_heads * (128 / BN);
  else if (KIND == kEpiSwiGLU) num_n = p.ffn / (BN / 2);
  else if (KIND == kEpiHead || KIND == kEpiLogits) num_n = (p.vocab + BN - 1) / BN;
  else num_n = p.d / BN;
  p.num_n = num_n;
  p.num_tiles = p.num_m * num_n;
  const int grid = p.num_tiles < pl.num_sms ? p.num_tiles : pl.num_sms;
  tc_gemm_kernel<KIND, MT, BN><<<grid, 192, TcCfg<MT, BN>::kSmem, st>>>(a, b0, b1, b2, p);
  return cudaGetLastError();
}

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
  CUtensorMap a;
  if (!encode_2d(pl, &a, A, (uint64_t)M, (uint64_t)p.K, 128)) {
    *err = "cuTensorMapEncodeTiled failed for the activation operand";
    return ESD_ERR_CUDA;
  }
  const bool head = (kind == kEpiHead || kind == kEpiLogits);
  // small M: narrow tiles to spread the weight stream over more SMs
  const int cfg = head ? (M <= 128 ? 1 : 2) : (M <= 128 ? 0 : (M <= 256 ? 1 : 2));
  cudaError_t r = cudaSuccess;
#define ESD_TC_KIND(KIND, B0, B1, B2)                                                   \
  do {                                                                                  \
    if (cfg == 0) r = tc_launch_cfg<KIND, 1, 64>(pl, a, B0##32[layer], B1##32[layer], B2##32[layer], p, st); \
    else if (cfg == 1 && !head) r = tc_launch_cfg<KIND, 2, 64>(pl, a, B0##32[layer], B1##32[layer], B2##32[layer], p, st); \
    else r = tc_launch_cfg<KIND, 2, 128>(pl, a, B0##64[layer], B1##64[layer], B2##64[layer], p, st); \
  } while (0)
  switch (kind) {
    case kEpiQKV: ESD_TC_KIND(kEpiQKV, pl.q, pl.k, pl.v); break;
    case kEpiResidualO: ESD_TC_KIND(kEpiResidualO, pl.o, pl.o, pl.o); break;
    case kEpiSwiGLU: ESD_TC_KIND(kEpiSwiGLU, pl.g, pl.u, pl.u); break;
    case kEpiResidualD: ESD_TC_KIND(kEpiResidualD, pl.d, pl.d, pl.d); break;
    case kEpiHead:
      if (cfg == 1) r = tc_launch_cfg<kEpiHead, 1, 128>(pl, a, pl.out64, pl.out64, pl.out64, p, st);
      else r = tc_launch_cfg<kEpiHead, 2, 128>(pl, a, pl.out64, pl.out64, pl.out64, p, st);
      break;
    case kEpiLogits:
      if (cfg == 1) r = tc_launch_cfg<kEpiLogits, 1, 128>(pl, a, pl.out64, pl.out64, pl.out64, p, st);
      else r = tc_launch_cfg<kEpiLogits, 2, 128>(pl, a, pl.out64, pl.out64, pl.out64, p, st);
      break;
    default: *err = "unknown GEMM kind"; return ESD_ERR_INVALID_ARG;
  }
#undef ESD_TC_KIND
  (*launches)++;
  if (r != cudaSuccess) {
    *err = std::string("tensor-core GEMM launch failed: ") + cudaGetErrorString(r);
    return ESD_ERR_CUDA;
  }
  return ESD_OK;
}

}  // namespace esd
