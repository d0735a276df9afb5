// Partial attention on the fifth-generation tensor cores (tcgen05), bf16,
// head_dim 128 ("DyLLM", technical summary section 2.B.2: the salient rows of
// the attention matrix are recomputed exactly; with every row selected this is
// the dense bidirectional attention).
//
// One CTA = 128 query rows of one head of one sequence, 6 warps:
//   warp 0      TMA: the Q tile once, then K/V tiles of 128 keys through a
//               two-stage ring (K and V of a tile share a stage; every tile is
//               two 64-column boxes with the 128-byte swizzle);
//   warp 1      TMEM allocator and the single MMA-issuing thread:
//               S_j = Q K_j^T (M 128 queries, N 128 keys, K 128 dims, both
//               operands K-major) into one of two TMEM S buffers, and
//               O += P_j V_j (A = P_j from shared memory, K-major; B = V_j in
//               its stored [keys][dims] layout, i.e. MN-major) into TMEM;
//   warps 2..5  one query row per thread: tcgen05.ld of the S_j row, online
//               softmax in base 2, P_j rounded to bf16 into a swizzled shared
//               tile (double-buffered), and the running-max correction of O.
// The correction is lazy: the row maximum used for P only moves when the
// tile's maximum exceeds it by more than 2^8 (P <= 256 otherwise), and then
// the thread rescales its O row in TMEM after the previous P V product has
// landed. The result O / l is exact either way; only how often O is rescaled
// changes. S_{j+1} is computed while the softmax of tile j runs. Keys beyond
// the sequence's L are masked; query rows beyond its R rows are computed and
// not stored. Every wait is bounded (error flag, drain, TMEM freed).
#pragma once

#include "tc_gemm.cuh"

namespace esd {

constexpr int kAtQ = 128;   // query rows per CTA
constexpr int kAtK = 128;   // keys per tile
constexpr int kAtHd = 128;  // head dim
constexpr int kAtBox = 128 * 64 * 2;             // one [128 rows][64 cols] bf16 box = 16 KB
constexpr int kAtQBytes = 2 * kAtBox;            // Q: dims 0-63 | 64-127
constexpr int kAtKVBytes = 4 * kAtBox;           // K (2 boxes) then V (2 boxes)
constexpr int kAtPBytes = 2 * kAtBox;            // P: keys 0-63 | 64-127
constexpr int kAtSmem = kAtQBytes + 2 * kAtKVBytes + 2 * kAtPBytes + 1024 + 256;
constexpr float kAtLazy = 8.0f;                  // log2 of the largest unnormalised P

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

// Q [B*R, H*128], K and V [B*L, H*128] (rows of the sequences back to back),
// O [B*R, H*128]; grid (ceil(R / 128), H, B). K and V rows [0, B*L) finite.
__global__ void __launch_bounds__(192, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O, int R,
                    int L, int H, float scale_log2, int* flag) {
  extern __shared__ __align__(1024) uint8_t smem_at_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_at_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + kAtQBytes;               // [stage][K0 K1 V0 V1]
  uint8_t* sP = sKV + 2 * kAtKVBytes;          // [buffer][P0 P1]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kAtPBytes);
  uint64_t* qfull = bars;        // Q landed
  uint64_t* kvfull = bars + 1;   // [2] K_j/V_j landed
  uint64_t* kvempty = bars + 3;  // [2] S_j and P_j V_j done with the stage
  uint64_t* sfull = bars + 5;    // [2] S_j in TMEM
  uint64_t* sfree = bars + 7;    // [2] S_j read (4 softmax warps)
  uint64_t* pfull = bars + 9;    // [2] P_j written and O corrected (4 warps)
  uint64_t* ofull = bars + 11;   // [2] P_j V_j accumulated (P buffer free again)
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kAtQ, h = blockIdx.y, b = blockIdx.z;
  const int n_tiles = (L + kAtK - 1) / kAtK;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(qfull), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&kvfull[i]), 1);
      mbar_init(smem_u32(&kvempty[i]), 1);
      mbar_init(smem_u32(&sfull[i]), 1);
      mbar_init(smem_u32(&sfree[i]), 4);
      mbar_init(smem_u32(&pfull[i]), 4);
      mbar_init(smem_u32(&ofull[i]), 1);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);  // S buffers: cols 0-255; O: 256-383
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem + 256u;

  if (warp == 0) {
    if (lane == 0 && n_tiles > 0) {
      // ---------------- TMA producer
      const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_last();
      const int kvrow = b * L;
      mbar_expect_tx(smem_u32(qfull), kAtQBytes);
      tma_load_2d(smem_u32(sQ), &tmQ, smem_u32(qfull), h * kAtHd, b * R + q0, pol_q);
      tma_load_2d(smem_u32(sQ + kAtBox), &tmQ, smem_u32(qfull), h * kAtHd + 64, b * R + q0, pol_q);
      int last = -1;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        if (!mbar_wait(smem_u32(&kvempty[s]), ((j >> 1) & 1) ^ 1u, abort_flag, flag)) break;
        const uint32_t fb = smem_u32(&kvfull[s]);
        mbar_expect_tx(fb, kAtKVBytes);
        uint8_t* st = sKV + s * kAtKVBytes;
        const int r = kvrow + j * kAtK;
        tma_load_2d(smem_u32(st), &tmK, fb, h * kAtHd, r, pol_kv);
        tma_load_2d(smem_u32(st + kAtBox), &tmK, fb, h * kAtHd + 64, r, pol_kv);
        tma_load_2d(smem_u32(st + 2 * kAtBox), &tmV, fb, h * kAtHd, r, pol_kv);
        tma_load_2d(smem_u32(st + 3 * kAtBox), &tmV, fb, h * kAtHd + 64, r, pol_kv);
        last = j;
      }
      // drain: every load issued has landed before the CTA exits
      for (uint32_t it = 0; it < kWaitLimit; ++it)
        if (mbar_try_wait(smem_u32(qfull), 0u)) break;
      for (int j = last - 1; j <= last; ++j) {
        if (j < 0) continue;
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(&kvfull[j & 1]), (uint32_t)((j >> 1) & 1))) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0) {
      // ---------------- MMA issuer
      constexpr uint32_t id_s = idesc_bf16_b(128, 128, 0);
      constexpr uint32_t id_o = idesc_bf16_b(128, 128, 1);
      bool issued = false;
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t par = (uint32_t)((j >> 1) & 1);
        if (!mbar_wait(smem_u32(&kvfull[s]), par, abort_flag, flag)) return false;
        if (!mbar_wait(smem_u32(&sfree[s]), par ^ 1u, abort_flag, flag)) return false;
        tc_fence_after();
        const uint32_t kb = smem_u32(sKV + s * kAtKVBytes), qb = smem_u32(sQ);
#pragma unroll
        for (int kk = 0; kk < kAtHd / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kAtBox + (kk & 3) * 32);
          tc_mma(tmem + (uint32_t)(s * 128), smem_desc_sw128(qb + off), smem_desc_sw128(kb + off), id_s,
                 kk != 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&sfull[s]));
        issued = true;
        return true;
      };
      bool ok = mbar_wait(smem_u32(qfull), 0u, abort_flag, flag) && issue_s(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !issue_s(j + 1)) break;
        const int s = j & 1;
        if (!mbar_wait(smem_u32(&pfull[s]), (uint32_t)((j >> 1) & 1), abort_flag, flag)) break;
        tc_fence_after();
        const uint32_t pb = smem_u32(sP + s * kAtPBytes);
        const uint32_t vb = smem_u32(sKV + s * kAtKVBytes + 2 * kAtBox);
#pragma unroll
        for (int kk = 0; kk < kAtK / 16; ++kk) {
          const uint32_t aoff = (uint32_t)((kk >> 2) * kAtBox + (kk & 3) * 32);  // P: 64 keys per box
          const uint32_t boff = (uint32_t)(kk * 16 * 128);                       // V: 16 key rows
          tc_mma(tmem_o, smem_desc_sw128(pb + aoff), smem_desc_sw128_mn(vb + boff, kAtBox), id_o,
                 (j | kk) != 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&ofull[s]));
        tc_commit(smem_u32(&kvempty[s]));
      }
      if (issued) {
        tc_commit(smem_u32(drain));
        for (uint32_t it = 0; it < kWaitLimit; ++it)
          if (mbar_try_wait(smem_u32(drain), 0u)) break;
      }
    }
  } else if (n_tiles > 0) {
    // ---------------- softmax warps: one query row per thread
    const int quarter = warp & 3;          // TMEM lanes a warp may access: 32 * (warp % 4) ...
    const int row = quarter * 32 + lane;   // query row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float m_use = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      const uint32_t par = (uint32_t)((j >> 1) & 1);
      if (!(ok = warp_wait(smem_u32(&sfull[s]), par, abort_flag, flag))) break;
      tc_fence_after();
      float sv[kAtK];
#pragma unroll
      for (int c = 0; c < kAtK; c += 16) {
        float v[16];
        tmem_ld16(tmem + lane_off + (uint32_t)(s * 128 + c), v);
#pragma unroll
        for (int i = 0; i < 16; ++i) sv[c + i] = v[i];
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sfree[s]));
      const int kbase = j * kAtK;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kAtK; ++i) {
        sv[i] = (kbase + i < L) ? sv[i] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, sv[i]);
      }
      // lazy correction of the running maximum (key j*128 < L: mx is finite)
      const bool need = mx > m_use + kAtLazy;
      if (j == 0) {
        m_use = mx;
      } else if (__any_sync(0xffffffffu, need)) {
        // O holds the products of tiles < j: wait for P_{j-1} V_{j-1}
        if (!(ok = warp_wait(smem_u32(&ofull[(j - 1) & 1]), (uint32_t)(((j - 1) >> 1) & 1), abort_flag,
                             flag)))
          break;
        tc_fence_after();
        const float f = need ? exp2f(m_use - mx) : 1.0f;
#pragma unroll
        for (int c = 0; c < kAtHd; c += 16) {
          float v[16];
          tmem_ld16(tmem_o + lane_off + (uint32_t)c, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= f;
          tmem_st16(tmem_o + lane_off + (uint32_t)c, v);
        }
        tmem_st_wait();
        if (need) {
          l *= f;
          m_use = mx;
        }
      }
      // P_j into buffer s once P_{j-2} V_{j-2} has read it
      if (j >= 2 && !(ok = warp_wait(smem_u32(&ofull[s]), par ^ 1u, abort_flag, flag))) break;
      uint8_t* pt = sP + s * kAtPBytes;
      float rs = 0.0f;
#pragma unroll
      for (int c = 0; c < kAtK / 8; ++c) {  // 16 chunks of 8 keys (16 B)
        float pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pv[i] = exp2f(sv[c * 8 + i] - m_use);
          rs += pv[i];
        }
        uint4 u;
        u.x = pack_bf16_tc(pv[0], pv[1]);
        u.y = pack_bf16_tc(pv[2], pv[3]);
        u.z = pack_bf16_tc(pv[4], pv[5]);
        u.w = pack_bf16_tc(pv[6], pv[7]);
        const int box = c >> 3, ch = c & 7;
        *reinterpret_cast<uint4*>(pt + box * kAtBox + row * 128 + ((ch ^ (row & 7)) << 4)) = u;
      }
      l += rs;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P visible to the tensor cores
      tc_fence_before();                                             // and the O correction
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&pfull[s]));
    }
    // O / l, rounded to bf16, for the query rows of this sequence
    const int jl = n_tiles - 1;
    if (ok && warp_wait(smem_u32(&ofull[jl & 1]), (uint32_t)((jl >> 1) & 1), abort_flag, flag)) {
      tc_fence_after();
      const int r = q0 + row;
      const float inv = 1.0f / l;
      __nv_bfloat16* dst = O + ((size_t)b * R + r) * ((size_t)H * kAtHd) + h * kAtHd;
#pragma unroll
      for (int c = 0; c < kAtHd; c += 16) {
        float v[16];
        tmem_ld16(tmem_o + lane_off + (uint32_t)c, v);
        tmem_ld_wait();
        if (r < R) {
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

inline int attention_tc_setup() {
  return cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAtSmem) !=
         cudaSuccess;
}

// Non-zero on failure (tensor-map encoding or launch).
inline int attention_tc_launch(const TcPlan& pl, const void* Q, const void* K, const void* V, void* O, int B,
                               int R, int L, int H, cudaStream_t st, uint64_t* launches) {
  const uint64_t d = (uint64_t)H * kAtHd;
  CUtensorMap mq, mk, mv;
  if (!encode_2d(pl, &mq, Q, (uint64_t)B * R, d, kAtQ) || !encode_2d(pl, &mk, K, (uint64_t)B * L, d, kAtK) ||
      !encode_2d(pl, &mv, V, (uint64_t)B * L, d, kAtK))
    return 1;
  const dim3 grid((R + kAtQ - 1) / kAtQ, H, B);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)kAtHd);
  attention_tc_kernel<<<grid, 192, kAtSmem, st>>>(mq, mk, mv, (__nv_bfloat16*)O, R, L, H, scale_log2, pl.flag);
  (*launches)++;
  return cudaGetLastError() != cudaSuccess;
}

}  // namespace esd
