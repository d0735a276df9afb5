// Partial attention for the bf16 models (head_dim 128): the selected queries of
// a sequence attend over the whole K/V of that sequence (the layer's cache after
// the fresh rows were scattered in), softmax(q K^T / sqrt(128)) V with an online
// softmax ("DyLLM", technical summary section 2.B.2: exact recomputation of the
// salient rows of the attention matrix). With every row selected this is the
// dense bidirectional attention.
//
// One CTA = 64 query rows x one head x one sequence x one slice of the keys, 4
// warps of 16 rows. Q is staged once; K/V tiles of 64 keys stream through a
// double-buffered shared-memory ring (cp.async, 16-byte chunks, XOR-swizzled
// rows so that ldmatrix is conflict-free). QK^T and PV use bf16 m16n8k16
// tensor-core MMAs with fp32 accumulation; P is rounded to bf16 for the PV
// product. When the keys are split over S CTAs (few query tiles: the selected
// rows of a sparse step), each CTA stores its unnormalised output, row maxima
// and row sums; the CTA that takes the last ticket of its (query tile, head,
// sequence) merges the S partials in split order and writes the result. No CTA
// waits for another.
#pragma once

#include "common.cuh"

namespace esd {

constexpr int kAttnQ = 64;
constexpr int kAttnK = 64;
constexpr int kAttnHd = 128;
constexpr int kAttnSmem = (kAttnQ + 4 * kAttnK) * kAttnHd * 2;  // Q + 2 x (K, V)

__device__ __forceinline__ uint32_t swz(int row, int chunk) {  // byte offset in a [rows][256 B] tile
  return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9},"
      " {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Load a [64 rows][128] bf16 tile (row stride ld elements) into swizzled smem;
// rows >= valid_rows are zero-filled.
__device__ __forceinline__ void load_tile64(uint32_t sbase, const __nv_bfloat16* g, size_t ld,
                                            int valid_rows, int tid) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = tid + i * 128;  // 1024 chunks of 16 B
    const int row = c >> 4, chunk = c & 15;
    const bool ok = row < valid_rows;
    const __nv_bfloat16* src = ok ? g + (size_t)row * ld + chunk * 8 : g;
    cp_async16(sbase + swz(row, chunk), src, ok);
  }
}

// Partials of one (query tile, head, sequence, key slice): unnormalised O
// [64][128], then row maximum (base 2) [64] and row sum [64].
constexpr int kAttnPartFloats = kAttnQ * kAttnHd + 2 * kAttnQ;

// Q [B*R, H*128] compact rows; K, V [B*L, H*128]; O [B*R, H*128].
// blockIdx.z = b * splits + split; split s covers key tiles [s*tps, (s+1)*tps).
__global__ void __launch_bounds__(128)
attention_mma_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                     const __nv_bfloat16* __restrict__ V, __nv_bfloat16* __restrict__ O, int R,
                     int L, int H, float scale_log2, int splits, int tps, float* __restrict__ part,
                     int* __restrict__ tickets) {
  __shared__ int s_last;
  extern __shared__ __align__(1024) uint8_t sm_attn[];
  grid_launch_dependents();
  const uint32_t sQ = smem_u32(sm_attn);
  const uint32_t sK[2] = {sQ + kAttnQ * 256, sQ + kAttnQ * 256 + 2 * kAttnK * 256};
  const uint32_t sV[2] = {sK[0] + kAttnK * 256, sK[1] + kAttnK * 256};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = blockIdx.x * kAttnQ, h = blockIdx.y;
  const int b = blockIdx.z / splits, split = blockIdx.z % splits;
  const size_t ld = (size_t)H * kAttnHd;
  const __nv_bfloat16* Qg = Q + ((size_t)b * R + q0) * ld + h * kAttnHd;
  const __nv_bfloat16* Kg = K + (size_t)b * L * ld + h * kAttnHd;
  const __nv_bfloat16* Vg = V + (size_t)b * L * ld + h * kAttnHd;

  const int t_begin = split * tps;
  const int t_end = min((L + kAttnK - 1) / kAttnK, t_begin + tps);
  load_tile64(sQ, Qg, ld, R - q0, tid);
  load_tile64(sK[0], Kg + (size_t)t_begin * kAttnK * ld, ld, L - t_begin * kAttnK, tid);
  load_tile64(sV[0], Vg + (size_t)t_begin * kAttnK * ld, ld, L - t_begin * kAttnK, tid);
  cp_async_commit();

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.0f, 0.0f};
  uint32_t qa[8][4];

  for (int t = t_begin; t < t_end; ++t) {
    const int buf = (t - t_begin) & 1;
    if (t + 1 < t_end) {
      const int k1 = (t + 1) * kAttnK;
      load_tile64(sK[buf ^ 1], Kg + (size_t)k1 * ld, ld, L - k1, tid);
      load_tile64(sV[buf ^ 1], Vg + (size_t)k1 * ld, ld, L - k1, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == t_begin) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int row = warp * 16 + (lane & 15);
        const int chunk = kk * 2 + (lane >> 4);
        ldsm_x4(sQ + swz(row, chunk), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }
    // S = Q K^T for 64 keys: 8 n-tiles of 8 keys
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // pairs of n-tiles (16 keys)
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int chunk = kk * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK[buf] + swz(key, chunk), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
        mma_bf16(s[2 * np + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
      }
    }
    // mask keys beyond L, online softmax (base 2)
    const int kbase = t * kAttnK;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kbase + n * 8 + 2 * (lane & 3) + (e & 1);
        float v = s[n][e] * scale_log2;
        if (key >= L) v = -INFINITY;
        s[n][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
    }
    float corr[2], mnew[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mnew[i] = fmaxf(m_r[i], mx[i]);
      corr[i] = (m_r[i] == -INFINITY) ? 0.0f : exp2f(m_r[i] - mnew[i]);
      m_r[i] = mnew[i];
    }
    float rs[2] = {0.0f, 0.0f};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[n][e] - mnew[e >> 1]);
        s[n][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) l_r[i] = l_r[i] * corr[i] + rs[i];
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
      o[dn][0] *= corr[0];
      o[dn][1] *= corr[0];
      o[dn][2] *= corr[1];
      o[dn][3] *= corr[1];
    }
    // O += P V: 4 k-steps of 16 keys, 16 n-tiles of 8 dims
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a0 = pack_bf16(s[2 * j][0], s[2 * j][1]);
      const uint32_t a1 = pack_bf16(s[2 * j][2], s[2 * j][3]);
      const uint32_t a2 = pack_bf16(s[2 * j + 1][0], s[2 * j + 1][1]);
      const uint32_t a3 = pack_bf16(s[2 * j + 1][2], s[2 * j + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {  // pairs of dim tiles (16 dims)
        const int key = j * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int chunk = dp * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV[buf] + swz(key, chunk), b0, b1, b2, b3);
        mma_bf16(o[2 * dp], a0, a1, a2, a3, b0, b1);
        mma_bf16(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();  // the buffer is refilled by the next iteration's prefetch
  }
  // row sums across the quad
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
  }
  const int lr0 = warp * 16 + (lane >> 2), lr1 = lr0 + 8;  // rows within the tile
  const int r0 = q0 + lr0, r1 = q0 + lr1;
  if (splits == 1) {
    const float inv0 = 1.0f / l_r[0], inv1 = 1.0f / l_r[1];
    __nv_bfloat16* O0 = O + ((size_t)b * R + r0) * ld + h * kAttnHd;
    __nv_bfloat16* O1 = O + ((size_t)b * R + r1) * ld + h * kAttnHd;
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
      const int col = dn * 8 + 2 * (lane & 3);
      if (r0 < R)
        *reinterpret_cast<__nv_bfloat162*>(O0 + col) = __floats2bfloat162_rn(o[dn][0] * inv0, o[dn][1] * inv0);
      if (r1 < R)
        *reinterpret_cast<__nv_bfloat162*>(O1 + col) = __floats2bfloat162_rn(o[dn][2] * inv1, o[dn][3] * inv1);
    }
    return;
  }
  // split keys: store this slice's partial, then the last CTA merges
  const int group = (b * gridDim.y + h) * gridDim.x + blockIdx.x;  // (sequence, head, query tile)
  float* mine = part + ((size_t)group * splits + split) * kAttnPartFloats;
#pragma unroll
  for (int dn = 0; dn < 16; ++dn) {
    const int col = dn * 8 + 2 * (lane & 3);
    __stcg(reinterpret_cast<float2*>(mine + lr0 * kAttnHd + col), make_float2(o[dn][0], o[dn][1]));
    __stcg(reinterpret_cast<float2*>(mine + lr1 * kAttnHd + col), make_float2(o[dn][2], o[dn][3]));
  }
  if ((lane & 3) == 0) {
    mine[kAttnQ * kAttnHd + lr0] = m_r[0];
    mine[kAttnQ * kAttnHd + lr1] = m_r[1];
    mine[kAttnQ * kAttnHd + kAttnQ + lr0] = l_r[0];
    mine[kAttnQ * kAttnHd + kAttnQ + lr1] = l_r[1];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(&tickets[group], 1);
    s_last = (old == splits - 1);
    if (s_last) tickets[group] = 0;  // ready for the next launch
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* base = part + (size_t)group * splits * kAttnPartFloats;
  // per-row merge weights 2^(m_s - max) / sum, then every output independently
  float* wsm = reinterpret_cast<float*>(sm_attn);  // [64 rows][splits] (Q/K/V tiles are dead now)
  if (tid < kAttnQ) {
    float mx = -INFINITY;
    for (int s2 = 0; s2 < splits; ++s2)
      mx = fmaxf(mx, __ldcg(base + (size_t)s2 * kAttnPartFloats + kAttnQ * kAttnHd + tid));
    float l = 0.0f;
    for (int s2 = 0; s2 < splits; ++s2) {
      const float* ps = base + (size_t)s2 * kAttnPartFloats;
      const float w = exp2f(__ldcg(ps + kAttnQ * kAttnHd + tid) - mx);
      wsm[tid * splits + s2] = w;
      l += __ldcg(ps + kAttnQ * kAttnHd + kAttnQ + tid) * w;
    }
    const float inv = 1.0f / l;
    for (int s2 = 0; s2 < splits; ++s2) wsm[tid * splits + s2] *= inv;
  }
  __syncthreads();
  // every output row is a weighted sum of the S partial rows; a thread
  // handles 4 consecutive dims of 4 rows and issues the loads of up to 4
  // splits before the first add (splits added in order)
  const int rows = min(kAttnQ, R - q0);
  constexpr int kMs = 4;
  for (int i0 = tid; i0 < rows * (kAttnHd / 4); i0 += 128 * 4) {
    float4 acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int sb = 0; sb < splits; sb += kMs) {
      float4 v[4][kMs];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 128;
        const int row = i / (kAttnHd / 4), c4 = (i % (kAttnHd / 4)) * 4;
#pragma unroll
        for (int j = 0; j < kMs; ++j)
          if (i < rows * (kAttnHd / 4) && sb + j < splits)
            v[u][j] = __ldcg(reinterpret_cast<const float4*>(base + (size_t)(sb + j) * kAttnPartFloats +
                                                             row * kAttnHd + c4));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 128;
        const int row = i / (kAttnHd / 4);
#pragma unroll
        for (int j = 0; j < kMs; ++j)
          if (i < rows * (kAttnHd / 4) && sb + j < splits) {
            const float w = wsm[row * splits + sb + j];
            acc[u].x += v[u][j].x * w;
            acc[u].y += v[u][j].y * w;
            acc[u].z += v[u][j].z * w;
            acc[u].w += v[u][j].w * w;
          }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * 128;
      if (i >= rows * (kAttnHd / 4)) break;
      const int row = i / (kAttnHd / 4), c4 = (i % (kAttnHd / 4)) * 4;
      __nv_bfloat16* dst = O + ((size_t)b * R + q0 + row) * ld + h * kAttnHd + c4;
      *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc[u].x, acc[u].y);
      *reinterpret_cast<__nv_bfloat162*>(dst + 2) = __floats2bfloat162_rn(acc[u].z, acc[u].w);
    }
  }
}

inline int attention_mma_setup() {
  return cudaFuncSetAttribute(attention_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kAttnSmem) != cudaSuccess;
}

// Key-split workspace: partials of at most kAttnMaxSplitCtas CTAs and one
// ticket per (sequence, head, query tile) of a split launch.
constexpr int kAttnMaxSplitCtas = 1184;
constexpr int kAttnMaxGroups = 1184;
inline size_t attention_ws_floats() { return (size_t)kAttnMaxSplitCtas * kAttnPartFloats; }

// returns non-zero on a launch error
inline int attention_mma_launch(const void* Q, const void* K, const void* V, void* O, int B, int R,
                                int L, int H, int num_sms, float* part, int* tickets,
                                cudaStream_t st, uint64_t* launches) {
  const int q_tiles = (R + kAttnQ - 1) / kAttnQ;
  const int k_tiles = (L + kAttnK - 1) / kAttnK;
  const int groups = q_tiles * H * B;
  // split the keys only when the query tiles leave most SMs idle (each CTA's
  // walk over the keys is latency-bound, so a split pays only when few CTAs
  // run: three splits of the 96 tiles of 192 queries x 32 heads measured no
  // faster than none)
  int splits = 1;
  if (part && tickets && 4 * groups <= num_sms && groups <= kAttnMaxGroups) {
    splits = (2 * num_sms + groups - 1) / groups;
    if (splits > k_tiles) splits = k_tiles;
    while (splits > 1 && groups * splits > kAttnMaxSplitCtas) --splits;
  }
  const int tps = (k_tiles + splits - 1) / splits;
  splits = (k_tiles + tps - 1) / tps;  // every slice non-empty
  dim3 grid(q_tiles, H, B * splits);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)kAttnHd);
  attention_mma_kernel<<<grid, 128, kAttnSmem, st>>>(
      (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, (__nv_bfloat16*)O, R, L,
      H, scale_log2, splits, tps, part, tickets);
  (*launches)++;
  return cudaGetLastError() != cudaSuccess;
}

}  // namespace esd
