// CUDA-core (SIMT) kernels with float32 accumulation: the exact-float32 path of
// the float32 models (tensor cores have no float32 operand kind). A plain tiled
// GEMM C = A W^T into a float32 workspace, then element-wise epilogues (RoPE +
// K/V scatter, residual add, SwiGLU), and a one-warp-per-(row, head) attention.
#pragma once

#include "common.cuh"

namespace esd {

// ---------------------------------------------------------------------------
// C[m, c_off + n] = sum_k A[m, k] * W[n, k]    (A [M, K] lda, W [N, K] ldw)
// 64x64 tile, BK = 16, 256 threads, 4x4 outputs per thread.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(const T* __restrict__ A, int lda, const T* __restrict__ W, int ldw,
                 float* __restrict__ C, int ldc, int c_off, int M, int N, int K) {
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64 + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  const int lr = tid >> 2;        // tile row loaded by this thread
  const int lk = (tid & 3) * 4;   // 4 consecutive k
  for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int kk = k0 + lk + q;
      const int ma = m0 + lr, nw = n0 + lr;
      As[lk + q][lr] = (ma < M && kk < K) ? Storage<T>::to_f(A[(size_t)ma * lda + kk]) : 0.0f;
      Ws[lk + q][lr] = (nw < N && kk < K) ? Storage<T>::to_f(W[(size_t)nw * ldw + kk]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < N) C[(size_t)m * ldc + c_off + n] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// QKV epilogue: row r (sequence b = r / R, position pos = idx ? idx[r] : r % R),
// scale by inv_rms[r], rotate q and k (pair j, j + hd/2) with the RoPE table,
// write q to Q[r], k and v to Kd/Vd[b*L + pos] (the K/V scatter); a negative
// position marks a padding row, of which nothing is written.
// C holds [R_total, 3d] = [q | k | v]. One thread per (row, head, pair j).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void epi_qkv_kernel(const float* __restrict__ C, const float* __restrict__ inv_rms,
                               const int32_t* __restrict__ idx, const float2* __restrict__ rope,
                               int rows, int R, int L, int H, int hd, T* __restrict__ Q,
                               T* __restrict__ Kd, T* __restrict__ Vd) {
  const int half = hd >> 1;
  const int d = H * hd;
  const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (size_t)rows * H * half) return;
  const int j = t % half;
  const int h = (t / half) % H;
  const int r = t / ((size_t)half * H);
  const int b = r / R;
  const int pos = idx ? idx[r] : r % R;
  if (pos < 0) return;
  const float inv = inv_rms[r];
  const float2 cs = rope[(size_t)pos * half + j];
  const float* c = C + (size_t)r * 3 * d + h * hd;
  const size_t kv_row = (size_t)b * L + pos;
  {
    const float a1 = c[j] * inv, a2 = c[j + half] * inv;
    T* q = Q + (size_t)r * d + h * hd;
    q[j] = Storage<T>::from_f(a1 * cs.x - a2 * cs.y);
    q[j + half] = Storage<T>::from_f(a2 * cs.x + a1 * cs.y);
  }
  {
    const float a1 = c[d + j] * inv, a2 = c[d + j + half] * inv;
    T* k = Kd + kv_row * d + h * hd;
    k[j] = Storage<T>::from_f(a1 * cs.x - a2 * cs.y);
    k[j + half] = Storage<T>::from_f(a2 * cs.x + a1 * cs.y);
  }
  {
    T* v = Vd + kv_row * d + h * hd;
    v[j] = Storage<T>::from_f(c[2 * d + j] * inv);
    v[j + half] = Storage<T>::from_f(c[2 * d + j + half] * inv);
  }
}

// x[r, c] = store(x[r, c] + C[r, c])
template <typename T>
__global__ void epi_residual_kernel(const float* __restrict__ C, T* __restrict__ x, size_t n) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  x[i] = Storage<T>::from_f(Storage<T>::to_f(x[i]) + C[i]);
}

// act[r, j] = store(silu(g) * u), g = inv*C[r, j], u = inv*C[r, F + j]
template <typename T>
__global__ void epi_swiglu_kernel(const float* __restrict__ C, const float* __restrict__ inv_rms,
                                  int rows, int F, T* __restrict__ act) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)rows * F) return;
  const int r = i / F, j = i % F;
  const float inv = inv_rms[r];
  const float g = C[(size_t)r * 2 * F + j] * inv;
  const float u = C[(size_t)r * 2 * F + F + j] * inv;
  act[i] = Storage<T>::from_f(g / (1.0f + expf(-g)) * u);
}

// logits[r, c] = inv_rms[r] * C[r, c]; the mask id column is -inf
__global__ void epi_logits_kernel(float* __restrict__ C, const float* __restrict__ inv_rms,
                                  int rows, int V, int mask_id) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)rows * V) return;
  const int r = i / V, c = i % V;
  C[i] = (c == mask_id) ? -INFINITY : C[i] * inv_rms[r];
}

// ---------------------------------------------------------------------------
// Attention, one warp per (query row r, head h): softmax(q K^T / sqrt(hd)) V over
// the L keys of row r's sequence (b = r / R). Q [rows, d] compact; K, V [B*L, d].
// Dynamic shared memory: per warp hd floats of q plus L floats of scores.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void simt_attention_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                      const T* __restrict__ V, T* __restrict__ O, int rows, int R,
                                      int L, int H, int hd, float scale) {
  extern __shared__ float sm_f32[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int gw = blockIdx.x * (blockDim.x >> 5) + w;
  if (gw >= rows * H) return;
  const int r = gw / H, h = gw % H;
  const int b = r / R;
  const int d = H * hd;
  float* qs = sm_f32 + (size_t)w * (hd + L);
  float* ps = qs + hd;
  for (int i = lane; i < hd; i += 32) qs[i] = Storage<T>::to_f(Q[(size_t)r * d + h * hd + i]);
  __syncwarp();
  const T* Kb = K + (size_t)b * L * d + h * hd;
  const T* Vb = V + (size_t)b * L * d + h * hd;
  float mx = -INFINITY;
  for (int j = lane; j < L; j += 32) {
    const T* kr = Kb + (size_t)j * d;
    float s = 0.0f;
    for (int i = 0; i < hd; ++i) s = fmaf(qs[i], Storage<T>::to_f(kr[i]), s);
    s *= scale;
    ps[j] = s;
    mx = fmaxf(mx, s);
  }
  mx = warp_max(mx);
  float sum = 0.0f;
  for (int j = lane; j < L; j += 32) {
    const float p = expf(ps[j] - mx);
    ps[j] = p;
    sum += p;
  }
  sum = warp_sum(sum);
  __syncwarp();
  const float inv = 1.0f / sum;
  for (int i = lane; i < hd; i += 32) {
    float o = 0.0f;
    for (int j = 0; j < L; ++j) o = fmaf(ps[j], Storage<T>::to_f(Vb[(size_t)j * d + i]), o);
    O[(size_t)r * d + h * hd + i] = Storage<T>::from_f(o * inv);
  }
}

}  // namespace esd
