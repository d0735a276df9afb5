// C ABI of the early-skipping denoising step (declared in include/esd.h):
// context lifetime, argument validation, and the step driver that enqueues the
// kernels of one dense or sparse denoising step on a CUDA stream.
//
// Method: "ES-dLLM: Efficient Inference for Diffusion Large Language Models by
// Early-Skipping" (technical summary sections 1, 2.A, 2.B) and "DyLLM: Efficient
// Diffusion LLM Inference via Saliency-based Token Selection and Partial
// Attention" (technical summary section 2.B.2, partial attention).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <utility>
#include <vector>

#include "esd.h"
#include "common.cuh"
#include "kernels_mem.cuh"
#include "kernels_simt.cuh"
#include "tc_gemm.cuh"
#include "tc_gemm2.cuh"
#include "tc_gemm_cl.cuh"
#include "tc_skinny.cuh"
#include "attention_mma.cuh"
#include "attention_pair.cuh"
#include "approx_attention.cuh"

using esd::HeadPartial;
using esd::StepParams;

namespace {
// vocabulary columns per head partial: the tensor-core head's N tile (bf16),
// or the partial width of the float32 path
constexpr int kHeadTileTc = 128;
constexpr int kHeadTileSimt = 256;
}

// A non-refresh DyLLM call captured as a CUDA graph: every count-dependent
// part (the rows the output projection and SwiGLU block run on, the moved
// rows of the approximate attention) is a conditional switch node whose body
// a kernel of the graph picks from the count on the device, so the call never
// waits for the host.
struct DyGraph {
  std::vector<uint64_t> key;  // layers, x, B, L, path, sim_out, thresholds, context buffers
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  uint64_t launches = 0;  // kernels outside the bodies plus those of the largest body of each switch
};

struct esd_ctx {
  esd_model_dims dims{};
  esd_run_config run{};
  int device = -1;
  size_t esz = 4;  // bytes per stored element
  bool bf16 = false;

  const void* embed = nullptr;
  const void* w_out = nullptr;
  std::vector<const void*> wq, wk, wv, wo, wg, wu, wd;

  // workspaces, [max_batch * max_len] rows
  void* x_full = nullptr;
  void* xs = nullptr;
  void* q = nullptr;
  void* attn = nullptr;
  void* act = nullptr;
  void* k_scr = nullptr;
  void* v_scr = nullptr;
  float* inv_rms = nullptr;
  float* rms_part = nullptr;  // [d / 128][256] partial sums of squares (swapped-operand GEMMs)
  float* c32 = nullptr;     // SIMT GEMM output (float32 models)
  float* logits = nullptr;  // SIMT head logits (float32 models)
  HeadPartial* part = nullptr;
  int n_head_tiles = 0;
  float* scores = nullptr;
  int32_t* idx = nullptr;
  float2* rope = nullptr;

  // block scope (run.scope == ESD_SCOPE_BLOCK)
  int32_t* pos_blk = nullptr;  // [B*R] positions of the block's rows
  int32_t* tok_blk = nullptr;  // [B*R] their tokens

  // second skip point (run.skip_layer2 > 0); h_sel, conf_sel, j2, flat2 also
  // serve the block scope's selection
  void* hc2 = nullptr;      // H cache at the second skip layer [B*L, d]
  void* xs2 = nullptr;      // the rows that go on [B*k2, d]
  void* h_sel = nullptr;    // hc2 rows of the rows that reached it [B*k1, d]
  float* conf_sel = nullptr;
  float* scores2 = nullptr;
  int32_t* j2 = nullptr;    // [B, k2] positions among the k1 rows
  int32_t* idx2 = nullptr;  // [B, k2] positions in [0, L)
  int32_t* flat2 = nullptr; // [B*k2] global rows

  // caches
  void* hc = nullptr;
  std::vector<void*> kc, vc;
  float* conf_c = nullptr;
  int32_t* tok_c = nullptr;

  // generation state
  int32_t* g_tok = nullptr;
  uint8_t* g_masked = nullptr;
  StepParams* params = nullptr;
  int* flag = nullptr;

  esd::TcPlan tc;  // tensor-core GEMM descriptors (bf16 models)

  // DyLLM token-selection layers (allocated by the first esd_dyllm_layers_forward)
  std::vector<void*> dy_ctx[2];  // per layer: the attention contexts of two steps
  std::vector<void*> dy_out;     // per layer: the cached layer outputs
  std::vector<int> dy_cur;       // per layer: the dy_ctx buffer holding the last step
  std::vector<char> dy_valid;    // per layer: filled by a refresh of dy_B x dy_L rows
  int dy_B = 0, dy_L = 0;
  void* dy_xs = nullptr;         // salient rows: inputs, then outputs
  void* dy_cs = nullptr;         // salient rows: contexts
  int32_t* dy_idx = nullptr;     // [B, L] salient positions per sequence
  int32_t* dy_counts = nullptr;  // [n_layers, B] salient rows per layer and sequence (row l*B + b)
  int32_t* dy_total = nullptr;   // [1] salient rows of the current layer, all sequences
  int32_t* dy_flat = nullptr;    // [T] global rows of the salient positions
  float* dy_sim = nullptr;       // [B*L]
  int32_t* dy_cnt_host = nullptr;  // pinned [n_layers * max_batch]
  cudaStream_t dy_cap = nullptr;   // graph capture: the call's static part
  cudaStream_t dy_body = nullptr;  // graph capture: the bodies of its switch nodes
  std::vector<DyGraph> dy_graphs;  // recently used graphs, most recent last
  bool capturing = false;
  // with the approximate attention (esd_dyllm_layers_forward_approx)
  std::vector<void*> dya_in, dya_k, dya_v;  // per layer: last input, K/V of every row
  std::vector<float*> dya_p;               // per layer: [B, H, L, L] cached probabilities
  std::vector<char> dya_valid;             // per layer: filled by an approximate refresh
  void* dya_vprev = nullptr;               // V before this call's update [B*L, d]
  int32_t* dya_mv_idx = nullptr;           // [B, L] moved positions per sequence
  int32_t* dya_mv_cnt = nullptr;           // [B]
  float* dya_flag = nullptr;               // [B*L]
  float* attn_part = nullptr;              // key-split partials of the 64-query attention kernel
  int* attn_tickets = nullptr;
  // bf16 approximate attention scratch (slot form, see approx_tc)
  void* apx_qs = nullptr;                  // [B*L, d] queries of the moved rows
  void* apx_os = nullptr;                  // [B*L, d] their exact contexts
  float2* apx_stat = nullptr;              // [B*L, H] row maximum and sum of the scores

  std::vector<void*> allocs;
  std::string err;
  uint64_t launches = 0;

  // instrumentation (esd_profile_enable)
  int prof_kernel = -1, prof_min = 0, prof_max = 0;
  std::vector<cudaEvent_t> prof_events;  // pairs
  size_t prof_used = 0;
};

namespace {

esd_status fail(esd_ctx* c, esd_status s, const char* fmt, ...) {
  if (c) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    c->err = buf;
  }
  return s;
}

#define ESD_CUDA(ctx, call)                                                                   \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess)                                                                    \
      return fail(ctx, ESD_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                  __FILE__, __LINE__);                                                        \
  } while (0)

#define ESD_LAUNCHED(ctx)                                                                     \
  do {                                                                                        \
    (ctx)->launches++;                                                                        \
    cudaError_t e_ = cudaGetLastError();                                                      \
    if (e_ != cudaSuccess)                                                                    \
      return fail(ctx, ESD_ERR_CUDA, "kernel launch failed: %s (%s:%d)", cudaGetErrorString(e_), \
                  __FILE__, __LINE__);                                                        \
  } while (0)

#define ESD_TRY(expr)               \
  do {                              \
    esd_status s_ = (expr);         \
    if (s_ != ESD_OK) return s_;    \
  } while (0)

// Event pair around one launch of the profiled family (no-op otherwise).
struct ProfScope {
  esd_ctx* c;
  cudaStream_t st;
  bool on = false;
  ProfScope(esd_ctx* c_, int kernel, int rows, cudaStream_t s) : c(c_), st(s) {
    if (c->capturing || c->prof_kernel != kernel || rows < c->prof_min || rows > c->prof_max) return;
    if (c->prof_used + 2 > c->prof_events.size()) {
      cudaEvent_t a, b;
      if (cudaEventCreate(&a) != cudaSuccess) return;
      if (cudaEventCreate(&b) != cudaSuccess) { cudaEventDestroy(a); return; }
      c->prof_events.push_back(a);
      c->prof_events.push_back(b);
    }
    cudaEventRecord(c->prof_events[c->prof_used], st);
    on = true;
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(c->prof_events[c->prof_used + 1], st);
    c->prof_used += 2;
  }
};

inline unsigned cdiv(size_t a, size_t b) { return (unsigned)((a + b - 1) / b); }

// One launch with programmatic dependent launch allowed: the kernel starts
// while its predecessor ends and waits for it (griddepcontrol.wait) before
// touching any data.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename T>
inline T* at(void* base, size_t elem) {
  return reinterpret_cast<T*>(base) + elem;
}

esd_status alloc(esd_ctx* c, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return ESD_OK;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(c, ESD_ERR_OOM, "cudaMalloc(%zu bytes) failed: %s", bytes, cudaGetErrorString(e));
  }
  c->allocs.push_back(*p);
  return ESD_OK;
}

void free_all(esd_ctx* c) {
  for (void* p : c->allocs) cudaFree(p);
  c->allocs.clear();
}

// ceil(ratio * n) clamped to [1, n] (1e-9 absorbs float noise above an integer)
int keep_of(float ratio, int n) {
  double v = std::ceil((double)ratio * (double)n - 1e-9);
  int k = (int)v;
  if (k < 1) k = 1;
  if (k > n) k = n;
  return k;
}

int keep_count(const esd_ctx* c, int L) { return keep_of(c->run.keep_ratio, L); }

// first layer with a K/V cache: the skip layer, or 0 with the block scope
bool region_scope(const esd_ctx* c) { return c->run.scope == ESD_SCOPE_BLOCK || c->run.scope == ESD_SCOPE_RESPONSE; }
int cache_base(const esd_ctx* c) { return region_scope(c) ? 0 : c->run.skip_layer; }

esd_status check_bl(esd_ctx* c, int B, int L) {
  if (B < 1 || B > c->run.max_batch)
    return fail(c, ESD_ERR_INVALID_ARG, "batch %d outside [1, %d]", B, c->run.max_batch);
  if (L < 1 || L > c->run.max_len)
    return fail(c, ESD_ERR_INVALID_ARG, "length %d outside [1, %d]", L, c->run.max_len);
  return ESD_OK;
}

esd_status check_blk(esd_ctx* c, int B, int L, int k) {
  ESD_TRY(check_bl(c, B, L));
  if (k < 1 || k > L) return fail(c, ESD_ERR_INVALID_ARG, "k = %d outside [1, L = %d]", k, L);
  return ESD_OK;
}

// ------------------------------------------------------------------ kernels
template <typename T>
esd_status k_embed(esd_ctx* c, const int32_t* tok, int rows, void* x, cudaStream_t st) {
  esd::embed_kernel<T><<<cdiv(rows, 8), 256, 0, st>>>(tok, (const T*)c->embed, (T*)x, rows,
                                                      c->dims.d, c->dims.vocab, c->flag);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

template <typename T>
esd_status k_rms(esd_ctx* c, const void* x, int rows, cudaStream_t st) {
  esd::rms_kernel<T><<<cdiv(rows, 8), 256, 0, st>>>((const T*)x, c->inv_rms, rows, c->dims.d,
                                                    c->dims.rms_eps);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

// C[:, c_off : c_off + N] = A W^T on CUDA cores (float32 accumulation)
template <typename T>
esd_status k_simt_gemm(esd_ctx* c, const void* A, int lda, const void* W, int ldw, float* C,
                       int ldc, int c_off, int M, int N, int K, cudaStream_t st) {
  dim3 grid(cdiv(N, 64), cdiv(M, 64));
  esd::simt_gemm_kernel<T><<<grid, 256, 0, st>>>((const T*)A, lda, (const T*)W, ldw, C, ldc,
                                                 c_off, M, N, K);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

template <typename T>
esd_status k_attention(esd_ctx* c, const void* Q, const void* K, const void* V, void* O, int rows,
                       int R, int L, cudaStream_t st) {
  const int H = c->dims.n_heads, hd = c->dims.head_dim;
  ProfScope ps(c, ESD_K_ATTENTION, rows, st);
  if constexpr (sizeof(T) == 2) {
    const int B = rows / R;
    // SM pairs of 256 queries, the keys split over the pairs of a cluster
    // when the pair-tiles leave SMs idle; up to 64 queries per sequence the
    // 64-query mma.sync kernel (a pair-tile would be three quarters empty:
    // 64 queries x 4096 keys x 16 x 32 heads measured 277 against 412 us)
    const int err = R <= esd::kAttnQ ? esd::attention_mma_launch(Q, K, V, O, B, R, L, H, c->tc.num_sms, c->attn_part,
                                                                 c->attn_tickets, st, &c->launches)
                                     : esd::attention_pair_launch(c->tc, Q, K, V, O, B, R, L, H, st, &c->launches);
    return err ? fail(c, ESD_ERR_CUDA, "attention launch failed: %s", cudaGetErrorString(cudaGetLastError()))
               : ESD_OK;
  } else {
    const size_t smem = (size_t)4 * (hd + L) * sizeof(float);
    esd::simt_attention_kernel<T><<<cdiv((size_t)rows * H, 4), 128, smem, st>>>(
        (const T*)Q, (const T*)K, (const T*)V, (T*)O, rows, R, L, H, hd, 1.0f / sqrtf((float)hd));
    ESD_LAUNCHED(c);
    return ESD_OK;
  }
}

// RMS statistic and Q/K/V with RoPE of X [B*R, d] at positions idx ([B*R],
// or r % R when null): Q into the workspace, K/V into kd/vd [B*L, d] (the
// layer's cache or the workspace).
// Whether the swapped-operand GEMM (tc_skinny.cuh) takes the layer GEMMs of
// `rows` rows: its residual epilogues then also emit the RMS statistic of the
// rows they update, as partial sums of squares in c->rms_part.
bool skinny_rows(const esd_ctx* c, int rows) { return c->bf16 && esd::tc_skinny_ok(c->tc, rows); }

// RMS statistic and Q/K/V with RoPE of X [B*R, d] at positions idx ([B*R],
// or r % R when null): Q into the workspace, K/V into kd/vd [B*L, d] (the
// layer's cache or the workspace). rms_ready: the previous residual epilogue
// left X's statistic in c->rms_part (swapped-operand GEMMs only).
template <typename T>
esd_status layer_qkv(esd_ctx* c, int layer, const int32_t* idx, int B, int R, int L, void* X, void* kd,
                     void* vd, cudaStream_t st, bool rms_ready = false) {
  const esd_model_dims& m = c->dims;
  const int d = m.d, rows = B * R;
  const bool fused = skinny_rows(c, rows);
  if (!fused) {
    ESD_TRY(k_rms<T>(c, X, rows, st));
  } else if (!rms_ready) {
    // the statistic in the residual epilogues' partial form (same bits)
    esd::rms_part_kernel<<<cdiv((size_t)rows * (d / 128), 256), 256, 0, st>>>((const __nv_bfloat16*)X, rows, d,
                                                                           c->rms_part);
    ESD_LAUNCHED(c);
  }
  if constexpr (sizeof(T) == 2) {
    esd::EpiArgs ea{};
    ea.inv_rms = c->inv_rms;
    if (fused) {
      ea.rms_part_in = c->rms_part;
      ea.rms_parts = d / 128;
      ea.rms_eps = m.rms_eps;
      ea.inv_out = c->inv_rms;
    }
    ea.idx = idx;
    ea.rope = c->rope;
    ea.R = R;
    ea.L = L;
    ea.out = c->q;
    ea.k_dst = kd;
    ea.v_dst = vd;
    {
      ProfScope ps(c, ESD_K_GEMM_QKV, rows, st);
      ESD_TRY(esd::tc_gemm(c->tc, esd::kEpiQKV, layer, X, rows, ea, st, &c->launches, &c->err));
    }
  } else {
    float* C = c->c32;
    ESD_TRY(k_simt_gemm<T>(c, X, d, c->wq[layer], d, C, 3 * d, 0, rows, d, d, st));
    ESD_TRY(k_simt_gemm<T>(c, X, d, c->wk[layer], d, C, 3 * d, d, rows, d, d, st));
    ESD_TRY(k_simt_gemm<T>(c, X, d, c->wv[layer], d, C, 3 * d, 2 * d, rows, d, d, st));
    const size_t nq = (size_t)rows * m.n_heads * (m.head_dim / 2);
    esd::epi_qkv_kernel<T><<<cdiv(nq, 256), 256, 0, st>>>(C, c->inv_rms, idx, c->rope, rows, R, L,
                                                         m.n_heads, m.head_dim, (T*)c->q, (T*)kd,
                                                         (T*)vd);
    ESD_LAUNCHED(c);
  }
  return ESD_OK;
}

// First half of a layer on X [B*R, d]: layer_qkv, then the attention of the
// B*R queries over the B*L keys into A [B*R, d].
template <typename T>
esd_status layer_attention_half(esd_ctx* c, int layer, const int32_t* idx, int B, int R, int L, void* X,
                                void* kd, void* vd, void* A, cudaStream_t st, bool rms_ready = false) {
  ESD_TRY(layer_qkv<T>(c, layer, idx, B, R, L, X, kd, vd, st, rms_ready));
  return k_attention<T>(c, c->q, kd, vd, A, B * R, R, L, st);
}

// Second half of a layer on `rows` rows: X += A Wo^T, then
// X += SwiGLU(RMSNorm(X)) Wd^T. With the swapped-operand GEMMs the O
// epilogue leaves the statistic the SwiGLU GEMM needs, and the down epilogue
// the one of the next layer's QKV (then *rms_next = true).
template <typename T>
esd_status layer_mlp_half(esd_ctx* c, int layer, const void* A, int rows, void* X, cudaStream_t st,
                          bool* rms_next = nullptr) {
  const esd_model_dims& m = c->dims;
  const int d = m.d, F = m.ffn;
  if (rms_next) *rms_next = false;
  if constexpr (sizeof(T) == 2) {
    const bool fused = skinny_rows(c, rows);
    esd::EpiArgs ea{};
    ea.out = X;
    if (fused) ea.rms_part_out = c->rms_part;
    {
      ProfScope ps(c, ESD_K_GEMM_O, rows, st);
      ESD_TRY(esd::tc_gemm(c->tc, esd::kEpiResidualO, layer, A, rows, ea, st, &c->launches, &c->err));
    }
    if (!fused) ESD_TRY(k_rms<T>(c, X, rows, st));
    ea = esd::EpiArgs{};
    ea.inv_rms = c->inv_rms;
    if (fused) {
      ea.rms_part_in = c->rms_part;
      ea.rms_parts = d / 128;
      ea.rms_eps = m.rms_eps;
      ea.inv_out = c->inv_rms;
    }
    ea.out = c->act;
    {
      ProfScope ps(c, ESD_K_GEMM_GATE_UP, rows, st);
      ESD_TRY(esd::tc_gemm(c->tc, esd::kEpiSwiGLU, layer, X, rows, ea, st, &c->launches, &c->err));
    }
    ea = esd::EpiArgs{};
    ea.out = X;
    if (fused) ea.rms_part_out = c->rms_part;
    {
      ProfScope ps(c, ESD_K_GEMM_DOWN, rows, st);
      ESD_TRY(esd::tc_gemm(c->tc, esd::kEpiResidualD, layer, c->act, rows, ea, st, &c->launches,
                           &c->err));
    }
    if (rms_next) *rms_next = fused;
  } else {
    float* C = c->c32;
    ESD_TRY(k_simt_gemm<T>(c, A, d, c->wo[layer], d, C, d, 0, rows, d, d, st));
    esd::epi_residual_kernel<T><<<cdiv((size_t)rows * d, 256), 256, 0, st>>>(C, (T*)X,
                                                                            (size_t)rows * d);
    ESD_LAUNCHED(c);
    ESD_TRY(k_rms<T>(c, X, rows, st));
    ESD_TRY(k_simt_gemm<T>(c, X, d, c->wg[layer], d, C, 2 * F, 0, rows, F, d, st));
    ESD_TRY(k_simt_gemm<T>(c, X, d, c->wu[layer], d, C, 2 * F, F, rows, F, d, st));
    esd::epi_swiglu_kernel<T><<<cdiv((size_t)rows * F, 256), 256, 0, st>>>(C, c->inv_rms, rows, F,
                                                                          (T*)c->act);
    ESD_LAUNCHED(c);
    ESD_TRY(k_simt_gemm<T>(c, c->act, F, c->wd[layer], F, C, d, 0, rows, d, F, st));
    esd::epi_residual_kernel<T><<<cdiv((size_t)rows * d, 256), 256, 0, st>>>(C, (T*)X,
                                                                            (size_t)rows * d);
    ESD_LAUNCHED(c);
  }
  return ESD_OK;
}

// One layer on X [B*R, d]: positions idx ([B*R], or r % R when null), K/V
// destination kd/vd [B*L, d] (the layer's cache or the workspace).
template <typename T>
esd_status layer_forward(esd_ctx* c, int layer, const int32_t* idx, int B, int R, int L, void* X,
                         void* kd, void* vd, cudaStream_t st, bool rms_ready, bool* rms_next) {
  ESD_TRY(layer_attention_half<T>(c, layer, idx, B, R, L, X, kd, vd, c->attn, st, rms_ready));
  return layer_mlp_half<T>(c, layer, c->attn, B * R, X, st, rms_next);
}

template <typename T>
esd_status layers_forward(esd_ctx* c, int l0, int l1, const int32_t* idx, int B, int R, int L,
                          void* X, cudaStream_t st) {
  const int base = cache_base(c);
  bool rms_ready = false;  // X's statistic is computed afresh for the first layer
  for (int l = l0; l < l1; ++l) {
    void* kd = l >= base ? c->kc[l - base] : c->k_scr;
    void* vd = l >= base ? c->vc[l - base] : c->v_scr;
    ESD_TRY(layer_forward<T>(c, l, idx, B, R, L, X, kd, vd, st, rms_ready, &rms_ready));
  }
  return ESD_OK;
}

// Head: final RMS statistic, logits, per-tile partials, reduction.
template <typename T>
esd_status head_forward(esd_ctx* c, const void* X, int rows, const int32_t* idx, int L, int k,
                        float* conf, int32_t* tok, cudaStream_t st) {
  const esd_model_dims& m = c->dims;
  ESD_TRY(k_rms<T>(c, X, rows, st));
  if constexpr (sizeof(T) == 2) {
    esd::EpiArgs ea{};
    ea.inv_rms = c->inv_rms;
    ea.part = c->part;
    ea.n_tiles = c->n_head_tiles;
    ProfScope ps(c, ESD_K_HEAD, rows, st);
    ESD_TRY(esd::tc_gemm(c->tc, esd::kEpiHead, 0, X, rows, ea, st, &c->launches, &c->err));
  } else {
    ESD_TRY(k_simt_gemm<T>(c, X, m.d, c->w_out, m.d, c->logits, m.vocab, 0, rows, m.vocab, m.d, st));
    esd::epi_logits_kernel<<<cdiv((size_t)rows * m.vocab, 256), 256, 0, st>>>(
        c->logits, c->inv_rms, rows, m.vocab, m.mask_id);
    ESD_LAUNCHED(c);
    esd::head_partials_from_logits<<<cdiv((size_t)rows * c->n_head_tiles, 8), 256, 0, st>>>(
        c->logits, rows, m.vocab, kHeadTileSimt, c->n_head_tiles, m.mask_id, c->part);
    ESD_LAUNCHED(c);
  }
  esd::head_finalize_kernel<<<cdiv(rows, 8), 256, 0, st>>>(c->part, rows, c->n_head_tiles, idx, L,
                                                          k, conf, tok);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

template <typename T>
esd_status logits_forward(esd_ctx* c, const void* X, int rows, float* out, cudaStream_t st) {
  const esd_model_dims& m = c->dims;
  ESD_TRY(k_rms<T>(c, X, rows, st));
  if constexpr (sizeof(T) == 2) {
    esd::EpiArgs ea{};
    ea.inv_rms = c->inv_rms;
    ea.out = out;
    ESD_TRY(esd::tc_gemm(c->tc, esd::kEpiLogits, 0, X, rows, ea, st, &c->launches, &c->err));
  } else {
    ESD_TRY(k_simt_gemm<T>(c, X, m.d, c->w_out, m.d, out, m.vocab, 0, rows, m.vocab, m.d, st));
    esd::epi_logits_kernel<<<cdiv((size_t)rows * m.vocab, 256), 256, 0, st>>>(
        out, c->inv_rms, rows, m.vocab, m.mask_id);
    ESD_LAUNCHED(c);
  }
  return ESD_OK;
}

esd_status k_score_select(esd_ctx* c, const void* x, const void* h, const float* conf, int B,
                          int L, int k, float* scores, int32_t* idx, cudaStream_t st) {
  const int rows = B * L, d = c->dims.d;
  const unsigned g = cdiv(rows, 8);
  ProfScope ps(c, ESD_K_SCORE_SELECT, rows, st);
  const bool cos_mode = c->run.score_mode == ESD_SCORE_COS;
  const float coef = cos_mode ? c->run.lambda_ : c->run.alpha;
  if (c->bf16) {
    using T = __nv_bfloat16;
    if (cos_mode)
      esd::score_kernel<T, 1><<<g, 256, 0, st>>>((const T*)x, (const T*)h, conf, scores, rows, d, coef);
    else
      esd::score_kernel<T, 0><<<g, 256, 0, st>>>((const T*)x, (const T*)h, conf, scores, rows, d, coef);
  } else {
    if (cos_mode)
      esd::score_kernel<float, 1><<<g, 256, 0, st>>>((const float*)x, (const float*)h, conf, scores,
                                                     rows, d, coef);
    else
      esd::score_kernel<float, 0><<<g, 256, 0, st>>>((const float*)x, (const float*)h, conf, scores,
                                                     rows, d, coef);
  }
  ESD_LAUNCHED(c);
  esd::topk_kernel<<<B, esd::kTopkThreads, (size_t)L * sizeof(uint32_t), st>>>(scores, L, k, idx);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

esd_status k_gather(esd_ctx* c, const void* x, const int32_t* idx, int B, int L, int k, void* xs,
                    void* hc, cudaStream_t st) {
  const int rows = B * k;
  if (c->bf16)
    esd::gather_kernel<__nv_bfloat16><<<cdiv(rows, 8), 256, 0, st>>>(
        (const __nv_bfloat16*)x, idx, L, k, rows, c->dims.d, (__nv_bfloat16*)xs,
        (__nv_bfloat16*)hc, c->flag);
  else
    esd::gather_kernel<float><<<cdiv(rows, 8), 256, 0, st>>>((const float*)x, idx, L, k, rows,
                                                            c->dims.d, (float*)xs, (float*)hc,
                                                            c->flag);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

esd_status k_remask(esd_ctx* c, int32_t* tok, uint8_t* masked, const float* conf,
                    const int32_t* tok_c, int B, int L, int b0, int b1, int n,
                    const StepParams* params, cudaStream_t st) {
  esd::remask_kernel<<<B, 256, 0, st>>>(tok, masked, conf, tok_c, L, b0, b1, n, params);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

template <typename T>
esd_status step_impl(esd_ctx* c, int32_t* tok, uint8_t* masked, int B, int L, int r0, int r1, int b0, int b1,
                     int n, bool dense, const StepParams* params, cudaStream_t st) {
  const esd_model_dims& m = c->dims;
  const int ls = c->run.skip_layer;
  const size_t rowb = (size_t)m.d * c->esz;
  const int ls2 = c->run.skip_layer2 > 0 ? c->run.skip_layer2 : m.n_layers;
  ESD_TRY(k_embed<T>(c, tok, B * L, c->x_full, st));
  if (dense) {
    ESD_TRY(layers_forward<T>(c, 0, ls, nullptr, B, L, L, c->x_full, st));
    ESD_CUDA(c, cudaMemcpyAsync(c->hc, c->x_full, (size_t)B * L * rowb, cudaMemcpyDeviceToDevice, st));
    ESD_TRY(layers_forward<T>(c, ls, ls2, nullptr, B, L, L, c->x_full, st));
    if (ls2 < m.n_layers) {
      ESD_CUDA(c, cudaMemcpyAsync(c->hc2, c->x_full, (size_t)B * L * rowb, cudaMemcpyDeviceToDevice, st));
      ESD_TRY(layers_forward<T>(c, ls2, m.n_layers, nullptr, B, L, L, c->x_full, st));
    }
    ESD_TRY(head_forward<T>(c, c->x_full, B * L, nullptr, L, L, c->conf_c, c->tok_c, st));
  } else if (region_scope(c)) {
    // S = the region [r0, r1) (the block, or the response after the prompt):
    // every layer recomputes only its rows, attending over every layer's K/V
    // cache with the region's fresh K/V scattered in
    const int R = r1 - r0, rows = B * R;
    const int k = keep_of(c->run.keep_ratio, R);
    esd::block_rows_kernel<<<cdiv(rows, 256), 256, 0, st>>>(tok, L, r0, R, rows, c->pos_blk, c->tok_blk);
    ESD_LAUNCHED(c);
    ESD_TRY(k_embed<T>(c, c->tok_blk, rows, c->x_full, st));
    ESD_TRY(layers_forward<T>(c, 0, ls, c->pos_blk, B, R, L, c->x_full, st));
    esd::gather_kernel<T><<<cdiv(rows, 8), 256, 0, st>>>((const T*)c->hc, c->pos_blk, L, R, rows, m.d,
                                                         (T*)c->h_sel, nullptr, c->flag);
    ESD_LAUNCHED(c);
    esd::gather_conf_kernel<<<cdiv(rows, 256), 256, 0, st>>>(c->conf_c, c->pos_blk, L, R, rows, c->conf_sel);
    ESD_LAUNCHED(c);
    ESD_TRY(k_score_select(c, c->x_full, c->h_sel, c->conf_sel, B, R, k, c->scores, c->j2, st));
    const int rk = B * k;
    esd::compose_idx_kernel<<<cdiv(rk, 256), 256, 0, st>>>(c->pos_blk, c->j2, L, R, k, rk, c->idx, c->flat2);
    ESD_LAUNCHED(c);
    esd::gather_kernel<T><<<cdiv(rk, 8), 256, 0, st>>>((const T*)c->x_full, c->j2, R, k, rk, m.d, (T*)c->xs,
                                                       nullptr, c->flag);
    ESD_LAUNCHED(c);
    esd::copy_rows_kernel<T><<<cdiv(rk, 8), 256, 0, st>>>((T*)c->hc, c->flat2, (const T*)c->xs, nullptr, rk, m.d);
    ESD_LAUNCHED(c);
    ESD_TRY(layers_forward<T>(c, ls, m.n_layers, c->idx, B, k, L, c->xs, st));
    ESD_TRY(head_forward<T>(c, c->xs, rk, c->idx, L, k, c->conf_c, c->tok_c, st));
  } else {
    const int k = keep_count(c, L);
    ESD_TRY(layers_forward<T>(c, 0, ls, nullptr, B, L, L, c->x_full, st));
    if (c->run.score_tensor == ESD_SCORE_ON_H) {
      ESD_TRY(k_score_select(c, c->x_full, c->hc, c->conf_c, B, L, k, c->scores, c->idx, st));
    } else {
      // the skip layer's keys and values of every row, against its K/V cache
      ESD_TRY(layer_qkv<T>(c, ls, nullptr, B, L, L, c->x_full, c->k_scr, c->v_scr, st));
      const bool on_k = c->run.score_tensor == ESD_SCORE_ON_K;
      ESD_TRY(k_score_select(c, on_k ? c->k_scr : c->v_scr, on_k ? c->kc[ls - cache_base(c)] : c->vc[ls - cache_base(c)],
                             c->conf_c, B, L, k, c->scores, c->idx, st));
    }
    ESD_TRY(k_gather(c, c->x_full, c->idx, B, L, k, c->xs, c->hc, st));
    ESD_TRY(layers_forward<T>(c, ls, ls2, c->idx, B, k, L, c->xs, st));
    void* xf = c->xs;
    const int32_t* idxf = c->idx;
    int kf = k;
    if (ls2 < m.n_layers) {
      // the k rows that reached the second skip point: scored against its H
      // cache and the cached confidence, the top k2 per sequence go on
      const int k2 = keep_of(c->run.keep_ratio2, k);
      const int r1 = B * k, r2 = B * k2;
      esd::gather_kernel<T><<<cdiv(r1, 8), 256, 0, st>>>((const T*)c->hc2, c->idx, L, k, r1, m.d, (T*)c->h_sel,
                                                         nullptr, c->flag);
      ESD_LAUNCHED(c);
      esd::gather_conf_kernel<<<cdiv(r1, 256), 256, 0, st>>>(c->conf_c, c->idx, L, k, r1, c->conf_sel);
      ESD_LAUNCHED(c);
      ESD_TRY(k_score_select(c, c->xs, c->h_sel, c->conf_sel, B, k, k2, c->scores2, c->j2, st));
      esd::compose_idx_kernel<<<cdiv(r2, 256), 256, 0, st>>>(c->idx, c->j2, L, k, k2, r2, c->idx2, c->flat2);
      ESD_LAUNCHED(c);
      esd::gather_kernel<T><<<cdiv(r2, 8), 256, 0, st>>>((const T*)c->xs, c->j2, k, k2, r2, m.d, (T*)c->xs2,
                                                         nullptr, c->flag);
      ESD_LAUNCHED(c);
      esd::copy_rows_kernel<T><<<cdiv(r2, 8), 256, 0, st>>>((T*)c->hc2, c->flat2, (const T*)c->xs2, nullptr, r2,
                                                            m.d);
      ESD_LAUNCHED(c);
      xf = c->xs2;
      idxf = c->idx2;
      kf = k2;
    }
    ESD_TRY(layers_forward<T>(c, ls2, m.n_layers, idxf, B, kf, L, xf, st));
    ESD_TRY(head_forward<T>(c, xf, B * kf, idxf, L, kf, c->conf_c, c->tok_c, st));
  }
  return k_remask(c, tok, masked, c->conf_c, c->tok_c, B, L, b0, b1, n, params, st);
}

esd_status step(esd_ctx* c, int32_t* tok, uint8_t* masked, int B, int L, int r0, int r1, int b0, int b1,
                int n, bool dense, const StepParams* params, cudaStream_t st) {
  if (c->bf16)
    return step_impl<__nv_bfloat16>(c, tok, masked, B, L, r0, r1, b0, b1, n, dense, params, st);
  return step_impl<float>(c, tok, masked, B, L, r0, r1, b0, b1, n, dense, params, st);
}

// Failure-path self-test: one thread waits, through the same bounded wait as
// the GEMM and attention kernels, on a barrier phase that nothing completes;
// after `polls` polls it records the timeout on the context's flag and returns.
__global__ void selftest_wait_kernel(uint32_t polls, int* flag) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    esd::mbar_init(esd::smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) esd::mbar_wait(esd::smem_u32(&bar), 0u, &abort_flag, flag, polls);
}

__global__ void init_generation_kernel(int32_t* tok, uint8_t* masked, int B, int L, int P,
                                       int mask_id) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)B * L) return;
  const int p = i % L;
  if (p >= P) tok[i] = mask_id;
  masked[i] = p >= P ? 1 : 0;
}

esd_status read_flag(esd_ctx* c, cudaStream_t st) {
  ESD_CUDA(c, cudaStreamSynchronize(st));
  int f = 0;
  ESD_CUDA(c, cudaMemcpy(&f, c->flag, sizeof(int), cudaMemcpyDeviceToHost));
  if (f != 0) {
    ESD_CUDA(c, cudaMemset(c->flag, 0, sizeof(int)));
    if (f == esd::kFlagTimeout) return fail(c, ESD_ERR_TIMEOUT, "a device-side wait timed out");
    return fail(c, ESD_ERR_CHECK, "a device-side check failed (code %d)", f);
  }
  return ESD_OK;
}

}  // namespace

// =========================================================================
// C ABI
// =========================================================================
namespace {

esd_status dy_alloc(esd_ctx* c) {
  if (!c->dy_out.empty()) return ESD_OK;
  const int n = c->dims.n_layers;
  const size_t rows = (size_t)c->run.max_batch * c->run.max_len, row_bytes = (size_t)c->dims.d * c->esz;
  for (int i = 0; i < 2; ++i) c->dy_ctx[i].assign(n, nullptr);
  c->dy_out.assign(n, nullptr);
  for (int l = 0; l < n; ++l)
    for (void** p : {&c->dy_ctx[0][l], &c->dy_ctx[1][l], &c->dy_out[l]}) ESD_TRY(alloc(c, p, rows * row_bytes));
  ESD_TRY(alloc(c, &c->dy_xs, rows * row_bytes));
  ESD_TRY(alloc(c, &c->dy_cs, rows * row_bytes));
  ESD_TRY(alloc(c, (void**)&c->dy_idx, rows * sizeof(int32_t)));
  ESD_TRY(alloc(c, (void**)&c->dy_flat, rows * sizeof(int32_t)));
  const size_t nc = (size_t)n * c->run.max_batch;
  ESD_TRY(alloc(c, (void**)&c->dy_counts, nc * sizeof(int32_t)));
  ESD_TRY(alloc(c, (void**)&c->dy_total, sizeof(int32_t)));
  ESD_TRY(alloc(c, (void**)&c->dy_sim, rows * sizeof(float)));
  // the rows past a layer's salient count, which the GEMMs of its capacity
  // read, start finite
  ESD_CUDA(c, cudaMemset(c->dy_xs, 0, rows * row_bytes));
  ESD_CUDA(c, cudaMemset(c->dy_cs, 0, rows * row_bytes));
  ESD_CUDA(c, cudaMallocHost((void**)&c->dy_cnt_host, nc * sizeof(int32_t)));
  ESD_CUDA(c, cudaStreamCreateWithFlags(&c->dy_cap, cudaStreamNonBlocking));
  ESD_CUDA(c, cudaStreamCreateWithFlags(&c->dy_body, cudaStreamNonBlocking));
  c->dy_cur.assign(n, 0);
  c->dy_valid.assign(n, 0);
  return ESD_OK;
}

template <typename T>
esd_status k_copy_rows(esd_ctx* c, void* dst, const int32_t* dmap, const void* src, const int32_t* smap, int n,
                       cudaStream_t st, const int32_t* n_dev = nullptr) {
  esd::copy_rows_kernel<T><<<cdiv(n, 8), 256, 0, st>>>((T*)dst, dmap, (const T*)src, smap, n, c->dims.d, n_dev);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

// Row capacities of the switch bodies for a count in [1, max_rows]: every 16
// rows up to 256 (the swapped-operand GEMMs take their token tile in steps of
// 16), every 256 up to 2048 (the SM-pair tiles), then steps of about a
// quarter; the last capacity is max_rows.
esd::BucketCaps bucket_caps(int max_rows) {
  esd::BucketCaps bc{};
  for (int v = 16; v < max_rows && bc.n < esd::kMaxBuckets - 1;) {
    bc.cap[bc.n++] = v;
    v = v < 256 ? v + 16 : (v < 2048 ? v + 256 : (v + v / 4 + 255) / 256 * 256);
  }
  bc.cap[bc.n++] = max_rows;
  return bc;
}

// A conditional handle of the graph being captured on c->dy_cap; `none`, the
// value at each launch until a kernel of the graph sets it.
esd_status cap_handle(esd_ctx* c, unsigned none, cudaGraphConditionalHandle* h) {
  cudaStreamCaptureStatus cs;
  cudaGraph_t g = nullptr;
  ESD_CUDA(c, cudaStreamGetCaptureInfo(c->dy_cap, &cs, nullptr, &g, nullptr, nullptr));
  if (cs != cudaStreamCaptureStatusActive || !g) return fail(c, ESD_ERR_CUDA, "graph capture not active");
  ESD_CUDA(c, cudaGraphConditionalHandleCreate(h, g, none, cudaGraphCondAssignDefault));
  return ESD_OK;
}

// A switch node on handle h with n bodies, after everything captured so far
// on c->dy_cap; body(k) enqueues body k on c->dy_body, which captures into it.
// *extra grows by the launches of every body but the largest.
template <class F>
esd_status cap_switch(esd_ctx* c, cudaGraphConditionalHandle h, int n, F&& body, uint64_t* extra) {
  cudaStreamCaptureStatus cs;
  cudaGraph_t g = nullptr;
  const cudaGraphNode_t* deps = nullptr;
  const cudaGraphEdgeData* edges = nullptr;
  size_t nd = 0;
  ESD_CUDA(c, cudaStreamGetCaptureInfo_v3(c->dy_cap, &cs, nullptr, &g, &deps, &edges, &nd));
  if (cs != cudaStreamCaptureStatusActive || !g) return fail(c, ESD_ERR_CUDA, "graph capture not active");
  cudaGraphNodeParams np = {cudaGraphNodeTypeConditional};  // the rest zero
  np.conditional.handle = h;
  np.conditional.type = cudaGraphCondTypeSwitch;
  np.conditional.size = (unsigned)n;
  cudaGraphNode_t node;
  ESD_CUDA(c, cudaGraphAddNode_v2(&node, g, deps, edges, nd, &np));
  std::vector<cudaGraph_t> bodies(np.conditional.phGraph_out, np.conditional.phGraph_out + n);
  ESD_CUDA(c, cudaStreamUpdateCaptureDependencies(c->dy_cap, &node, 1, cudaStreamSetCaptureDependencies));
  uint64_t sum = 0, most = 0;
  for (int k = 0; k < n; ++k) {
    ESD_CUDA(c, cudaStreamBeginCaptureToGraph(c->dy_body, bodies[k], nullptr, nullptr, 0,
                                              cudaStreamCaptureModeThreadLocal));
    const uint64_t before = c->launches;
    const esd_status st = body(k);
    cudaGraph_t bg = nullptr;
    const cudaError_t e = cudaStreamEndCapture(c->dy_body, &bg);
    if (st != ESD_OK) return st;
    ESD_CUDA(c, e);
    sum += c->launches - before;
    most = std::max(most, c->launches - before);
  }
  *extra += sum - most;
  return ESD_OK;
}

esd_status dya_alloc(esd_ctx* c) {
  if (!c->dya_p.empty()) return ESD_OK;
  const int n = c->dims.n_layers;
  const size_t rows = (size_t)c->run.max_batch * c->run.max_len, row_bytes = (size_t)c->dims.d * c->esz;
  const size_t pf = (size_t)c->run.max_batch * c->dims.n_heads * c->run.max_len * c->run.max_len;
  c->dya_in.assign(n, nullptr);
  c->dya_k.assign(n, nullptr);
  c->dya_v.assign(n, nullptr);
  c->dya_p.assign(n, nullptr);
  for (int l = 0; l < n; ++l) {
    for (void** q : {&c->dya_in[l], &c->dya_k[l], &c->dya_v[l]}) {
      ESD_TRY(alloc(c, q, rows * row_bytes));
      ESD_CUDA(c, cudaMemset(*q, 0, rows * row_bytes));
    }
    ESD_TRY(alloc(c, (void**)&c->dya_p[l], pf * sizeof(float)));
    ESD_CUDA(c, cudaMemset(c->dya_p[l], 0, pf * sizeof(float)));
  }
  ESD_TRY(alloc(c, &c->dya_vprev, rows * row_bytes));
  ESD_TRY(alloc(c, (void**)&c->dya_mv_idx, rows * sizeof(int32_t)));
  ESD_TRY(alloc(c, (void**)&c->dya_mv_cnt, (size_t)c->run.max_batch * sizeof(int32_t)));
  ESD_TRY(alloc(c, (void**)&c->dya_flag, rows * sizeof(float)));
  c->dya_valid.assign(n, 0);
  return ESD_OK;
}

esd_status apx_alloc(esd_ctx* c) {
  if (c->apx_qs) return ESD_OK;
  const size_t rows = (size_t)c->run.max_batch * c->run.max_len, row_bytes = (size_t)c->dims.d * c->esz;
  ESD_TRY(alloc(c, &c->apx_qs, rows * row_bytes));
  ESD_CUDA(c, cudaMemset(c->apx_qs, 0, rows * row_bytes));  // rows past the moved ones stay finite
  ESD_TRY(alloc(c, &c->apx_os, rows * row_bytes));
  ESD_TRY(alloc(c, (void**)&c->apx_stat, rows * c->dims.n_heads * sizeof(float2)));
  return ESD_OK;
}

// The bf16 approximate attention of one layer on tensor cores, with no host
// synchronisation; the moved rows of sequence b are slots a < cnt[b] with
// positions idx[b*L + a] (ascending). In order on the stream:
//   update (optional): c_out_i = c_in_i + sum_a P[i, idx_a] (V - V_prev)[idx_a]
//     for every row i (V_prev row b*L + a if vprev_slots, else by position);
//   the moved rows' queries in slot form, rpad rows per sequence (given so,
//   or gathered from q; rpad 0: L);
//   their exact attention over all L keys on the SM-pair kernel (slot form
//   output; rpad, the largest moved count when the host knows it, sizes its
//   grid and key split), which also reports each moved row's maximum and sum
//   of its scores; the P rows 2^(score - max) / sum from the scores
//   recomputed on tensor cores; the contexts scattered into c_out at their
//   positions.
// Without the update every row must be a moved row (a refresh).
esd_status approx_tc(esd_ctx* c, const void* q, bool q_slots, const void* k, const void* v, const void* v_prev,
                     bool vprev_slots, const int32_t* idx, const int32_t* cnt, int B, int L, const void* c_in,
                     void* c_out, float* p, bool update, cudaStream_t st, int rpad = 0) {
  using T = __nv_bfloat16;
  ESD_TRY(apx_alloc(c));
  const int H = c->dims.n_heads, d = c->dims.d;
  if (update) {
    ESD_CUDA(c, launch_pdl(esd::approx_update_mma_kernel, dim3(cdiv(L, esd::kAuRows), H, B), dim3(128), st, p,
                           (const T*)v, (const T*)v_prev, vprev_slots ? 1 : 0, idx, cnt, L, H, (const T*)c_in,
                           (T*)c_out, c->flag));
    ESD_LAUNCHED(c);
  }
  const int R = rpad > 0 ? rpad : L;
  const void* qs = q;
  if (!q_slots) {
    ESD_CUDA(c, launch_pdl(esd::slot_rows_kernel<false>, dim3(R, B), dim3(128), st, (T*)c->apx_qs, (const T*)q, idx,
                           cnt, L, R, d, c->flag));
    ESD_LAUNCHED(c);
    qs = c->apx_qs;
  }
  if (esd::attention_pair_launch(c->tc, qs, k, v, c->apx_os, B, R, L, H, st, &c->launches, idx, c->apx_stat, cnt,
                                 L))
    return fail(c, ESD_ERR_CUDA, "attention launch failed: %s", cudaGetErrorString(cudaGetLastError()));
  const float scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c->dims.head_dim));
  // the key tiles split so that the grid fills the SMs about twice
  const int rt = (int)cdiv(R, esd::kPrRows), ntiles = (int)cdiv(L, esd::kPrKeys);
  int ks = (int)cdiv((size_t)2 * c->tc.num_sms, (size_t)rt * H * B);
  ks = std::max(1, std::min(std::min(ks, ntiles), 65535 / std::max(B, 1)));
  ESD_CUDA(c, launch_pdl(esd::prob_rows_mma_kernel, dim3(rt, H, B * ks), dim3(128), st, (const T*)qs, (const T*)k,
                         idx, cnt, (const float2*)c->apx_stat, p, R, L, H, scale_log2, ks, c->flag));
  ESD_LAUNCHED(c);
  ESD_CUDA(c, launch_pdl(esd::slot_rows_kernel<true>, dim3(R, B), dim3(128), st, (T*)c_out, (const T*)c->apx_os,
                         idx, cnt, L, R, d, c->flag));
  ESD_LAUNCHED(c);
  return ESD_OK;
}

// Contexts of layer l with the saliency-aware approximate attention into
// `cur` (prev: the contexts of the layer's previous call): the moved rows are
// the rows whose input differs bit for bit from the layer's previous input
// (all on a refresh). bf16: Q/K/V of the moved rows only (one GEMM per
// sequence on its gathered rows; an unmoved row's input and so its cached K/V
// are unchanged), V before the update kept in slot form, and approx_tc
// (tensor cores). Outside a refresh this runs inside a graph capture: a
// switch node sized by the largest moved count of a sequence (or copying the
// contexts when nothing moved) holds everything sized by it. float32: Q/K/V of
// every row (the unmoved rows' K/V repeat bit for bit) and the SIMT kernels of
// esd_approx_attention.
template <typename T>
esd_status dya_contexts(esd_ctx* c, int l, void* x, int B, int L, bool refresh, void* prev, void* cur,
                        cudaStream_t st, uint64_t* extra = nullptr) {
  const int rows = B * L, d = c->dims.d;
  const size_t bytes = (size_t)rows * d * c->esz;
  if (refresh) {
    ESD_CUDA(c, cudaMemsetAsync(c->dya_flag, 0, rows * sizeof(float), st));
  } else {
    esd::row_changed_kernel<T><<<cdiv(rows, 8), 256, 0, st>>>((const T*)x, (const T*)c->dya_in[l], rows, d,
                                                               c->dya_flag);
    ESD_LAUNCHED(c);
  }
  esd::compact_below_kernel<<<B, esd::kCompactThreads, 0, st>>>(c->dya_flag, L, 0.5f, c->dya_mv_idx, c->dya_mv_cnt);
  ESD_LAUNCHED(c);
  if constexpr (sizeof(T) == 2) {
    const size_t row_bytes = (size_t)d * c->esz;
    if (refresh) {
      // every row moves: Q/K/V of all rows (slot a = position a)
      ESD_CUDA(c, cudaMemcpyAsync(c->dya_in[l], x, bytes, cudaMemcpyDeviceToDevice, st));
      ESD_TRY(layer_qkv<T>(c, l, nullptr, B, L, L, x, c->dya_k[l], c->dya_v[l], st));
      return approx_tc(c, c->q, true, c->dya_k[l], c->dya_v[l], nullptr, false, c->dya_mv_idx, c->dya_mv_cnt, B, L,
                       nullptr, cur, c->dya_p[l], false, st);
    }
    if (!c->capturing || st != c->dy_cap) return fail(c, ESD_ERR_CUDA, "approximate contexts outside a capture");
    // switch value 0: nothing moved, every context stays; 1 + k: capacity k
    const esd::BucketCaps caps = bucket_caps(L);
    cudaGraphConditionalHandle h;
    ESD_TRY(cap_handle(c, 0u, &h));
    esd::select_bucket_kernel<<<1, 32, 0, st>>>(c->dya_mv_cnt, B, 1, caps, 1u, 0u, h, nullptr);
    ESD_LAUNCHED(c);
    auto body = [&](int k) -> esd_status {
      const cudaStream_t bs = c->dy_body;
      if (k == 0) {
        ESD_CUDA(c, cudaMemcpyAsync(cur, prev, bytes, cudaMemcpyDeviceToDevice, bs));
        return ESD_OK;
      }
      // R slots per sequence, R at least every sequence's moved count
      const int R = caps.cap[k - 1];
      ESD_CUDA(c, cudaMemcpyAsync(c->dya_in[l], x, bytes, cudaMemcpyDeviceToDevice, bs));
      // V of the moved rows before their update, and their inputs, in slot form
      esd::slot_rows_kernel<false><<<dim3(R, B), 128, 0, bs>>>((T*)c->dya_vprev, (const T*)c->dya_v[l],
                                                               c->dya_mv_idx, c->dya_mv_cnt, L, L, d, c->flag);
      ESD_LAUNCHED(c);
      esd::slot_rows_kernel<false><<<dim3(R, B), 128, 0, bs>>>((T*)c->dy_xs, (const T*)x, c->dya_mv_idx,
                                                               c->dya_mv_cnt, L, L, d, c->flag);
      ESD_LAUNCHED(c);
      // Q/K/V of R slots per sequence: the slots past its count have position
      // -1 (compact_below_kernel), so the epilogue writes nothing of them
      for (int b = 0; b < B; ++b) {
        const size_t off = (size_t)b * L * row_bytes;
        ESD_TRY(layer_qkv<T>(c, l, c->dya_mv_idx + (size_t)b * L, 1, R, L, (char*)c->dy_xs + off,
                             (char*)c->dya_k[l] + off, (char*)c->dya_v[l] + off, bs));
        ESD_CUDA(c, cudaMemcpyAsync((char*)c->apx_qs + (size_t)b * R * row_bytes, c->q, (size_t)R * row_bytes,
                                    cudaMemcpyDeviceToDevice, bs));
      }
      return approx_tc(c, c->apx_qs, true, c->dya_k[l], c->dya_v[l], c->dya_vprev, true, c->dya_mv_idx,
                       c->dya_mv_cnt, B, L, prev, cur, c->dya_p[l], true, bs, R);
    };
    return cap_switch(c, h, caps.n + 1, body, extra);
  } else {
    ESD_CUDA(c, cudaMemcpyAsync(c->dya_in[l], x, bytes, cudaMemcpyDeviceToDevice, st));
    ESD_CUDA(c, cudaMemcpyAsync(c->dya_vprev, c->dya_v[l], bytes, cudaMemcpyDeviceToDevice, st));
    ESD_TRY(layer_qkv<T>(c, l, nullptr, B, L, L, x, c->dya_k[l], c->dya_v[l], st));
    ESD_CUDA(c, cudaMemcpyAsync(cur, prev, bytes, cudaMemcpyDeviceToDevice, st));
    const int H = c->dims.n_heads, hd = c->dims.head_dim;
    const dim3 grid(cdiv(L, esd::kApxRows), H, B);
    const float scale = (float)(1.0 / std::sqrt((double)hd));
    esd::approx_update_kernel<T><<<grid, esd::kApxThreads, 0, st>>>(
        (const T*)c->dya_v[l], (const T*)c->dya_vprev, c->dya_p[l], c->dya_mv_idx, c->dya_mv_cnt, L, H, hd, (T*)cur,
        c->flag);
    ESD_LAUNCHED(c);
    esd::approx_exact_rows_kernel<T><<<grid, esd::kApxThreads, 0, st>>>(
        (const T*)c->q, (const T*)c->dya_k[l], (const T*)c->dya_v[l], c->dya_mv_idx, c->dya_mv_cnt, L, H, hd, scale,
        (T*)cur, c->dya_p[l], c->flag);
    ESD_LAUNCHED(c);
    return ESD_OK;
  }
}

// The layers [l0, l1) of a non-refresh DyLLM call, enqueued on c->dy_cap
// while it captures a graph. Per layer: the contexts (exact, or approximate
// with their own switch), the similarities and the salient rows; then a
// switch node on the total salient count whose body of capacity R gathers the
// salient rows' inputs and contexts (rows past the count are left as they
// are: every kernel works per row, and their results are never copied back),
// runs the output projection and the SwiGLU block on R rows and scatters the
// salient rows' outputs into the layer's output cache; then the cache into x.
template <typename T>
esd_status dy_capture_layers(esd_ctx* c, int l0, int l1, void* x, int B, int L, const float* tau, float* sim_out,
                             bool approx, uint64_t* extra) {
  const cudaStream_t st = c->dy_cap;
  const int rows = B * L, d = c->dims.d;
  const size_t bytes = (size_t)rows * d * c->esz;
  const esd::BucketCaps caps = bucket_caps(rows);
  for (int l = l0; l < l1; ++l) {
    void* prev = c->dy_ctx[c->dy_cur[l]][l];
    void* cur = c->dy_ctx[1 - c->dy_cur[l]][l];
    if (approx) {
      ESD_TRY(dya_contexts<T>(c, l, x, B, L, false, prev, cur, st, extra));
    } else {
      // every row's context, exactly
      ESD_TRY(layer_attention_half<T>(c, l, nullptr, B, L, L, x, c->k_scr, c->v_scr, cur, st));
    }
    float* sim = sim_out ? sim_out + (size_t)(l - l0) * rows : c->dy_sim;
    int32_t* cnt = c->dy_counts + (size_t)l * B;
    esd::context_sim_kernel<T><<<cdiv(rows, 8), 256, 0, st>>>((const T*)cur, (const T*)prev, sim, rows, d);
    ESD_LAUNCHED(c);
    esd::compact_below_kernel<<<B, esd::kCompactThreads, 0, st>>>(sim, L, tau[l - l0], c->dy_idx, cnt);
    ESD_LAUNCHED(c);
    esd::flatten_rows_kernel<<<B, 256, 0, st>>>(c->dy_idx, cnt, L, c->dy_flat);
    ESD_LAUNCHED(c);
    cudaGraphConditionalHandle h;
    ESD_TRY(cap_handle(c, (unsigned)caps.n, &h));
    esd::select_bucket_kernel<<<1, 32, 0, st>>>(cnt, B, 0, caps, 0u, (unsigned)caps.n, h, c->dy_total);
    ESD_LAUNCHED(c);
    auto body = [&](int k) -> esd_status {
      const cudaStream_t bs = c->dy_body;
      const int R = caps.cap[k];
      ESD_TRY(k_copy_rows<T>(c, c->dy_xs, nullptr, x, c->dy_flat, R, bs, c->dy_total));
      ESD_TRY(k_copy_rows<T>(c, c->dy_cs, nullptr, cur, c->dy_flat, R, bs, c->dy_total));
      ESD_TRY(layer_mlp_half<T>(c, l, c->dy_cs, R, c->dy_xs, bs));
      return k_copy_rows<T>(c, c->dy_out[l], c->dy_flat, c->dy_xs, nullptr, R, bs, c->dy_total);
    };
    ESD_TRY(cap_switch(c, h, caps.n, body, extra));
    ESD_CUDA(c, cudaMemcpyAsync(x, c->dy_out[l], bytes, cudaMemcpyDeviceToDevice, st));
  }
  return ESD_OK;
}

// The graph of a non-refresh call: from the cache when the same call (layers,
// x, shape, path, sim_out, thresholds and context buffers) ran recently, else
// captured and instantiated (the oldest of 8 cached graphs goes).
template <typename T>
esd_status dy_graph(esd_ctx* c, int l0, int l1, void* x, int B, int L, const float* tau, float* sim_out,
                    bool approx, DyGraph** out) {
  std::vector<uint64_t> key = {(uint64_t)l0, (uint64_t)l1, (uint64_t)(uintptr_t)x, (uint64_t)B, (uint64_t)L,
                               approx ? 1u : 0u, (uint64_t)(uintptr_t)sim_out};
  for (int l = l0; l < l1; ++l) {
    uint32_t bits;
    std::memcpy(&bits, &tau[l - l0], sizeof(bits));
    key.push_back(((uint64_t)bits << 1) | (uint64_t)c->dy_cur[l]);
  }
  for (size_t i = 0; i < c->dy_graphs.size(); ++i)
    if (c->dy_graphs[i].key == key) {
      std::rotate(c->dy_graphs.begin() + i, c->dy_graphs.begin() + i + 1, c->dy_graphs.end());
      *out = &c->dy_graphs.back();
      return ESD_OK;
    }
  const uint64_t launches0 = c->launches;
  uint64_t extra = 0;
  ESD_CUDA(c, cudaStreamBeginCapture(c->dy_cap, cudaStreamCaptureModeThreadLocal));
  c->capturing = true;
  const esd_status s = dy_capture_layers<T>(c, l0, l1, x, B, L, tau, sim_out, approx, &extra);
  c->capturing = false;
  cudaGraph_t g = nullptr;
  const cudaError_t e = cudaStreamEndCapture(c->dy_cap, &g);
  const uint64_t launched = c->launches - launches0 - extra;
  c->launches = launches0;
  if (s != ESD_OK || e != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return s != ESD_OK ? s : fail(c, ESD_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(e));
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t ei = cudaGraphInstantiate(&exec, g, 0);
  if (ei != cudaSuccess) {
    cudaGraphDestroy(g);
    return fail(c, ESD_ERR_CUDA, "graph instantiation failed: %s", cudaGetErrorString(ei));
  }
  if (c->dy_graphs.size() >= 8) {
    cudaGraphExecDestroy(c->dy_graphs.front().exec);
    cudaGraphDestroy(c->dy_graphs.front().graph);
    c->dy_graphs.erase(c->dy_graphs.begin());
  }
  DyGraph dg;
  dg.key = std::move(key);
  dg.graph = g;
  dg.exec = exec;
  dg.launches = launched;
  c->dy_graphs.push_back(std::move(dg));
  *out = &c->dy_graphs.back();
  return ESD_OK;
}

// counts_out [(l1 - l0) * B] from the per-layer counts: device memory by an
// asynchronous copy, host memory after a synchronisation of the stream.
esd_status dy_counts_out(esd_ctx* c, int l0, int l1, int B, int32_t* counts_out, cudaStream_t st) {
  if (!counts_out) return ESD_OK;
  const size_t n = (size_t)(l1 - l0) * B;
  const int32_t* src = c->dy_counts + (size_t)l0 * B;
  cudaPointerAttributes a{};
  const bool dev = cudaPointerGetAttributes(&a, counts_out) == cudaSuccess &&
                   (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged);
  cudaGetLastError();
  if (dev) {
    ESD_CUDA(c, cudaMemcpyAsync(counts_out, src, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
    return ESD_OK;
  }
  ESD_CUDA(c, cudaMemcpyAsync(c->dy_cnt_host, src, n * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  ESD_CUDA(c, cudaStreamSynchronize(st));
  std::memcpy(counts_out, c->dy_cnt_host, n * sizeof(int32_t));
  return ESD_OK;
}

template <typename T>
esd_status dyllm_layers(esd_ctx* c, int l0, int l1, void* x, int B, int L, const float* tau, bool refresh,
                        int32_t* counts_out, float* sim_out, cudaStream_t st, bool approx = false) {
  const int rows = B * L;
  const size_t bytes = (size_t)rows * c->dims.d * c->esz;
  if (refresh) {
    for (int l = l0; l < l1; ++l) {
      void* prev = c->dy_ctx[c->dy_cur[l]][l];
      void* cur = c->dy_ctx[1 - c->dy_cur[l]][l];
      if (approx)
        ESD_TRY(dya_contexts<T>(c, l, x, B, L, true, prev, cur, st));
      else
        ESD_TRY(layer_attention_half<T>(c, l, nullptr, B, L, L, x, c->k_scr, c->v_scr, cur, st));
      ESD_TRY(layer_mlp_half<T>(c, l, cur, rows, x, st));
      ESD_CUDA(c, cudaMemcpyAsync(c->dy_out[l], x, bytes, cudaMemcpyDeviceToDevice, st));
      c->dy_cur[l] = 1 - c->dy_cur[l];
    }
    const int n = (l1 - l0) * B;
    esd::fill_i32_kernel<<<cdiv(n, 256), 256, 0, st>>>(c->dy_counts + (size_t)l0 * B, n, L);
    ESD_LAUNCHED(c);
    for (int l = l0; l < l1; ++l) (approx ? c->dya_valid : c->dy_valid)[l] = 1;
  } else {
    DyGraph* g = nullptr;
    ESD_TRY(dy_graph<T>(c, l0, l1, x, B, L, tau, sim_out, approx, &g));
    ESD_CUDA(c, cudaGraphLaunch(g->exec, st));
    c->launches += g->launches;
    for (int l = l0; l < l1; ++l) c->dy_cur[l] = 1 - c->dy_cur[l];
  }
  return dy_counts_out(c, l0, l1, B, counts_out, st);
}

}  // namespace

extern "C" {

esd_status esd_create(const esd_model_dims* dims, const esd_weights* w, const esd_run_config* run,
                      esd_ctx** out) {
  if (!out) return ESD_ERR_INVALID_ARG;
  *out = nullptr;
  if (!dims || !w || !run) return ESD_ERR_INVALID_ARG;
  const esd_model_dims& m = *dims;
  if (m.n_layers < 2 || m.d < 8 || m.n_heads < 1 || m.head_dim < 2 || m.ffn < 8 || m.vocab < 2)
    return ESD_ERR_INVALID_ARG;
  if (m.d != m.n_heads * m.head_dim || (m.head_dim & 1) || m.d % 8 || m.ffn % 8)
    return ESD_ERR_INVALID_ARG;
  if (m.mask_id < 0 || m.mask_id >= m.vocab || !(m.rms_eps >= 0.0f) || !(m.rope_theta > 0.0f))
    return ESD_ERR_INVALID_ARG;
  if (m.dtype != ESD_DTYPE_F32 && m.dtype != ESD_DTYPE_BF16) return ESD_ERR_INVALID_ARG;
  if (run->skip_layer < 1 || run->skip_layer >= m.n_layers) return ESD_ERR_INVALID_ARG;
  if (!(run->keep_ratio > 0.0f && run->keep_ratio <= 1.0f)) return ESD_ERR_INVALID_ARG;
  if (run->score_tensor < ESD_SCORE_ON_H || run->score_tensor > ESD_SCORE_ON_V) return ESD_ERR_INVALID_ARG;
  if (run->scope != ESD_SCOPE_ALL && run->scope != ESD_SCOPE_BLOCK && run->scope != ESD_SCOPE_RESPONSE)
    return ESD_ERR_INVALID_ARG;
  if (run->scope != ESD_SCOPE_ALL && (run->score_tensor != ESD_SCORE_ON_H || run->skip_layer2 != 0))
    return ESD_ERR_UNSUPPORTED;
  if (run->skip_layer2 != 0 && (run->skip_layer2 <= run->skip_layer || run->skip_layer2 >= m.n_layers ||
                                !(run->keep_ratio2 > 0.0f && run->keep_ratio2 <= 1.0f)))
    return ESD_ERR_INVALID_ARG;
  if (run->score_mode != ESD_SCORE_ES && run->score_mode != ESD_SCORE_COS) return ESD_ERR_INVALID_ARG;
  if (run->refresh_interval < 0 || run->max_batch < 1 || run->max_len < 1) return ESD_ERR_INVALID_ARG;
  if (!w->embed || !w->w_out || !w->wq || !w->wk || !w->wv || !w->wo || !w->wg || !w->wu || !w->wd)
    return ESD_ERR_INVALID_ARG;
  for (int l = 0; l < m.n_layers; ++l)
    if (!w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->wg[l] || !w->wu[l] || !w->wd[l])
      return ESD_ERR_INVALID_ARG;
  if (m.dtype == ESD_DTYPE_BF16) {
    if (m.head_dim != 128 || m.d % 128 || m.ffn % 128) return ESD_ERR_UNSUPPORTED;
  } else {
    if (m.head_dim > 128) return ESD_ERR_UNSUPPORTED;
    if ((size_t)4 * (m.head_dim + run->max_len) * sizeof(float) > 200 * 1024) return ESD_ERR_UNSUPPORTED;
  }
  if (run->max_len > 65536) return ESD_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ESD_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ESD_ERR_CUDA;
  if (prop.major != 10) return ESD_ERR_UNSUPPORTED;

  esd_ctx* c = new esd_ctx();
  c->dims = m;
  c->run = *run;
  c->device = dev;
  c->bf16 = m.dtype == ESD_DTYPE_BF16;
  c->esz = c->bf16 ? 2 : 4;
  c->embed = w->embed;
  c->w_out = w->w_out;
  for (int l = 0; l < m.n_layers; ++l) {
    c->wq.push_back(w->wq[l]);
    c->wk.push_back(w->wk[l]);
    c->wv.push_back(w->wv[l]);
    c->wo.push_back(w->wo[l]);
    c->wg.push_back(w->wg[l]);
    c->wu.push_back(w->wu[l]);
    c->wd.push_back(w->wd[l]);
  }
  const size_t rows = (size_t)run->max_batch * run->max_len;
  const size_t rb = (size_t)m.d * c->esz;
  const int nc = m.n_layers - (run->scope != ESD_SCOPE_ALL ? 0 : run->skip_layer);
  const int head_tile = c->bf16 ? kHeadTileTc : kHeadTileSimt;
  c->n_head_tiles = (m.vocab + head_tile - 1) / head_tile;
  esd_status s = ESD_OK;
  auto A = [&](void** p, size_t bytes) {
    if (s == ESD_OK) s = alloc(c, p, bytes);
  };
  A(&c->x_full, rows * rb);
  A(&c->xs, rows * rb);
  A(&c->q, rows * rb);
  A(&c->attn, rows * rb);
  A(&c->act, rows * (size_t)m.ffn * c->esz);
  A(&c->k_scr, rows * rb);
  A(&c->v_scr, rows * rb);
  A((void**)&c->inv_rms, rows * sizeof(float));
  A((void**)&c->rms_part, (size_t)(m.d / 128 + 1) * esd::kSkMaxRows * sizeof(float));
  A((void**)&c->part, rows * (size_t)c->n_head_tiles * sizeof(HeadPartial));
  A((void**)&c->scores, rows * sizeof(float));
  A((void**)&c->idx, rows * sizeof(int32_t));
  A((void**)&c->rope, (size_t)run->max_len * (m.head_dim / 2) * sizeof(float2));
  A(&c->hc, rows * rb);
  if (run->skip_layer2 > 0) {
    A(&c->hc2, rows * rb);
    A(&c->xs2, rows * rb);
    A((void**)&c->scores2, rows * sizeof(float));
    A((void**)&c->idx2, rows * sizeof(int32_t));
  }
  if (run->skip_layer2 > 0 || run->scope != ESD_SCOPE_ALL) {
    A(&c->h_sel, rows * rb);
    A((void**)&c->conf_sel, rows * sizeof(float));
    A((void**)&c->j2, rows * sizeof(int32_t));
    A((void**)&c->flat2, rows * sizeof(int32_t));
  }
  if (run->scope != ESD_SCOPE_ALL) {
    A((void**)&c->pos_blk, rows * sizeof(int32_t));
    A((void**)&c->tok_blk, rows * sizeof(int32_t));
  }
  c->kc.assign(nc, nullptr);
  c->vc.assign(nc, nullptr);
  for (int i = 0; i < nc; ++i) {
    A(&c->kc[i], rows * rb);
    A(&c->vc[i], rows * rb);
  }
  A((void**)&c->conf_c, rows * sizeof(float));
  A((void**)&c->tok_c, rows * sizeof(int32_t));
  A((void**)&c->g_tok, rows * sizeof(int32_t));
  A((void**)&c->g_masked, rows);
  A((void**)&c->params, sizeof(StepParams));
  A((void**)&c->flag, sizeof(int));
  if (!c->bf16) {
    const size_t wide = std::max<size_t>(3 * (size_t)m.d, 2 * (size_t)m.ffn);
    A((void**)&c->c32, rows * wide * sizeof(float));
    A((void**)&c->logits, rows * (size_t)m.vocab * sizeof(float));
  }
  if (s != ESD_OK) {
    free_all(c);
    delete c;
    return s;
  }
  cudaMemset(c->flag, 0, sizeof(int));
  cudaMemset(c->hc, 0, rows * rb);
  cudaMemset(c->conf_c, 0, rows * sizeof(float));
  cudaMemset(c->tok_c, 0, rows * sizeof(int32_t));
  const int half = m.head_dim / 2;
  esd::rope_table_kernel<<<cdiv((size_t)run->max_len * half, 256), 256>>>(c->rope, run->max_len, half,
                                                                         (double)m.rope_theta);
  c->launches++;
  if (!c->bf16) {
    const int smem = 4 * (m.head_dim + run->max_len) * (int)sizeof(float);
    cudaFuncSetAttribute(esd::simt_attention_kernel<float>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  } else {
    esd::TcWeights tw{};
    tw.d = m.d;
    tw.ffn = m.ffn;
    tw.vocab = m.vocab;
    tw.mask_id = m.mask_id;
    tw.n_heads = m.n_heads;
    tw.n_layers = m.n_layers;
    tw.w_out = w->w_out;
    tw.wq = c->wq.data();
    tw.wk = c->wk.data();
    tw.wv = c->wv.data();
    tw.wo = c->wo.data();
    tw.wg = c->wg.data();
    tw.wu = c->wu.data();
    tw.wd = c->wd.data();
    std::string e;
    esd_status ts = esd::tc_plan_create(&c->tc, tw, &e, c->flag);
    esd::tc2_set_attr_all();
    esd::tc_skinny_set_attr_all();
    esd::tc_cl_init(c->tc);
    if (ts == ESD_OK) {
      // split-K partials of the small-M GEMMs
      c->tc.max_tiles = esd::tc_max_units(c->tc.num_sms);
      c->tc.ws_floats = esd::tc_workspace_floats(c->tc.num_sms);
      ts = alloc(c, (void**)&c->tc.ws, c->tc.ws_floats * sizeof(float));
    }
    if (ts != ESD_OK) {
      free_all(c);
      delete c;
      return ts;
    }
    if (alloc(c, (void**)&c->attn_part, esd::attention_ws_floats() * sizeof(float)) != ESD_OK ||
        alloc(c, (void**)&c->attn_tickets, esd::kAttnMaxGroups * sizeof(int)) != ESD_OK) {
      free_all(c);
      delete c;
      return ESD_ERR_OOM;
    }
    cudaMemset(c->attn_tickets, 0, esd::kAttnMaxGroups * sizeof(int));
    if (esd::attention_mma_setup() || esd::attention_pair_setup(&c->tc)) {
      free_all(c);
      delete c;
      return ESD_ERR_CUDA;
    }
  }
  if (cudaDeviceSynchronize() != cudaSuccess) {
    free_all(c);
    delete c;
    return ESD_ERR_CUDA;
  }
  *out = c;
  return ESD_OK;
}

esd_status esd_destroy(esd_ctx* c) {
  if (!c) return ESD_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  if (c->dy_cnt_host) cudaFreeHost(c->dy_cnt_host);
  for (DyGraph& g : c->dy_graphs) {
    cudaGraphExecDestroy(g.exec);
    cudaGraphDestroy(g.graph);
  }
  if (c->dy_cap) cudaStreamDestroy(c->dy_cap);
  if (c->dy_body) cudaStreamDestroy(c->dy_body);
  for (cudaEvent_t e : c->prof_events) cudaEventDestroy(e);
  free_all(c);
  delete c;
  return ESD_OK;
}

const char* esd_last_error(const esd_ctx* c) { return c ? c->err.c_str() : "null context"; }

int esd_keep_count(const esd_ctx* c, int L) {
  if (!c || L < 1) return 0;
  return keep_count(c, L);
}

uint64_t esd_launch_count(const esd_ctx* c) { return c ? c->launches : 0; }

esd_status esd_state(esd_ctx* c, esd_state_view* out) {
  if (!c || !out) return ESD_ERR_INVALID_ARG;
  out->h_cache = c->hc;
  out->k_cache = c->kc.data();
  out->v_cache = c->vc.data();
  out->conf_cache = c->conf_c;
  out->tok_cache = c->tok_c;
  out->n_cached_layers = (int)c->kc.size();
  out->max_batch = c->run.max_batch;
  out->max_len = c->run.max_len;
  return ESD_OK;
}

esd_status esd_embed(esd_ctx* c, const int32_t* tok, int B, int L, void* x, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_bl(c, B, L));
  if (!tok || !x) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = (cudaStream_t)stream;
  return c->bf16 ? k_embed<__nv_bfloat16>(c, tok, B * L, x, st) : k_embed<float>(c, tok, B * L, x, st);
}

esd_status esd_importance_select(esd_ctx* c, const void* x, const void* h, const float* conf,
                                 int B, int L, int k, float* scores_out, int32_t* idx_out,
                                 void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_blk(c, B, L, k));
  if (!x || !h || !conf || !idx_out) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  float* sc = scores_out ? scores_out : c->scores;
  return k_score_select(c, x, h, conf, B, L, k, sc, idx_out, (cudaStream_t)stream);
}

esd_status esd_context_saliency(esd_ctx* c, const void* cur, const void* prev, int B, int L, float tau,
                                float* sim_out, int32_t* idx_out, int32_t* count_out, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_bl(c, B, L));
  if (!cur || !prev || !idx_out || !count_out) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = (cudaStream_t)stream;
  float* sim = sim_out ? sim_out : c->scores;
  const int rows = B * L, d = c->dims.d;
  if (c->bf16) {
    using T = __nv_bfloat16;
    esd::context_sim_kernel<T><<<cdiv(rows, 8), 256, 0, st>>>((const T*)cur, (const T*)prev, sim, rows, d);
  } else {
    esd::context_sim_kernel<float><<<cdiv(rows, 8), 256, 0, st>>>((const float*)cur, (const float*)prev, sim,
                                                                 rows, d);
  }
  ESD_LAUNCHED(c);
  esd::compact_below_kernel<<<B, esd::kCompactThreads, 0, st>>>(sim, L, tau, idx_out, count_out);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

esd_status esd_approx_attention(esd_ctx* c, const void* q, const void* k, const void* v, const void* v_prev,
                                const int32_t* changed_idx, const int32_t* changed_count, int B, int L,
                                void* ctx_io, float* p, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_bl(c, B, L));
  if (!q || !k || !v || !v_prev || !changed_idx || !changed_count || !ctx_io || !p)
    return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  const int H = c->dims.n_heads, hd = c->dims.head_dim;
  if (hd > esd::kApxMaxHd) return fail(c, ESD_ERR_UNSUPPORTED, "head_dim %d above %d", hd, esd::kApxMaxHd);
  if (H > 65535 || B > 65535) return fail(c, ESD_ERR_UNSUPPORTED, "grid limits");
  cudaStream_t st = (cudaStream_t)stream;
  const dim3 grid(cdiv(L, esd::kApxRows), H, B);
  const float scale = (float)(1.0 / std::sqrt((double)hd));
  if (c->bf16) {
    // tensor cores: the update, then the moved rows exactly (in place)
    return approx_tc(c, q, false, k, v, v_prev, false, changed_idx, changed_count, B, L, ctx_io, ctx_io, p, true,
                     st);
  } else {
    esd::approx_update_kernel<float><<<grid, esd::kApxThreads, 0, st>>>(
        (const float*)v, (const float*)v_prev, p, changed_idx, changed_count, L, H, hd, (float*)ctx_io, c->flag);
    ESD_LAUNCHED(c);
    esd::approx_exact_rows_kernel<float><<<grid, esd::kApxThreads, 0, st>>>(
        (const float*)q, (const float*)k, (const float*)v, changed_idx, changed_count, L, H, hd, scale,
        (float*)ctx_io, p, c->flag);
  }
  ESD_LAUNCHED(c);
  return ESD_OK;
}

esd_status esd_dyllm_layers_forward(esd_ctx* c, int l0, int l1, void* x, int B, int L, const float* tau,
                                    int refresh, int32_t* counts_out, float* sim_out, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_bl(c, B, L));
  if (!x || (!refresh && !tau)) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  if (l0 < 0 || l1 > c->dims.n_layers || l0 >= l1)
    return fail(c, ESD_ERR_INVALID_ARG, "layers [%d, %d) outside [0, %d)", l0, l1, c->dims.n_layers);
  ESD_TRY(dy_alloc(c));
  if (refresh) {
    c->dy_B = B;
    c->dy_L = L;
  } else {
    if (B != c->dy_B || L != c->dy_L)
      return fail(c, ESD_ERR_INVALID_ARG, "batch %d x length %d differ from the refresh (%d x %d)", B, L, c->dy_B,
                  c->dy_L);
    for (int l = l0; l < l1; ++l)
      if (!c->dy_valid[l]) return fail(c, ESD_ERR_INVALID_ARG, "layer %d has no refresh yet", l);
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (c->bf16) return dyllm_layers<__nv_bfloat16>(c, l0, l1, x, B, L, tau, refresh != 0, counts_out, sim_out, st);
  return dyllm_layers<float>(c, l0, l1, x, B, L, tau, refresh != 0, counts_out, sim_out, st);
}

esd_status esd_dyllm_layers_forward_approx(esd_ctx* c, int l0, int l1, void* x, int B, int L, const float* tau,
                                           int refresh, int32_t* counts_out, float* sim_out, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_bl(c, B, L));
  if (!x || (!refresh && !tau)) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  if (l0 < 0 || l1 > c->dims.n_layers || l0 >= l1)
    return fail(c, ESD_ERR_INVALID_ARG, "layers [%d, %d) outside [0, %d)", l0, l1, c->dims.n_layers);
  if (c->dims.head_dim > esd::kApxMaxHd)
    return fail(c, ESD_ERR_UNSUPPORTED, "head_dim %d above %d", c->dims.head_dim, esd::kApxMaxHd);
  ESD_TRY(dy_alloc(c));
  ESD_TRY(dya_alloc(c));
  if (c->bf16) ESD_TRY(apx_alloc(c));  // before any capture: a capture allocates nothing
  if (refresh) {
    c->dy_B = B;
    c->dy_L = L;
  } else {
    if (B != c->dy_B || L != c->dy_L)
      return fail(c, ESD_ERR_INVALID_ARG, "batch %d x length %d differ from the refresh (%d x %d)", B, L, c->dy_B,
                  c->dy_L);
    for (int l = l0; l < l1; ++l)
      if (!c->dya_valid[l]) return fail(c, ESD_ERR_INVALID_ARG, "layer %d has no approximate refresh yet", l);
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (c->bf16)
    return dyllm_layers<__nv_bfloat16>(c, l0, l1, x, B, L, tau, refresh != 0, counts_out, sim_out, st, true);
  return dyllm_layers<float>(c, l0, l1, x, B, L, tau, refresh != 0, counts_out, sim_out, st, true);
}

esd_status esd_topk_select(esd_ctx* c, const float* scores, int B, int L, int k, int32_t* idx_out,
                           void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_blk(c, B, L, k));
  if (!scores || !idx_out) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  esd::topk_kernel<<<B, esd::kTopkThreads, (size_t)L * sizeof(uint32_t), (cudaStream_t)stream>>>(
      scores, L, k, idx_out);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

esd_status esd_gather_rows(esd_ctx* c, const void* x, const int32_t* idx, int B, int L, int k,
                           void* x_sel, void* h_cache, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_blk(c, B, L, k));
  if (!x || !idx || !x_sel) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  return k_gather(c, x, idx, B, L, k, x_sel, h_cache, (cudaStream_t)stream);
}

esd_status esd_sparse_layers_forward(esd_ctx* c, int l0, int l1, const int32_t* idx, int B, int L,
                                     int k, void* x_sel, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_blk(c, B, L, k));
  if (!x_sel) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  if (l0 < 0 || l1 > c->dims.n_layers || l0 >= l1)
    return fail(c, ESD_ERR_INVALID_ARG, "layer range [%d, %d) invalid", l0, l1);
  if (idx && l0 < c->run.skip_layer)
    return fail(c, ESD_ERR_INVALID_ARG, "selected rows need layer_begin >= skip_layer (%d)",
                c->run.skip_layer);
  if (!idx && k != L) return fail(c, ESD_ERR_INVALID_ARG, "dense call (idx NULL) needs k == L");
  cudaStream_t st = (cudaStream_t)stream;
  if (c->bf16) return layers_forward<__nv_bfloat16>(c, l0, l1, idx, B, k, L, x_sel, st);
  return layers_forward<float>(c, l0, l1, idx, B, k, L, x_sel, st);
}

esd_status esd_partial_attention(esd_ctx* c, const void* q, const void* kc, const void* vc, int B,
                                 int L, int k, void* out, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_blk(c, B, L, k));
  if (!q || !kc || !vc || !out) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = (cudaStream_t)stream;
  if (c->bf16) return k_attention<__nv_bfloat16>(c, q, kc, vc, out, B * k, k, L, st);
  return k_attention<float>(c, q, kc, vc, out, B * k, k, L, st);
}

esd_status esd_confidence_argmax(esd_ctx* c, const void* x_rows, const int32_t* idx, int B, int L,
                                 int k, float* conf_out, int32_t* tok_out, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_blk(c, B, L, k));
  if (!x_rows || !conf_out || !tok_out) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = (cudaStream_t)stream;
  if (c->bf16) return head_forward<__nv_bfloat16>(c, x_rows, B * k, idx, L, k, conf_out, tok_out, st);
  return head_forward<float>(c, x_rows, B * k, idx, L, k, conf_out, tok_out, st);
}

esd_status esd_logits(esd_ctx* c, const void* x_rows, int rows, float* logits_out, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  if (rows < 1 || (size_t)rows > (size_t)c->run.max_batch * c->run.max_len)
    return fail(c, ESD_ERR_INVALID_ARG, "rows %d out of range", rows);
  if (!x_rows || !logits_out) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = (cudaStream_t)stream;
  if (c->bf16) return logits_forward<__nv_bfloat16>(c, x_rows, rows, logits_out, st);
  return logits_forward<float>(c, x_rows, rows, logits_out, st);
}

esd_status esd_remask(esd_ctx* c, int32_t* tok, uint8_t* masked, const float* conf,
                      const int32_t* tok_c, int B, int L, int b0, int b1, int n, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_bl(c, B, L));
  if (!tok || !masked || !conf || !tok_c) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  if (b0 < 0 || b1 > L || b0 >= b1 || n < 1)
    return fail(c, ESD_ERR_INVALID_ARG, "block [%d, %d) / n %d invalid", b0, b1, n);
  return k_remask(c, tok, masked, conf, tok_c, B, L, b0, b1, n, nullptr, (cudaStream_t)stream);
}

esd_status esd_denoise_step_region(esd_ctx* c, int32_t* tok, uint8_t* masked, int B, int L, int r0, int r1,
                                   int b0, int b1, int n, int force_dense, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  ESD_TRY(check_bl(c, B, L));
  if (!tok || !masked) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  if (b0 < 0 || b1 > L || b0 >= b1 || n < 1)
    return fail(c, ESD_ERR_INVALID_ARG, "block [%d, %d) / n %d invalid", b0, b1, n);
  if (r0 < 0 || r1 > L || r0 >= r1)
    return fail(c, ESD_ERR_INVALID_ARG, "region [%d, %d) invalid for length %d", r0, r1, L);
  if (c->run.scope == ESD_SCOPE_ALL && (r0 != 0 || r1 != L))
    return fail(c, ESD_ERR_INVALID_ARG, "the all-positions scope recomputes [0, L)");
  return step(c, tok, masked, B, L, r0, r1, b0, b1, n, force_dense != 0, nullptr, (cudaStream_t)stream);
}

esd_status esd_denoise_step(esd_ctx* c, int32_t* tok, uint8_t* masked, int B, int L, int b0, int b1,
                            int n, int force_dense, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  if (c->run.scope == ESD_SCOPE_RESPONSE && !force_dense)
    return fail(c, ESD_ERR_INVALID_ARG, "response-only steps take their region from esd_denoise_step_region");
  const bool blk = c->run.scope == ESD_SCOPE_BLOCK;
  return esd_denoise_step_region(c, tok, masked, B, L, blk ? b0 : 0, blk ? b1 : L, b0, b1, n, force_dense, stream);
}

esd_status esd_generate(esd_ctx* c, const int32_t* prompt, int B, int P, int G, int block_len,
                        int n_unmask, int vanilla, int32_t* out, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  if (!prompt || !out) return fail(c, ESD_ERR_INVALID_ARG, "null pointer");
  if (P < 0 || G < 1 || block_len < 1 || n_unmask < 1 || G % block_len || block_len % n_unmask)
    return fail(c, ESD_ERR_INVALID_ARG, "need G %% block_len == 0 and block_len %% n_unmask == 0");
  const int L = P + G;
  ESD_TRY(check_bl(c, B, L));
  cudaStream_t st = (cudaStream_t)stream;
  ESD_CUDA(c, cudaMemsetAsync(c->g_tok, 0, (size_t)B * L * sizeof(int32_t), st));
  if (P > 0)
    ESD_CUDA(c, cudaMemcpy2DAsync(c->g_tok, (size_t)L * sizeof(int32_t), prompt,
                                  (size_t)P * sizeof(int32_t), (size_t)P * sizeof(int32_t), B,
                                  cudaMemcpyDefault, st));
  init_generation_kernel<<<cdiv((size_t)B * L, 256), 256, 0, st>>>(c->g_tok, c->g_masked, B, L, P,
                                                                  c->dims.mask_id);
  ESD_LAUNCHED(c);
  const int steps = block_len / n_unmask;
  const int R = c->run.refresh_interval;
  for (int blk = 0; blk < G / block_len; ++blk) {
    const int b0 = P + blk * block_len, b1 = b0 + block_len;
    for (int j = 0; j < steps; ++j) {
      const bool dense = vanilla || j == 0 || (R > 0 && j % R == 0);
      const int r0 = c->run.scope == ESD_SCOPE_RESPONSE ? P : (c->run.scope == ESD_SCOPE_BLOCK ? b0 : 0);
      const int r1 = c->run.scope == ESD_SCOPE_BLOCK ? b1 : L;
      ESD_TRY(step(c, c->g_tok, c->g_masked, B, L, r0, r1, b0, b1, n_unmask, dense, nullptr, st));
    }
  }
  ESD_CUDA(c, cudaMemcpy2DAsync(out, (size_t)G * sizeof(int32_t), c->g_tok + P,
                                (size_t)L * sizeof(int32_t), (size_t)G * sizeof(int32_t), B,
                                cudaMemcpyDefault, st));
  return read_flag(c, st);
}

esd_status esd_profile_enable(esd_ctx* c, int kernel, int rows_min, int rows_max) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->prof_kernel = kernel;
  c->prof_min = rows_min;
  c->prof_max = rows_max;
  c->prof_used = 0;
  return ESD_OK;
}

esd_status esd_profile_read(esd_ctx* c, double* total_ms, uint64_t* launches, int reset) {
  if (!c || !total_ms || !launches) return ESD_ERR_INVALID_ARG;
  double t = 0.0;
  for (size_t i = 0; i + 1 < c->prof_used; i += 2) {
    ESD_CUDA(c, cudaEventSynchronize(c->prof_events[i + 1]));
    float ms = 0.0f;
    ESD_CUDA(c, cudaEventElapsedTime(&ms, c->prof_events[i], c->prof_events[i + 1]));
    t += ms;
  }
  *total_ms = t;
  *launches = c->prof_used / 2;
  if (reset) c->prof_used = 0;
  return ESD_OK;
}

esd_status esd_selftest_wait_timeout(esd_ctx* c, unsigned polls, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  if (polls == 0 || polls > esd::kWaitLimit) return fail(c, ESD_ERR_INVALID_ARG, "polls %u outside [1, 2^24]", polls);
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(polls, c->flag);
  ESD_LAUNCHED(c);
  return ESD_OK;
}

esd_status esd_sync_check(esd_ctx* c, void* stream) {
  if (!c) return ESD_ERR_INVALID_ARG;
  c->err.clear();
  return read_flag(c, (cudaStream_t)stream);
}

}  // extern "C"

// =========================================================================
// Allocation-free head (esd_confidence_argmax_noalloc): its workspace is a
// file-scope device array instead of context memory, for callers that cannot
// allocate device memory. Layout per call: inv_rms [rows] float, then the
// head partials [rows, ceil(vocab / 128)] (both fully rewritten by each call).
// =========================================================================
#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ESD_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;

struct NoallocDevice {
  bool ready = false;
  void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int num_sms = 0;
};

std::mutex g_noalloc_mu;
NoallocDevice g_noalloc_dev[kNoallocMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_noalloc_encode = nullptr;

// Once per device, with that device current: resolve the array's device
// address (host code may not use the symbol itself), the SM count, the
// tensor-map encoder and the GEMM's shared-memory attribute.
esd_status noalloc_setup(int dev, NoallocDevice** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocDevice& nd = g_noalloc_dev[dev];
  if (!nd.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ESD_ERR_CUDA;
    if (cudaDeviceGetAttribute(&nd.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ESD_ERR_CUDA;
    if (!g_noalloc_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return ESD_ERR_UNSUPPORTED;
      g_noalloc_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (cudaFuncSetAttribute(esd::tc_gemm_kernel<esd::kEpiHead, 128, 128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             esd::TcCfg<128, 128>::kSmem) != cudaSuccess ||
        cudaFuncSetAttribute(esd::tc_gemm_kernel<esd::kEpiHead, 256, 128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             esd::TcCfg<256, 128>::kSmem) != cudaSuccess)
      return ESD_ERR_CUDA;
    nd.scratch = p;
    nd.ready = true;
  }
  *out = &nd;
  return ESD_OK;
}

bool noalloc_encode(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return g_noalloc_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scratch layout of one call: the status word (its own 256-byte slot), then
// inv_rms [rows] float, then the head partials [rows, ceil(vocab / 128)].
constexpr size_t kNoallocStatusBytes = 256;

size_t noalloc_part_offset(int rows) {
  return kNoallocStatusBytes + (((size_t)rows * sizeof(float) + 255) & ~(size_t)255);
}

}  // namespace

extern "C" esd_status esd_confidence_argmax_noalloc(const void* x_rows, int rows, const void* w_out,
                                                    int d, int vocab, int mask_id, float rms_eps,
                                                    const int32_t* idx, int L, int k,
                                                    float* conf_out, int32_t* tok_out,
                                                    void* stream) {
  if (!x_rows || !w_out || !conf_out || !tok_out) return ESD_ERR_INVALID_ARG;
  if (rows < 1 || d < 128 || d % 128 || vocab < 2 || mask_id < 0 || mask_id >= vocab ||
      !(rms_eps >= 0.0f))
    return ESD_ERR_INVALID_ARG;
  if (idx && (k < 1 || L < k || rows % k)) return ESD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x_rows) | reinterpret_cast<uintptr_t>(w_out)) & 15u)
    return ESD_ERR_INVALID_ARG;
  // every size rejection happens here, before the device is touched
  const int n_tiles = (vocab + 127) / 128;
  const size_t part_off = noalloc_part_offset(rows);
  if (part_off + (size_t)rows * n_tiles * sizeof(HeadPartial) > (size_t)ESD_NOALLOC_SCRATCH_BYTES)
    return ESD_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ESD_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return ESD_ERR_UNSUPPORTED;
  NoallocDevice* nd = nullptr;
  esd_status s = noalloc_setup(dev, &nd);
  if (s != ESD_OK) return s;
  unsigned char* base = reinterpret_cast<unsigned char*>(nd->scratch);
  int* status = reinterpret_cast<int*>(base);
  float* inv_rms = reinterpret_cast<float*>(base + kNoallocStatusBytes);
  HeadPartial* part = reinterpret_cast<HeadPartial*>(base + part_off);
  cudaStream_t st = (cudaStream_t)stream;
  // a bounded wait of the GEMM that runs out records ESD_ERR_TIMEOUT here
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return ESD_ERR_CUDA;

  esd::rms_kernel<__nv_bfloat16><<<cdiv(rows, 8), 256, 0, st>>>((const __nv_bfloat16*)x_rows, inv_rms,
                                                                rows, d, rms_eps);
  if (cudaGetLastError() != cudaSuccess) return ESD_ERR_CUDA;
  const int mt = rows <= 128 ? 1 : 2;
  CUtensorMap ta, tb;
  if (!noalloc_encode(&ta, x_rows, (uint64_t)rows, (uint64_t)d, 128 * mt) ||
      !noalloc_encode(&tb, w_out, (uint64_t)vocab, (uint64_t)d, 64))
    return ESD_ERR_CUDA;
  esd::GemmParams p{};
  p.M = rows;
  p.K = d;
  p.d = d;
  p.vocab = vocab;
  p.mask_id = mask_id;
  p.e.inv_rms = inv_rms;
  p.e.part = part;
  p.e.n_tiles = n_tiles;
  p.flag = status;
  p.num_m = (rows + mt * 128 - 1) / (mt * 128);
  p.num_n = n_tiles;
  p.num_tiles = p.num_m * p.num_n;
  p.splits = 1;
  p.num_units = p.num_tiles;
  p.ws = nullptr;
  const int grid = p.num_units < nd->num_sms ? p.num_units : nd->num_sms;
  if (mt == 1)
    esd::tc_gemm_kernel<esd::kEpiHead, 128, 128><<<grid, 192, esd::TcCfg<128, 128>::kSmem, st>>>(ta, tb, tb, tb, p);
  else
    esd::tc_gemm_kernel<esd::kEpiHead, 256, 128><<<grid, 192, esd::TcCfg<256, 128>::kSmem, st>>>(ta, tb, tb, tb, p);
  if (cudaGetLastError() != cudaSuccess) return ESD_ERR_CUDA;
  esd::head_finalize_kernel<<<cdiv(rows, 8), 256, 0, st>>>(part, rows, n_tiles, idx, L, idx ? k : 1,
                                                          conf_out, tok_out);
  if (cudaGetLastError() != cudaSuccess) return ESD_ERR_CUDA;
  return ESD_OK;
}

extern "C" esd_status esd_noalloc_check(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ESD_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return ESD_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_dev[dev].ready) return ESD_OK;  // no call on this device yet
    scratch = g_noalloc_dev[dev].scratch;
  }
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return ESD_ERR_CUDA;
  int f = 0;
  if (cudaMemcpy(&f, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ESD_ERR_CUDA;
  if (f == esd::kFlagTimeout) return ESD_ERR_TIMEOUT;
  return f == 0 ? ESD_OK : ESD_ERR_CHECK;
}

extern "C" esd_status esd_noalloc_selftest_wait_timeout(unsigned polls, void* stream) {
  if (polls == 0 || polls > esd::kWaitLimit) return ESD_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ESD_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return ESD_ERR_UNSUPPORTED;
  NoallocDevice* nd = nullptr;
  esd_status s = noalloc_setup(dev, &nd);
  if (s != ESD_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  int* status = reinterpret_cast<int*>(nd->scratch);
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return ESD_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, st>>>(polls, status);
  return cudaGetLastError() == cudaSuccess ? ESD_OK : ESD_ERR_CUDA;
}
