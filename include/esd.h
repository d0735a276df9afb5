/*
 * esd.h - C ABI of the early-skipping sparse denoising step for bidirectional
 * masked-diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * Method sources (web summaries; cited by title and section):
 *  [ES]    "ES-dLLM: Efficient Inference for Diffusion Large Language Models by
 *          Early-Skipping", technical summary, sections 1 (problem), 2.A
 *          (importance score), 2.B (selection, early skip, partial cache,
 *          periodic refresh).
 *  [DyLLM] "DyLLM: Efficient Diffusion LLM Inference via Saliency-based Token
 *          Selection and Partial Attention", technical summary, sections 2.A
 *          (temporal saliency of the attention context), 2.B.1 (per-layer
 *          threshold, recompute the salient tokens only) and 2.B.2 (exact
 *          recomputation of the salient rows of attention).
 *
 * Conventions for every call below
 *  - Tensor arguments are DEVICE pointers unless a call says otherwise. They are
 *    borrowed for the duration of the call (weights: for the context's life).
 *  - "storage type" is float32 for ESD_DTYPE_F32 models and bfloat16 for
 *    ESD_DTYPE_BF16 models. Hidden-state rows are [rows, d] row-major; a batch of
 *    B sequences of length L is B*L rows, sequence b occupying rows b*L..b*L+L-1.
 *    Selected-row tensors are [B*k, d], sequence b occupying rows b*k..b*k+k-1.
 *  - Index lists idx are int32 [B, k]: for each sequence, k distinct positions in
 *    [0, L), strictly ascending.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) unless they say they synchronise. Kernel faults surface as
 *    ESD_ERR_CUDA from the next call that checks; bounded device waits that
 *    expire set a device flag that esd_sync_check() reports as ESD_ERR_TIMEOUT.
 *  - No call aborts the process. On failure the call returns a non-zero status
 *    and esd_last_error() describes it; outputs are then unspecified.
 *  - A context is not thread-safe: use one context per host thread.
 *  - The CUDA kernels require a B200-class GPU (sm_100a). bf16 models need
 *    head_dim == 128, d % 128 == 0 and ffn % 128 == 0; float32 models need
 *    head_dim even and <= 128. Other shapes return ESD_ERR_UNSUPPORTED.
 */
#ifndef ESD_H
#define ESD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ESD_OK = 0,
  ESD_ERR_INVALID_ARG = 1, /* bad pointer, shape or configuration */
  ESD_ERR_CUDA = 2,        /* a CUDA runtime/driver call failed */
  ESD_ERR_OOM = 3,         /* device allocation failed */
  ESD_ERR_UNSUPPORTED = 4, /* shape or device the kernels do not handle */
  ESD_ERR_TIMEOUT = 5,     /* a bounded device-side wait expired */
  ESD_ERR_CHECK = 6        /* a device-side consistency check failed */
} esd_status;

typedef enum { ESD_DTYPE_F32 = 0, ESD_DTYPE_BF16 = 1 } esd_dtype;
typedef enum { ESD_SCORE_ES = 0, ESD_SCORE_COS = 1 } esd_score_mode;

/* Model shape. The model is a pre-norm bidirectional transformer without biases:
 * RMSNorm (gain 1; fold learned gains into the next projection's input columns),
 * rotate-half RoPE at absolute positions, full (unmasked) softmax attention,
 * SwiGLU FFN, final RMSNorm and an untied vocabulary head. [ES] section 1: every
 * iteration processes the whole bidirectional sequence. */
typedef struct {
  int n_layers;
  int d;          /* hidden size = n_heads * head_dim */
  int n_heads;
  int head_dim;
  int ffn;        /* SwiGLU inner width */
  int vocab;
  int mask_id;    /* id of the mask token; never predicted */
  float rope_theta;
  float rms_eps;
  int dtype;      /* esd_dtype: storage type of weights, activations and caches */
} esd_model_dims;

/* Weights in the storage type, each matrix [out, in] row-major, device memory
 * owned by the caller and borrowed for the context's lifetime. Per-layer
 * arguments are host arrays of n_layers device pointers (copied at create). */
typedef struct {
  const void* embed;         /* [vocab, d] */
  const void* w_out;         /* [vocab, d] */
  const void* const* wq;     /* [d, d] per layer */
  const void* const* wk;     /* [d, d] */
  const void* const* wv;     /* [d, d] */
  const void* const* wo;     /* [d, d] */
  const void* const* wg;     /* [ffn, d] */
  const void* const* wu;     /* [ffn, d] */
  const void* const* wd;     /* [d, ffn] */
} esd_weights;

/* Early-skipping configuration ([ES] sections 2.A and 2.B). */
typedef enum { ESD_SCORE_ON_H = 0, ESD_SCORE_ON_K = 1, ESD_SCORE_ON_V = 2 } esd_score_tensor;
typedef enum { ESD_SCOPE_ALL = 0, ESD_SCOPE_BLOCK = 1, ESD_SCOPE_RESPONSE = 2 } esd_scope;

typedef struct {
  int score_mode;        /* esd_score_mode */
  float alpha;           /* ES: weight of the previous confidence (0.5 in [ES] 2.A) */
  float lambda_;         /* COS: weight of (1 - previous confidence) */
  int skip_layer;        /* l_s in [1, n_layers): layers >= l_s run on the selected rows */
  float keep_ratio;      /* k = ceil(keep_ratio * L) = (1 - r_l)|S| of [ES] 2.B */
  int refresh_interval;  /* 0: dense refresh at the first step of each block only;
                            R > 0: also every R-th step of a block */
  int max_batch;         /* capacity of the context's caches and workspaces */
  int max_len;
  int skip_layer2;       /* second skip point ([ES] 2.B: early layers such as 4 and 8 of
                            32): 0 = none, else in (skip_layer, n_layers); the rows that
                            reach it are scored again against a second H cache and
                            k2 = ceil(keep_ratio2 * k) of them (per sequence) go on */
  float keep_ratio2;     /* in (0, 1] when skip_layer2 > 0 */
  int score_tensor;      /* esd_score_tensor: the tensor whose variation the score at
                            skip_layer measures ([ES] 2.A, the cached H, K and V of 2.B):
                            the layer's input (H, default) or its fresh keys or values
                            against the layer's K/V cache (K, V; the keys and values of
                            every row are computed first). The second skip point scores H. */
  int scope;             /* esd_scope: the selection set S ([ES] 2.B): every position
                            (default), or the current block of the step — every layer then
                            recomputes only the block's rows, attending over every layer's
                            K/V cache (all layers are cached), k = ceil(keep_ratio * block
                            length); scores H, with one skip point. ESD_SCOPE_RESPONSE: the
                            response-only steps of [DyLLM] 2.B.3 (only the response tokens
                            are processed, the whole context at intervals): the same step
                            over the region [P, L) after the prompt, whose K/V stay as the
                            last full step left them (refresh_interval sets how often a full
                            step runs within a block); the region comes from
                            esd_denoise_step_region or, in esd_generate, from P */
} esd_run_config;

typedef struct esd_ctx esd_ctx;

/* Create a context: validates the shapes, allocates the caches (H, K/V for
 * layers >= skip_layer, confidence/prediction) and workspaces for max_batch x
 * max_len, builds the TMA descriptors of the weights and the RoPE table.
 * Returns ESD_ERR_OOM if the device memory does not fit, ESD_ERR_UNSUPPORTED on
 * a non-sm_100 device or an unsupported shape. */
esd_status esd_create(const esd_model_dims* dims, const esd_weights* weights,
                      const esd_run_config* run, esd_ctx** out);

/* Synchronise the device and free everything the context owns (not the weights). */
esd_status esd_destroy(esd_ctx* ctx);

/* Text of the last error on this context (never NULL; "" after success). */
const char* esd_last_error(const esd_ctx* ctx);

/* k = ceil(keep_ratio * L) clamped to [1, L] ([ES] section 2.B, k = (1 - r_l)|S|). */
int esd_keep_count(const esd_ctx* ctx, int L);

/* Device pointers of the context-owned state, for a batch of B sequences of
 * length L (entry (b, i) is row b*L + i): H cache [B*L, d] (storage type),
 * K and V caches of layers skip_layer..n_layers-1, each [B*L, d] laid out as
 * [B, L, n_heads, head_dim] (storage type), confidence cache [B*L] float32,
 * prediction cache [B*L] int32. Valid until esd_destroy. */
typedef struct {
  void* h_cache;
  void* const* k_cache;   /* n_cached_layers pointers */
  void* const* v_cache;
  float* conf_cache;
  int32_t* tok_cache;
  int n_cached_layers;    /* n_layers - skip_layer (k_cache[i] is layer skip_layer + i), or
                             n_layers with the block scope (k_cache[i] is layer i) */
  int max_batch;
  int max_len;
} esd_state_view;
esd_status esd_state(esd_ctx* ctx, esd_state_view* out);

/* x[b*L + i, :] = embed[tok[b, i], :]. tok int32 [B, L], ids in [0, vocab). */
esd_status esd_embed(esd_ctx* ctx, const int32_t* tok, int B, int L, void* x, void* stream);

/* Importance score and per-sequence top-k ([ES] sections 2.A and 2.B).
 * x, h_cache: [B*L, d] storage type (current skip-layer input and its cache);
 * conf_prev: [B*L] float32 cached confidence. Score per row (float32):
 *   ES : alpha*c + (1-alpha)*||x-H||_1 / max(sqrt(d)*||H||_2, 1e-12)
 *   COS: max(1 - cos(x, H), 0) + lambda*(1 - c),
 *        cos = x.H / sqrt(max(||x||^2 ||H||^2, 1e-24)).
 * Selection: the k highest scores of each sequence under the total order
 * (score descending, index ascending; -0 == +0; NaN lowest), written to
 * idx_out [B, k] in ascending index order. scores_out [B*L] may be NULL.
 * Requires 1 <= k <= L <= max_len, B <= max_batch. */
esd_status esd_importance_select(esd_ctx* ctx, const void* x, const void* h_cache,
                                 const float* conf_prev, int B, int L, int k,
                                 float* scores_out, int32_t* idx_out, void* stream);

/* Context saliency ([DyLLM] sections 2.A and 2.B.1): for every row of the B
 * sequences, the cosine between its attention context at this step, c_cur,
 * and at the previous step, c_prev (both [B*L, d] storage type, d = the
 * concatenated heads; the caller keeps two buffers per layer and swaps them),
 *   s = c_cur.c_prev / sqrt(max(||c_cur||^2 ||c_prev||^2, 1e-24))  (float32),
 * and, per sequence, the salient rows s < tau (the layer's threshold) in
 * ascending order: idx_out [B, L] int32 holds sequence b's salient positions
 * in idx_out[b*L .. b*L + count_out[b] - 1] and -1 after them; count_out [B]
 * int32. sim_out [B*L] float32 may be NULL. NaN similarities are never
 * salient. Requires 1 <= L <= max_len, B <= max_batch. */
esd_status esd_context_saliency(esd_ctx* ctx, const void* c_cur, const void* c_prev, int B, int L,
                                float tau, float* sim_out, int32_t* idx_out, int32_t* count_out,
                                void* stream);

/* DyLLM token-selection layers ([DyLLM] sections 2.A and 2.B.1) on x [B*L, d]
 * storage type: in, the input of layer_begin; out, the output of layer
 * layer_end - 1. For each layer l: every row's attention context C (the
 * attention output of all B*L queries over all keys, exact); unless refresh,
 * the similarity of C with the context of the previous call and the salient
 * rows (below tau[l - layer_begin], a HOST float array, as in
 * esd_context_saliency); then the output projection and the SwiGLU block run
 * on the salient rows only (every row when refresh != 0), and every other row
 * takes its cached output of layer l. The context and output caches of the
 * layer are updated. A non-refresh call needs an earlier refresh of the same
 * layers with the same B and L. counts_out: int32
 * [(layer_end - layer_begin) * B], the salient rows per layer and sequence
 * (L on a refresh), device memory (written asynchronously) or host memory
 * (the call then synchronises the stream once, at its end, to fill it), may
 * be NULL; sim_out: device float32 [(layer_end - layer_begin) * B*L], the
 * similarities, may be NULL (unused on a refresh). The host never waits for
 * the salient count: a non-refresh call runs as a CUDA graph in which a
 * kernel picks, from the count on the device, the body of a conditional
 * switch node that runs the output projection and the SwiGLU block on a
 * capacity of rows (every 16 up to 256 rows, every 256 up to 2048, then
 * steps of a quarter) at or above the count; rows past the count are
 * computed and discarded. The graph is captured on the first call with the
 * same layers, x, B, L, thresholds, sim_out and context buffers (which
 * alternate between consecutive calls) and reused from a cache of 8. The
 * first call allocates the caches: 3 x n_layers x max_batch*max_len rows of
 * d storage-type elements, plus work buffers. */
esd_status esd_dyllm_layers_forward(esd_ctx* ctx, int layer_begin, int layer_end, void* x, int B,
                                    int L, const float* tau, int refresh, int32_t* counts_out,
                                    float* sim_out, void* stream);

/* The same token-selection layers with the contexts from DyLLM's
 * saliency-aware approximate attention ([DyLLM] section 2.B.2) instead of
 * exact attention of every row. Per layer: the rows whose values moved are the
 * rows whose layer input differs (bitwise) from the input the layer saw at
 * its previous call - with the salient rows of the layer below recomputed and
 * the others copied from the output cache, these are the rows that layer
 * changed; their Q/K/V go into the layer's own K/V cache (an unmoved row's
 * input, so its K/V, is unchanged; float32 models recompute every row); the moved
 * rows get exact attention rows (and rewrite their cached probabilities) and
 * every other row's context moves by its cached probabilities times the moved
 * rows' change of V (esd_approx_attention's arithmetic). Saliency, the output
 * projection, SwiGLU and the caches then as esd_dyllm_layers_forward. A
 * refresh computes every row exactly and fills the caches; a non-refresh call
 * needs an earlier refresh through this call, same B and L. The first call
 * allocates, per layer, the last input and the K/V of max_batch*max_len rows
 * of d storage-type elements and float32 probabilities [max_batch, n_heads,
 * max_len, max_len] (ESD_ERR_OOM if that does not fit), besides the caches of
 * esd_dyllm_layers_forward. Synchronises like esd_dyllm_layers_forward (only
 * for a host counts_out); bf16 models compute Q/K/V of the moved rows only,
 * in a second switch node per layer whose body capacity is at or above the
 * largest moved count of a sequence (a body that copies the contexts when
 * nothing moved). */
esd_status esd_dyllm_layers_forward_approx(esd_ctx* ctx, int layer_begin, int layer_end, void* x, int B,
                                           int L, const float* tau, int refresh, int32_t* counts_out,
                                           float* sim_out, void* stream);

/* DyLLM saliency-aware approximate attention of one layer ([DyLLM] section
 * 2.B.2). The changed rows of sequence b (the tokens whose values V moved
 * since the previous step) are changed_idx[b*L .. b*L + changed_count[b] - 1],
 * strictly ascending positions in [0, L), as esd_context_saliency writes them
 * (both device int32; changed_idx [B, L], changed_count [B]). Per head h:
 *   every row i:        C_i += sum over changed j of P[b, h, i, j] (V_j - V_prev_j)
 *   then changed row j: P[b, h, j, :] = softmax(q_j K_b^T / sqrt(head_dim))
 *                       over all L keys (exact), C_j = P[b, h, j, :] V_b
 * so the non-changed rows cost O(L x changed) instead of O(L^2).
 * q, k, v, v_prev: [B*L, d] laid out as [B, L, n_heads, head_dim], storage
 * type, RoPE already applied to q and k; only the changed rows of q are read.
 * ctx_io: [B*L, d] storage type, the contexts of the previous step in, the
 * new contexts out. p: [B, n_heads, L, L] float32, each row's attention
 * probabilities from the last step that computed it exactly, in; the changed
 * rows rewritten, out. All device memory owned by the caller; q, k, v, v_prev
 * must not overlap ctx_io or p. No synchronisation. bf16 models: tensor-core
 * kernels (the update as a bf16 product of the cached probabilities' moved
 * columns and the change of V, fp32 sums; the moved rows on the SM-pair
 * attention kernel, their probability rows normalised from its scores);
 * float32 models: two SIMT kernels.
 * Requires 1 <= L <= max_len, B <= max_batch. A count outside [0, L] or a
 * position out of range or out of order is skipped and reported as
 * ESD_ERR_CHECK by the next esd_sync_check. */
esd_status esd_approx_attention(esd_ctx* ctx, const void* q, const void* k, const void* v,
                                const void* v_prev, const int32_t* changed_idx,
                                const int32_t* changed_count, int B, int L, void* ctx_io,
                                float* p, void* stream);

/* The selection step alone, from given scores [B*L] float32 (same order and
 * output as esd_importance_select). */
esd_status esd_topk_select(esd_ctx* ctx, const float* scores, int B, int L, int k,
                           int32_t* idx_out, void* stream);

/* Gather the selected rows and refresh their H-cache entries ([ES] section 2.B:
 * in-place scatter of the selected tokens' cache entries):
 *   x_sel[b*k + j] = x[b*L + idx[b, j]];  h_cache[b*L + idx[b, j]] = x[b*L + idx[b, j]]
 * h_cache may be NULL (gather only). x and h_cache must not overlap. */
esd_status esd_gather_rows(esd_ctx* ctx, const void* x, const int32_t* idx, int B, int L,
                           int k, void* x_sel, void* h_cache, void* stream);

/* Run layers [layer_begin, layer_end) on rows x_sel [B*k, d] (in place).
 * With idx (int32 [B, k]): the rows are the selected positions; each layer
 * projects Q/K/V of the selected rows (RoPE at position idx), scatters the
 * fresh K/V into that layer's cache at idx, and the selected queries attend
 * over the whole cache of their sequence ([ES] section 2.B; [DyLLM] section
 * 2.B.2), then O projection, residual, SwiGLU FFN, residual. Requires
 * layer_begin >= skip_layer. Entries of idx are positions in [0, L); a
 * negative entry marks a padding row, of which no K/V is written (its output
 * row is unspecified).
 * With idx == NULL: k must equal L and every row is processed (dense); layers
 * >= skip_layer write all rows of their K/V cache, layers below use a
 * workspace. Each call overwrites the context's per-layer workspaces. */
esd_status esd_sparse_layers_forward(esd_ctx* ctx, int layer_begin, int layer_end,
                                     const int32_t* idx, int B, int L, int k,
                                     void* x_sel, void* stream);

/* Partial attention alone ([DyLLM] section 2.B.2: the salient rows of the
 * attention matrix are recomputed exactly): out[b*k + j] = softmax(q[b*k + j]
 * K_b^T / sqrt(head_dim)) V_b per head, over all L keys of sequence b.
 * q, out: [B*k, d] (RoPE already applied to q); k_cache, v_cache: [B*L, d] laid
 * out as [B, L, n_heads, head_dim]; storage type. This is the attention that
 * esd_sparse_layers_forward runs after scattering the fresh K/V. */
esd_status esd_partial_attention(esd_ctx* ctx, const void* q, const void* k_cache,
                                 const void* v_cache, int B, int L, int k, void* out,
                                 void* stream);

/* Head: final RMSNorm, vocabulary projection, softmax maximum and argmax
 * ([ES] section 2.A: c is the maximum probability) of rows x_rows [B*k, d].
 * The mask id is excluded from the softmax and the argmax; argmax ties go to
 * the lower id. Logits are never written to memory.
 * With idx == NULL, row r's result goes to conf_out[r], tok_out[r] (B*k rows).
 * With idx ([B, k]), row b*k + j's result goes to conf_out[b*L + idx[b, j]] and
 * tok_out[b*L + idx[b, j]] (scatter into [B*L] caches; other entries untouched). */
esd_status esd_confidence_argmax(esd_ctx* ctx, const void* x_rows, const int32_t* idx,
                                 int B, int L, int k, float* conf_out, int32_t* tok_out,
                                 void* stream);

/* Test helper: final RMSNorm and vocabulary logits of rows [rows, d] into
 * logits_out [rows, vocab] float32 (the mask id's logit is written as -inf). */
esd_status esd_logits(esd_ctx* ctx, const void* x_rows, int rows, float* logits_out,
                      void* stream);

/* Remask ([ES] section 1: only the most confident masked tokens are unmasked
 * per step): for each sequence, among the masked positions i in
 * [block_begin, block_end), the n_unmask with the highest conf_cache (ties to
 * the lower position; all of them if fewer remain) get tok = tok_cache and
 * masked = 0. tok int32 [B, L], masked uint8 [B, L]. */
esd_status esd_remask(esd_ctx* ctx, int32_t* tok, uint8_t* masked, const float* conf_cache,
                      const int32_t* tok_cache, int B, int L, int block_begin, int block_end,
                      int n_unmask, void* stream);

/* One denoising step on tok/masked ([B, L], device) using the context's caches.
 * Dense (force_dense != 0): embed, every layer on every row (fills the H cache
 * with the skip layer's input and every K/V cache), head on every row into the
 * confidence/prediction caches, remask. This is the periodic full refresh of
 * [ES] section 2.B and, taken at every step, the vanilla every-token baseline.
 * Sparse: embed, layers < skip_layer dense, esd_importance_select,
 * esd_gather_rows (with the H cache), esd_sparse_layers_forward over the
 * remaining layers, esd_confidence_argmax scattering into the caches, remask.
 * A sparse step needs the caches filled by an earlier dense step at the same
 * (B, L). */
esd_status esd_denoise_step(esd_ctx* ctx, int32_t* tok, uint8_t* masked, int B, int L,
                            int block_begin, int block_end, int n_unmask, int force_dense,
                            void* stream);

/* The same step with the recomputed region given apart from the unmasking
 * block: with ESD_SCOPE_BLOCK or ESD_SCOPE_RESPONSE a sparse step recomputes
 * rows [region_begin, region_end) in every layer (every other row keeps its
 * caches), selects k = ceil(keep_ratio * region length) of them at the skip
 * layer, and remasks within [block_begin, block_end). esd_denoise_step is this
 * call with the region = the block (block scope) or the whole sequence (all
 * positions). With ESD_SCOPE_ALL the region must be [0, L); with
 * ESD_SCOPE_RESPONSE, esd_denoise_step itself returns ESD_ERR_INVALID_ARG (it
 * has no prompt length) and this call takes region [P, L). Dense steps ignore
 * the region. */
esd_status esd_denoise_step_region(esd_ctx* ctx, int32_t* tok, uint8_t* masked, int B, int L,
                                   int region_begin, int region_end, int block_begin, int block_end,
                                   int n_unmask, int force_dense, void* stream);

/* Whole generation: tok = prompt followed by G mask tokens; for each block of
 * block_len positions, block_len / n_unmask steps (dense at a block's first
 * step and every refresh_interval steps, else sparse - over the response
 * [P, L) with ESD_SCOPE_RESPONSE; every step dense when vanilla != 0);
 * finally out[b, j] = tok[b, P + j]. prompt [B, P] and out
 * [B, G] (int32) may be host or device pointers. Synchronises `stream` before
 * returning and reports device-side timeouts. Requires G % block_len == 0 and
 * block_len % n_unmask == 0. */
esd_status esd_generate(esd_ctx* ctx, const int32_t* prompt, int B, int P, int G,
                        int block_len, int n_unmask, int vanilla, int32_t* out,
                        void* stream);

/* Failure-path self-test (no counterpart on the pages): launches one block whose
 * thread waits, through the same bounded wait as the step's kernels, on a
 * barrier phase that nothing completes, for at most `polls` polls (1 ..
 * 2^24), and then records the timeout on the context's device flag exactly as
 * an expired wait of a GEMM or attention kernel does. The next
 * esd_sync_check() returns ESD_ERR_TIMEOUT and clears the flag; the context
 * stays usable. No fault, trap or unbounded wait is involved. */
esd_status esd_selftest_wait_timeout(esd_ctx* ctx, unsigned polls, void* stream);

/* Synchronise `stream` and report any device-side flag (ESD_ERR_TIMEOUT,
 * ESD_ERR_CHECK) raised since the last check, clearing it. */
esd_status esd_sync_check(esd_ctx* ctx, void* stream);

/* Number of kernels this context has launched since it was created (for
 * accounting of GPU launches). */
uint64_t esd_launch_count(const esd_ctx* ctx);

/* Kernel families for esd_profile_enable. */
typedef enum {
  ESD_K_GEMM_QKV = 0,      /* QKV projection + RoPE + K/V scatter */
  ESD_K_GEMM_O = 1,        /* attention output projection + residual */
  ESD_K_GEMM_GATE_UP = 2,  /* gate/up projection + SwiGLU */
  ESD_K_GEMM_DOWN = 3,     /* down projection + residual */
  ESD_K_HEAD = 4,          /* fused vocabulary head (partials) */
  ESD_K_ATTENTION = 6,     /* partial / dense attention */
  ESD_K_SCORE_SELECT = 7   /* importance score + top-k */
} esd_kernel_id;

/* Instrumentation: when enabled, every launch of kernel family `kernel` whose
 * row count lies in [rows_min, rows_max] is bracketed by two CUDA events
 * recorded on its launching stream. kernel < 0 disables. Events are created on
 * demand (not inside stream capture). */
esd_status esd_profile_enable(esd_ctx* ctx, int kernel, int rows_min, int rows_max);

/* Synchronises the recorded events and returns the summed device time (ms) and
 * the number of timed launches since the last reset; reset != 0 starts over. */
esd_status esd_profile_read(esd_ctx* ctx, double* total_ms, uint64_t* launches, int reset);

/* ---------------------------------------------------------------------------
 * Allocation-free head (no counterpart in the papers: a deployment addition).
 *
 * Some callers cannot allocate device memory at all: code running under a
 * memory pool or allocator that must not be bypassed, plug-ins whose host
 * forbids cudaMalloc after start-up, or processes whose device memory is fully
 * reserved. esd_create allocates caches and workspaces, so this call needs no
 * context: it computes the same result as esd_confidence_argmax (final
 * RMSNorm, vocabulary projection on the tensor cores, softmax maximum and
 * argmax with the mask id excluded, optional scatter through idx) for a bf16
 * model, taking its workspace from a fixed array inside the library.
 *
 * x_rows [rows = B*k, d] bf16 and w_out [vocab, d] bf16 are device pointers
 * (16-byte aligned); d must be a multiple of 128. idx, L, k, conf_out and
 * tok_out mean what they mean for esd_confidence_argmax (idx may be NULL, then
 * L and k are ignored and row r writes conf_out[r], tok_out[r]).
 *
 * Scratch: 256 + round_up(4 * rows, 256) + 12 * rows * ceil(vocab / 128)
 * bytes must not exceed ESD_NOALLOC_SCRATCH_BYTES (at vocab 126464 about 690
 * rows); larger requests return ESD_ERR_INVALID_ARG before the device is
 * touched. The array (8 MiB) lives in the library's device image: every GPU
 * that loads the library holds it until the process exits. Every call shares
 * it and it keeps the last call's contents (each call overwrites what it
 * reads), so calls that may overlap on the GPU - on different streams, or from
 * several host threads - race and must be serialised by the caller.
 * The first call on a device sets up that device (resolves the array's device
 * address, sets kernel attributes); make that first call before any stream
 * capture. No call allocates device memory or frees it.
 *
 * Status: the call returns before its kernels finish. Its first 256 bytes of
 * scratch hold a status word that the call clears on `stream` before its
 * kernels run; if a bounded wait inside the GEMM runs out, the kernel records
 * ESD_ERR_TIMEOUT there and the outputs are unspecified. The outputs of the
 * last call on the current device are valid only when esd_noalloc_check
 * returns ESD_OK. */
#define ESD_NOALLOC_SCRATCH_BYTES (8u << 20)
esd_status esd_confidence_argmax_noalloc(const void* x_rows, int rows, const void* w_out, int d,
                                         int vocab, int mask_id, float rms_eps,
                                         const int32_t* idx, int L, int k, float* conf_out,
                                         int32_t* tok_out, void* stream);

/* Synchronises `stream` and reads the status word of the allocation-free head
 * on the current device: ESD_OK (or no call made on this device yet),
 * ESD_ERR_TIMEOUT (a device wait of the last call ran out: its outputs are
 * unspecified), ESD_ERR_CUDA. Allocates nothing. */
esd_status esd_noalloc_check(void* stream);

/* Failure-path self-test of the allocation-free head: clears its status word
 * and runs, on `stream`, one bounded wait on a barrier phase that nothing
 * completes, giving up after `polls` polls (1 .. 2^24), so that the next
 * esd_noalloc_check returns ESD_ERR_TIMEOUT without any fault. Shares the
 * scratch array like the head (do not overlap it with a head call).
 * Allocates nothing. */
esd_status esd_noalloc_selftest_wait_timeout(unsigned polls, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ESD_H */
