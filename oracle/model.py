"""Plain float64 oracle of the early-skipping denoising step (test infrastructure only).

Model (the pages name LLaDA-8B and Dream-7B but print no architecture; the
shapes come from the workload configurations): a pre-norm bidirectional
transformer without biases and with an untied head. For each layer

    h  = x / sqrt(mean(x^2) + eps)                      (RMSNorm, gain 1)
    q, k, v = h Wq^T, h Wk^T, h Wv^T                     (weights stored [out, in])
    q, k = RoPE(q, pos), RoPE(k, pos)                    (rotate-half, freq_j = theta^(-2j/hd))
    a  = softmax(q k^T / sqrt(hd)) v                     (all L keys: no mask)
    x  = x + a Wo^T
    h2 = RMSNorm(x)
    x  = x + (silu(h2 Wg^T) * (h2 Wu^T)) Wd^T

and the head is ``logits = RMSNorm(x) W_out^T`` with the mask id's logit
excluded; confidence = max softmax = 1 / sum_j exp(l_j - l_max) and the
prediction is the argmax (ties to the lower id).

Storage points (values rounded to the storage type "f32" or "bf16", round to
nearest even, and nowhere else): x after the embedding and after each residual
add; q, k, v after RoPE; the attention output; the SwiGLU product; every cache
entry (they are copies of stored values). Scores and confidences are float32.
Everything between storage points is float64.

Early skipping ("ES-dLLM: Efficient Inference for Diffusion Large Language
Models by Early-Skipping", technical summary section 2; "DyLLM: Efficient
Diffusion LLM Inference via Saliency-based Token Selection and Partial
Attention", technical summary section 2.B.2), with the readings this oracle
takes where the summaries are silent:

* H is the residual-stream input of the skip layer l_s; H^(t-1) and c^(t-1)
  are the cache entries, i.e. the values from the last step that recomputed
  the row.
* S is every position of a sequence (prompt and all generation positions);
  k = ceil(keep_ratio * L) per sequence.
* Top-k uses the total order (score descending, index ascending); -0 counts
  as +0; NaN ranks below everything; the selected indices are returned in
  ascending order.
* Layers below l_s run densely on all rows at every step (their K/V are not
  cached). Layers from l_s on run only on the selected rows; their fresh K/V
  are scattered into the layer's cache before the selected queries attend
  over the whole cache (partial attention).
* The head runs on the selected rows only; skipped rows keep their cached
  confidence and prediction.
* A dense refresh (all layers, all rows) is taken at the first step of every
  block and, if refresh_interval R > 0, at every R-th step of a block. It
  fills H, every K/V cache and every confidence/prediction.
* Every step ends by unmasking, among the masked positions of the current
  block, the n with the highest cached confidence (ties to the lower
  position), writing the cached prediction there.
* ES score: alpha*c + (1-alpha)*||x - H||_1 / max(sqrt(d)*||H||_2, 1e-12).
  The variation is taken on the skip layer's input by default; with
  score_tensor "k" or "v" on that layer's fresh keys or values against its
  K/V cache (the summaries name H, K and V as the cached intermediate tensors).
  COS score (the small configuration): max(1 - cos(x, H), 0) + lam*(1 - c),
  cos = x.H / sqrt(max(||x||^2 ||H||^2, 1e-24)).
* DyLLM saliency (the token-selection variant of "DyLLM", technical summary
  sections 2.A and 2.B.1): C_{t-1} is the context of the previous step (the
  caller keeps two context buffers per layer and swaps them), the similarity
  uses the same floored cosine, and a row is salient when its float32
  similarity is below float32(tau).

Parity status: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py`` against closed forms, library routines, invariants
or brute force, except the quality of generation on real text, which needs
trained weights and datasets (parity unpinned; not part of this oracle).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

from synth import ModelDims, RunConfig

__all__ = [
    "round_bf16", "store", "prepare_weights", "rms_inv", "rope", "attention",
    "silu", "dense_layer", "sparse_layer", "logits", "head", "importance_es",
    "importance_cos", "importance", "topk_select", "topk_margin", "remask",
    "keep_count", "logit_scale", "State", "new_state", "embed", "dense_step", "sparse_step",
    "generate", "ModelDims", "RunConfig", "context_cosine", "salient_rows", "dyllm_layer", "approx_contexts",
    "attention_probs", "dyllm_layer_approx",
]


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------
def round_bf16(x) -> np.ndarray:
    """Round float64 values to bfloat16 (8 significant bits), nearest-even.

    Written from the format's definition: a bf16 number has the float32
    exponent range and an 8-bit significand, so the quantum of a value with
    binary exponent e (x = m 2^e, 1/2 <= |m| < 1) is 2^(e-8), and never below
    2^-133 (the subnormal quantum). Values whose rounding reaches 2^128
    overflow to infinity.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.maximum(e - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(x, -q)), q)
    big = np.abs(r) >= 2.0 ** 128
    if np.any(big):
        r = np.where(big, np.copysign(np.inf, x), r)
    return r


def store(x, dtype: str) -> np.ndarray:
    """Value of ``x`` after being stored in ``dtype`` ("f32" or "bf16"; "f64"
    keeps every value, for the pins that compare against library routines)."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f64":
        return x
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(dtype)


def prepare_weights(w32: dict, dims: ModelDims) -> dict:
    """float32 weights from ``synth`` -> float64 arrays holding storage values."""
    cv = lambda a: store(np.asarray(a, dtype=np.float64), dims.dtype)
    return {"embed": cv(w32["embed"]), "w_out": cv(w32["w_out"]),
            "layers": [{k: cv(v) for k, v in lw.items()} for lw in w32["layers"]]}


# --------------------------------------------------------------------------
# transformer pieces
# --------------------------------------------------------------------------
def rms_inv(x: np.ndarray, eps: float) -> np.ndarray:
    """1 / sqrt(mean(x^2) + eps) over the last axis."""
    return 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding of x [R, H, hd] at absolute positions pos [R].

    Pair (j, j + hd/2) is rotated by the angle pos * theta^(-2j/hd).
    """
    hd = x.shape[-1]
    half = hd // 2
    freq = theta ** (-2.0 * np.arange(half, dtype=np.float64) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * freq[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) v per head, over all keys (no mask).

    q [R, H, hd]; k, v [L, H, hd] -> [R, H, hd].
    """
    hd = q.shape[-1]
    s = np.einsum("rhd,lhd->hrl", q, k) / math.sqrt(hd)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.einsum("hrl,lhd->rhd", p, v)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def _qkv(x, pos, lw, dims):
    """Normalised projections with RoPE, rounded at the storage points."""
    R = x.shape[0]
    H, hd, dt = dims.n_heads, dims.head_dim, dims.dtype
    h = x * rms_inv(x, dims.rms_eps)[:, None]
    q = rope((h @ lw["wq"].T).reshape(R, H, hd), pos, dims.rope_theta)
    k = rope((h @ lw["wk"].T).reshape(R, H, hd), pos, dims.rope_theta)
    v = (h @ lw["wv"].T).reshape(R, H, hd)
    return store(q, dt), store(k, dt), store(v, dt)


def _attn_out_and_ffn(x, a, lw, dims, trace=None):
    """x + a Wo^T, then the SwiGLU block, rounded at the storage points.

    ``trace`` (a dict, optional) receives "residual_terms": per output element
    the 2-norm of the terms of its last sum, sqrt(x^2 + sum_j (act_j Wd_ij)^2)
    - the scale that perturbations of the stored operands (x, act) move the
    sum by (reported for the parity tests; it does not change the result)."""
    dt = dims.dtype
    R = x.shape[0]
    a = store(a, dt).reshape(R, dims.d)
    x = store(x + a @ lw["wo"].T, dt)
    h2 = x * rms_inv(x, dims.rms_eps)[:, None]
    act = store(silu(h2 @ lw["wg"].T) * (h2 @ lw["wu"].T), dt)
    down = act @ lw["wd"].T
    if trace is not None:
        trace["residual_terms"] = np.sqrt(x * x + (act * act) @ (lw["wd"] * lw["wd"]).T)
    return store(x + down, dt)


def dense_layer(x: np.ndarray, lw: dict, dims: ModelDims, trace=None):
    """One layer over all L rows of one sequence (x [L, d]).

    Returns (x_out [L, d], k [L, H, hd], v [L, H, hd]). Full bidirectional
    attention: every row attends over every row ("ES-dLLM", technical summary
    section 1: the whole sequence is processed at every iteration).
    """
    L = x.shape[0]
    q, k, v = _qkv(x, np.arange(L), lw, dims)
    a = attention(q, k, v)
    return _attn_out_and_ffn(x, a, lw, dims, trace), k, v


def approx_contexts(q, k, v, v_prev, c_prev, p_prev, changed):
    """Saliency-aware approximate attention ("DyLLM", technical summary
    section 2.B.2): the rows in ``changed`` (the tokens whose values moved, the
    salient ones) get exact attention rows; every other row updates its cached
    context by the change of the salient values weighted by its cached
    attention probabilities, C_i += sum_{j in changed} P_ij (V_j - V_prev_j),
    which costs O(L x |changed|) instead of O(L^2).

    q, k, v, v_prev, c_prev [L, H, hd]; p_prev [H, L, L] (each row's
    probabilities from the last step that computed it exactly). Returns the
    contexts [L, H, hd] and the probabilities with the exact rows refreshed.
    """
    L, H, hd = q.shape
    changed = np.asarray(changed, dtype=np.int64)
    c = np.array(c_prev, dtype=np.float64, copy=True)
    p = np.array(p_prev, dtype=np.float64, copy=True)
    if len(changed):
        dv = (v - v_prev)[changed]                                  # [A, H, hd]
        c += np.einsum("hia,ahd->ihd", p_prev[:, :, changed], dv)
        sc = np.einsum("ahd,lhd->hal", q[changed], k) / math.sqrt(hd)
        sc = sc - sc.max(axis=-1, keepdims=True)
        e = np.exp(sc)
        pe = e / e.sum(axis=-1, keepdims=True)
        p[:, changed, :] = pe
        c[changed] = np.einsum("hal,lhd->ahd", pe, v)
    return c, p


def dyllm_layer(x: np.ndarray, lw: dict, dims: ModelDims, c_prev, out_prev, tau: float,
                refresh: bool, salient=None, trace=None):
    """One layer of the DyLLM token-selection variant over the L rows of one
    sequence ("DyLLM", technical summary sections 2.A and 2.B.1).

    Every row's attention context C (the attention output, stored) is computed
    exactly; a row is salient when the cosine of C with the previous step's
    context c_prev falls below tau (every row on a refresh); the output
    projection and the SwiGLU block run on the salient rows only, and every
    other row takes its cached output out_prev of this layer. ``salient`` (the
    ascending positions) overrides the decision, for teacher-forced checks.

    Returns (out [L, d], C [L, d], salient positions, similarity or None).
    """
    L = x.shape[0]
    q, k, v = _qkv(x, np.arange(L), lw, dims)
    a = store(attention(q, k, v), dims.dtype).reshape(L, dims.d)
    sim = None if refresh else context_cosine(a, c_prev)
    if salient is None:
        salient = np.arange(L, dtype=np.int32) if refresh else salient_rows(sim, tau)
    out = np.array(out_prev, dtype=np.float64, copy=True) if not refresh else np.zeros_like(x)
    if len(salient):
        tr = {} if trace is not None else None
        out[salient] = _attn_out_and_ffn(x[salient], a[salient], lw, dims, tr)
        if trace is not None:
            trace["salient_terms"] = tr["residual_terms"]
    return out, a, np.asarray(salient, dtype=np.int32), sim


def attention_probs(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) per head: q [R, H, hd], k [L, H, hd] -> [H, R, L]."""
    hd = q.shape[-1]
    s = np.einsum("rhd,lhd->hrl", q, k) / math.sqrt(hd)
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def dyllm_layer_approx(x: np.ndarray, lw: dict, dims: ModelDims, cache: dict, tau: float,
                       refresh: bool, salient=None, trace=None):
    """One layer of the DyLLM token-selection variant with the saliency-aware
    approximate attention ("DyLLM", technical summary sections 2.B.1 and
    2.B.2) over the L rows of one sequence.

    The rows whose values moved are the rows whose layer input x differs from
    the input this layer saw at the previous call (their q, k, v are the only
    ones that change); they get exact attention rows over the keys with their
    fresh keys and values in place, and every other row's context moves by
    sum_{moved j} P_ij (V_j - V_prev_j) with its cached probabilities
    (approx_contexts). Contexts are stored in the storage type. Then, as in
    dyllm_layer: rows whose context cosine with the previous context is below
    tau are salient and get the output projection + SwiGLU; the others keep the
    cached output. A refresh computes every row exactly and fills the cache.

    cache (per layer and sequence, updated in place): "x" the layer input, "k",
    "v" [L, H, hd], "c" the stored contexts [L, d], "p" [H, L, L] float64,
    "out" [L, d]. Returns (out, contexts, salient positions, similarity or
    None, moved positions).
    """
    L = x.shape[0]
    H, hd, dt = dims.n_heads, dims.head_dim, dims.dtype
    q, k, v = _qkv(x, np.arange(L), lw, dims)
    if refresh:
        moved = np.arange(L, dtype=np.int32)
        a = store(attention(q, k, v), dt).reshape(L, dims.d)
        p = attention_probs(q, k)
        sim = None
        sal = np.arange(L, dtype=np.int32) if salient is None else np.asarray(salient, dtype=np.int32)
        out = np.zeros_like(x)
    else:
        moved = np.nonzero(np.any(x != cache["x"], axis=-1))[0].astype(np.int32)
        v_prev = cache["v"]
        c, p = approx_contexts(q, k, v, v_prev, cache["c"].reshape(L, H, hd), cache["p"], moved)
        a = store(c, dt).reshape(L, dims.d)
        sim = context_cosine(a, cache["c"])
        sal = salient_rows(sim, tau) if salient is None else np.asarray(salient, dtype=np.int32)
        out = np.array(cache["out"], dtype=np.float64, copy=True)
    if len(sal):
        tr = {} if trace is not None else None
        out[sal] = _attn_out_and_ffn(x[sal], a[sal], lw, dims, tr)
        if trace is not None:
            trace["salient_terms"] = tr["residual_terms"]
    cache.update(x=np.array(x, copy=True), k=k, v=v, c=a, p=p, out=np.array(out, copy=True))
    return out, a, sal, sim, moved


def sparse_layer(xs: np.ndarray, idx: np.ndarray, kc: np.ndarray, vc: np.ndarray,
                 lw: dict, dims: ModelDims, trace=None) -> np.ndarray:
    """One layer over the selected rows of one sequence.

    xs [k, d] are the rows at positions idx [k]; kc, vc [L, H, hd] are this
    layer's K/V cache and are updated in place: the selected rows' fresh K/V
    are scattered in ("ES-dLLM", technical summary section 2.B: in-place cache
    update for selected tokens, reuse for skipped ones), then the selected
    queries attend over the whole cache ("DyLLM", technical summary section
    2.B.2: the salient rows of the attention matrix are recomputed exactly).
    """
    q, k, v = _qkv(xs, idx, lw, dims)
    kc[idx] = k
    vc[idx] = v
    a = attention(q, kc, vc)
    return _attn_out_and_ffn(xs, a, lw, dims, trace)


def logits(x: np.ndarray, w_out: np.ndarray, dims: ModelDims) -> np.ndarray:
    """Final RMSNorm then the vocabulary projection (float64, mask id at -inf)."""
    h = x * rms_inv(x, dims.rms_eps)[:, None]
    lg = h @ w_out.T
    lg[:, dims.mask_id] = -np.inf
    return lg


def head(x: np.ndarray, w_out: np.ndarray, dims: ModelDims):
    """Confidence (max softmax probability) and prediction for rows x [R, d].

    The confidence is the maximum softmax probability ("ES-dLLM", technical
    summary section 2.A, definition of c): 1 / sum_j exp(l_j - l_max), the
    mask id excluded. The argmax is taken on the float32 logits (ties to the
    lower id), the precision in which the kernels decide it.
    Returns (conf float32 values as float64 [R], tok int32 [R], top-2 margin
    of the float32 logits [R]).
    """
    lg = logits(x, w_out, dims)
    m = lg.max(axis=1)
    conf = store(1.0 / np.exp(lg - m[:, None]).sum(axis=1), "f32")
    lg32 = lg.astype(np.float32)
    tok = np.argmax(lg32, axis=1).astype(np.int32)
    srt = np.sort(lg32, axis=1)
    margin = (srt[:, -1].astype(np.float64) - srt[:, -2].astype(np.float64))
    return conf, tok, margin


def logit_scale(x: np.ndarray, w_out: np.ndarray, dims: ModelDims) -> np.ndarray:
    """Largest finite |logit| of each row (the scale of a row's argmax margins)."""
    lg = logits(x, w_out, dims)
    return np.max(np.where(np.isfinite(lg), np.abs(lg), 0.0), axis=1)


# --------------------------------------------------------------------------
# importance score, selection, remasking
# --------------------------------------------------------------------------
def importance_es(x: np.ndarray, hc: np.ndarray, conf: np.ndarray, alpha: float) -> np.ndarray:
    """ES-dLLM importance score ("ES-dLLM", technical summary section 2.A):

        I_i = alpha * c_i + (1 - alpha) * ||x_i - H_i||_1 / (sqrt(d) * ||H_i||_2)

    x, hc [L, d] (current and cached hidden states at the skip layer), conf [L]
    (cached confidence). The denominator is floored at 1e-12. float32 result.
    """
    d = x.shape[-1]
    l1 = np.abs(x - hc).sum(axis=-1)
    den = np.maximum(math.sqrt(d) * np.sqrt((hc * hc).sum(axis=-1)), 1e-12)
    return store(alpha * conf + (1.0 - alpha) * (l1 / den), "f32")


def importance_cos(x: np.ndarray, hc: np.ndarray, conf: np.ndarray, lam: float) -> np.ndarray:
    """Cosine-variation importance: max(1 - cos(x_i, H_i), 0) + lam * (1 - c_i).

    cos = x.H / sqrt(max(||x||^2 ||H||^2, 1e-24)). float32 result.
    """
    dot = (x * hc).sum(axis=-1)
    na = (x * x).sum(axis=-1)
    nb = (hc * hc).sum(axis=-1)
    cos = dot / np.sqrt(np.maximum(na * nb, 1e-24))
    return store(np.maximum(1.0 - cos, 0.0) + lam * (1.0 - conf), "f32")


def importance(x, hc, conf, run: RunConfig) -> np.ndarray:
    if run.score_mode == "es":
        return importance_es(x, hc, conf, run.alpha)
    if run.score_mode == "cos":
        return importance_cos(x, hc, conf, run.lam)
    raise ValueError(run.score_mode)


def context_cosine(c_cur: np.ndarray, c_prev: np.ndarray) -> np.ndarray:
    """Temporal similarity of the attention contexts of each row ("DyLLM",
    technical summary section 2.A: the cosine between a token's attention
    context vectors C_{t,l} and C_{t-1,l} at adjacent denoising steps):

        s_i = C_t,i . C_t-1,i / sqrt(max(||C_t,i||^2 ||C_t-1,i||^2, 1e-24))

    c_cur, c_prev [L, d] (d = heads x head_dim, the concatenated contexts).
    The floor makes a zero row similarity 0. float32 result.
    """
    dot = (c_cur * c_prev).sum(axis=-1)
    na = (c_cur * c_cur).sum(axis=-1)
    nb = (c_prev * c_prev).sum(axis=-1)
    return store(dot / np.sqrt(np.maximum(na * nb, 1e-24)), "f32")


def salient_rows(sim: np.ndarray, tau: float) -> np.ndarray:
    """Rows whose similarity falls below the layer's threshold ("DyLLM",
    technical summary sections 2.A and 2.B.1: a token is salient when its
    temporal similarity drops below tau; only salient tokens are recomputed),
    in ascending order. The comparison is taken on the float32 similarity
    against float32(tau); NaN is never below tau."""
    s = np.asarray(sim, dtype=np.float32)
    return np.flatnonzero(s < np.float32(tau)).astype(np.int32)


def keep_count(keep_ratio: float, length: int) -> int:
    """k = ceil(keep_ratio * L) per sequence ("ES-dLLM", technical summary
    section 2.B: k = (1 - r_l)|S| with r_l the skip rate and S all positions),
    clamped to [1, L]; 1e-9 absorbs float noise just above an integer."""
    return max(1, min(length, int(math.ceil(keep_ratio * length - 1e-9))))


def _rank_keys(s: np.ndarray):
    s = np.asarray(s, dtype=np.float32).astype(np.float64)
    s = np.where(s == 0.0, 0.0, s)          # -0 -> +0
    nan = np.isnan(s)
    s = np.where(nan, 0.0, s)
    return nan, s


def topk_select(s: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k highest scores of one sequence, in ascending order.

    Total order: NaN last, then score descending, then index ascending.
    """
    nan, sv = _rank_keys(s)
    order = np.lexsort((np.arange(sv.shape[0]), -sv, nan))
    return np.sort(order[:k]).astype(np.int32)


def topk_margin(s: np.ndarray, k: int) -> float:
    """Gap between the k-th and (k+1)-th ranked scores (inf when k == L)."""
    nan, sv = _rank_keys(s)
    if k >= sv.shape[0]:
        return math.inf
    order = np.lexsort((np.arange(sv.shape[0]), -sv, nan))
    return float(sv[order[k - 1]] - sv[order[k]])


def remask(tok, masked, conf_c, tok_c, b0: int, b1: int, n: int):
    """Unmask the n most confident masked positions of block [b0, b1) of one sequence.

    "ES-dLLM", technical summary section 1: only the highest-confidence masked
    tokens are unmasked at each step. Candidates are the masked positions of
    the current block; ties go to the lower position; if fewer than n remain,
    all are unmasked. Updates tok/masked in place; returns (positions, margin).
    """
    cand = np.array([i for i in range(b0, b1) if masked[i]], dtype=np.int64)
    if cand.size == 0:
        return cand, math.inf
    c = np.asarray(conf_c, dtype=np.float32)[cand].astype(np.float64)
    order = np.lexsort((cand, -c))
    pick = cand[order[:n]]
    tok[pick] = tok_c[pick]
    masked[pick] = 0
    margin = math.inf if cand.size <= n else float(c[order[n - 1]] - c[order[n]])
    return np.sort(pick), margin


# --------------------------------------------------------------------------
# the step and the generation loop
# --------------------------------------------------------------------------
@dataclasses.dataclass
class State:
    tok: np.ndarray       # [B, L] int32
    masked: np.ndarray    # [B, L] uint8
    hc: np.ndarray        # [B, L, d]   hidden-state cache at the skip layer
    hc2: np.ndarray       # [B, L, d]   hidden-state cache at the second skip layer (if any)
    kc: list              # [N - l_s] of [B, L, H, hd]
    vc: list
    conf_c: np.ndarray    # [B, L] float32 values
    tok_c: np.ndarray     # [B, L] int32

    def copy(self) -> "State":
        return State(self.tok.copy(), self.masked.copy(), self.hc.copy(), self.hc2.copy(),
                     [a.copy() for a in self.kc], [a.copy() for a in self.vc],
                     self.conf_c.copy(), self.tok_c.copy())


def cache_base(run: RunConfig) -> int:
    """First layer with a K/V cache: the skip layer, or 0 when the selection
    is scoped to the current block (every layer then reuses the other rows'
    cached K/V)."""
    return 0 if run.scope in ("block", "response") else run.skip_layer


def new_state(dims: ModelDims, run: RunConfig, tok: np.ndarray, masked: np.ndarray) -> State:
    B, L = tok.shape
    nc = dims.n_layers - cache_base(run)
    shp = (B, L, dims.n_heads, dims.head_dim)
    return State(tok.astype(np.int32).copy(), masked.astype(np.uint8).copy(),
                 np.zeros((B, L, dims.d)), np.zeros((B, L, dims.d)), [np.zeros(shp) for _ in range(nc)],
                 [np.zeros(shp) for _ in range(nc)], np.zeros((B, L)),
                 np.zeros((B, L), dtype=np.int32))


def embed(tok_row: np.ndarray, w: dict) -> np.ndarray:
    return w["embed"][tok_row].copy()


def dense_step(w: dict, dims: ModelDims, run: RunConfig, st: State,
               b0: int, b1: int, n: int) -> dict:
    """Dense refresh: every layer on every row; refills H, all K/V caches and
    every confidence/prediction, then remasks ("ES-dLLM", technical summary
    section 2.B: periodic full refresh)."""
    B = st.tok.shape[0]
    ls = run.skip_layer
    base = cache_base(run)
    info = {"dense": True, "argmax_margin": [], "remask_margin": [], "unmasked": [],
            "row_margin": [], "row_scale": []}
    for b in range(B):
        x = embed(st.tok[b], w)
        for layer in range(dims.n_layers):
            if layer == ls:
                st.hc[b] = x
            if run.skip_layer2 and layer == run.skip_layer2:
                st.hc2[b] = x
            x, k, v = dense_layer(x, w["layers"][layer], dims)
            if layer >= base:
                st.kc[layer - base][b] = k
                st.vc[layer - base][b] = v
        conf, tp, mg = head(x, w["w_out"], dims)
        st.conf_c[b] = conf
        st.tok_c[b] = tp
        info["argmax_margin"].append(float(mg.min()))
        info["row_margin"].append(mg)
        info["row_scale"].append(logit_scale(x, w["w_out"], dims))
    for b in range(B):
        pick, mg = remask(st.tok[b], st.masked[b], st.conf_c[b], st.tok_c[b], b0, b1, n)
        info["unmasked"].append(pick)
        info["remask_margin"].append(mg)
    return info


def sparse_step(w: dict, dims: ModelDims, run: RunConfig, st: State,
                b0: int, b1: int, n: int, k: int | None = None,
                idx_override=None, region=None) -> dict:
    """Early-skipping step ("ES-dLLM", technical summary section 2.B).

    Layers below l_s on all rows; importance scores at l_s; per-sequence top-k;
    H cache scatter; the selected rows through layers l_s..N-1 with K/V
    scatter and partial attention; head on the selected rows with the
    confidence/prediction scatter; remask. ``idx_override`` [B, k] replaces
    the selection (teacher forcing).

    With a second skip point l_s2 (section 2.B: skipping at early layers such
    as 4 and 8 of 32; k = (1 - r_l)|S| with S the tokens that reach layer l),
    the k selected rows run layers l_s..l_s2-1, are scored again at l_s2
    against the second H cache and the cached confidence, the top
    k2 = ceil(keep_ratio2 * k) of them (per sequence) update that cache and
    continue through l_s2..N-1 and the head; the others keep their caches
    from l_s2 on.

    With the selection scoped to the current block [b0, b1) (the block-wise
    cache of the DualCache comparison, section 2.B: refresh "the prompt or the
    current block"), S is the block: the early layers run on the block's rows
    only, attending over every layer's K/V cache with the block's fresh K/V
    scattered in, and k = ceil(keep_ratio * (b1 - b0)) of the block's rows are
    selected.

    Response-only steps ("DyLLM", technical summary section 2.B.3: only the
    response tokens are processed, the whole context only every few steps):
    with scope "response" the recomputed region is ``region`` = (P, L), the
    positions after the prompt, handled as the block scope handles its block
    (the prompt rows' K/V are those of the last full step); unmasking stays
    within the current block [b0, b1).
    """
    B, L = st.tok.shape
    ls = run.skip_layer
    base = cache_base(run)
    block = run.scope in ("block", "response")
    if run.scope == "response":
        assert region is not None, "a response-only step needs its region (P, L)"
        r0, r1 = region
    else:
        r0, r1 = (b0, b1) if region is None else region
    pos = np.arange(r0, r1) if block else np.arange(L)
    if k is None:
        k = keep_count(run.keep_ratio, len(pos))
    info = {"dense": False, "scores": [], "idx": [], "x_ls": [], "xs_out": [],
            "topk_margin": [], "argmax_margin": [], "remask_margin": [], "unmasked": [],
            "row_margin": [], "row_scale": []}
    for b in range(B):
        x = embed(st.tok[b], w)
        if block:
            x = x[pos]
            for layer in range(ls):
                x = sparse_layer(x, pos, st.kc[layer][b], st.vc[layer][b], w["layers"][layer], dims)
        else:
            for layer in range(ls):
                x, _, _ = dense_layer(x, w["layers"][layer], dims)
        if block:
            assert run.score_tensor == "h", "block scope scores the hidden state"
            s = importance(x, st.hc[b][pos], st.conf_c[b][pos], run)
        elif run.score_tensor == "h":
            s = importance(x, st.hc[b], st.conf_c[b], run)
        else:
            # the variation of the skip layer's keys or values ("ES-dLLM",
            # technical summary section 2.A: H, K or V can carry the score),
            # against that layer's K/V cache
            _, k_all, v_all = _qkv(x, np.arange(L), w["layers"][ls], dims)
            fresh, cache = ((k_all, st.kc[ls - base][b]) if run.score_tensor == "k"
                            else (v_all, st.vc[ls - base][b]))
            s = importance(fresh.reshape(L, dims.d), cache.reshape(L, dims.d), st.conf_c[b], run)
        if idx_override is None:
            j = topk_select(s, k)
        else:
            j = np.searchsorted(pos, np.asarray(idx_override[b], dtype=np.int32))
        idx = pos[j].astype(np.int32)
        info["scores"].append(s)
        info["idx"].append(idx)
        info["x_ls"].append(x)
        info["topk_margin"].append(topk_margin(s, k))
        st.hc[b][idx] = x[j]
        xs = x[j]
        ls2 = run.skip_layer2 if run.skip_layer2 else dims.n_layers
        for layer in range(ls, ls2):
            xs = sparse_layer(xs, idx, st.kc[layer - base][b], st.vc[layer - base][b],
                              w["layers"][layer], dims)
        if run.skip_layer2:
            s2 = importance(xs, st.hc2[b][idx], st.conf_c[b][idx], run)
            k2 = keep_count(run.keep_ratio2, len(idx))
            j2 = topk_select(s2, k2)
            info.setdefault("scores2", []).append(s2)
            info.setdefault("topk2_margin", []).append(topk_margin(s2, k2))
            idx = idx[j2]
            xs = xs[j2]
            st.hc2[b][idx] = xs
            info.setdefault("idx2", []).append(idx)
        for layer in range(ls2, dims.n_layers):
            xs = sparse_layer(xs, idx, st.kc[layer - base][b], st.vc[layer - base][b],
                              w["layers"][layer], dims)
        info["xs_out"].append(xs)
        conf, tp, mg = head(xs, w["w_out"], dims)
        st.conf_c[b][idx] = conf
        st.tok_c[b][idx] = tp
        info["argmax_margin"].append(float(mg.min()))
        info["row_margin"].append(mg)
        info["row_scale"].append(logit_scale(xs, w["w_out"], dims))
    for b in range(B):
        pick, mg = remask(st.tok[b], st.masked[b], st.conf_c[b], st.tok_c[b], b0, b1, n)
        info["unmasked"].append(pick)
        info["remask_margin"].append(mg)
    return info


def generate(w: dict, dims: ModelDims, run: RunConfig, prompt: np.ndarray, gen: int,
             block: int, n_unmask: int, vanilla: bool = False, k: int | None = None):
    """Block-wise generation: prompt followed by ``gen`` mask tokens, blocks of
    ``block`` positions, ``block // n_unmask`` steps per block. A step is
    dense at the first step of a block (and every refresh_interval steps), or
    at every step when ``vanilla`` (every token recomputed every iteration).
    Returns (generated ids [B, gen], per-step info list)."""
    B, P = prompt.shape
    L = P + gen
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = prompt
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    st = new_state(dims, run, tok, masked)
    log = []
    steps = block // n_unmask
    for blk in range(gen // block):
        b0 = P + blk * block
        b1 = b0 + block
        for j in range(steps):
            dense = vanilla or j == 0 or (run.refresh_interval > 0 and j % run.refresh_interval == 0)
            if dense:
                log.append(dense_step(w, dims, run, st, b0, b1, n_unmask))
            else:
                log.append(sparse_step(w, dims, run, st, b0, b1, n_unmask, k=k,
                                       region=(P, L) if run.scope == "response" else None))
    return st.tok[:, P:].copy(), log
