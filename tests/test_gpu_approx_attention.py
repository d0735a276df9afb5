"""Saliency-aware approximate attention on the GPU ("DyLLM: Efficient Diffusion
LLM Inference via Saliency-based Token Selection and Partial Attention",
technical summary section 2.B.2) against the oracle's approx_contexts, through
esd_approx_attention: the rows whose values moved get exact attention rows
(and their cached probabilities rewritten), every other row moves its cached
context by sum_j P_ij (V_j - V_prev_j) over the moved rows.

Contexts within the model's tolerance, probabilities (float32 arithmetic on
both models) within the float32 tolerance, the probability rows of unmoved
tokens bit-identical, and no moved row at all leaves the contexts bit-identical.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import TOL, assert_parity, make_context, to_gpu, to_np

pytestmark = pytest.mark.gpu


def _softmax_rows(rng, B, H, L):
    lg = rng.standard_normal((B, H, L, L)) * 2.0
    e = np.exp(lg - lg.max(-1, keepdims=True))
    return (e / e.sum(-1, keepdims=True)).astype(np.float32).astype(np.float64)


def _changed_sets(rng, kind, B, L):
    sets = []
    for b in range(B):
        if kind == "none":
            s = np.array([], dtype=np.int64)
        elif kind == "all":
            s = np.arange(L)
        elif kind == "last":
            s = np.array([L - 1])
        elif kind == "mixed":                      # sequence 0 none, sequence 1 every row
            s = np.array([], dtype=np.int64) if b == 0 else np.arange(L)
        else:                                      # a different third of the rows per sequence
            s = np.sort(rng.choice(L, max(1, L // 3), replace=False))
        sets.append(s)
    return sets


def _device_list(sets, B, L):
    idx = np.full((B, L), -1, dtype=np.int32)
    cnt = np.zeros(B, dtype=np.int32)
    for b, s in enumerate(sets):
        idx[b, :len(s)] = s
        cnt[b] = len(s)
    return to_gpu(idx, torch.int32), to_gpu(cnt, torch.int32)


def _run(ctx, dims, q, k, v, v_prev, c_prev, p_prev, sets, B, L):
    tdt = torch.bfloat16 if dims.dtype == "bf16" else torch.float32
    flat = lambda a: to_gpu(a.reshape(B * L, dims.d), tdt)
    idx, cnt = _device_list(sets, B, L)
    c = flat(c_prev)
    p = to_gpu(p_prev, torch.float32)
    ctx.approx_attention(flat(q), flat(k), flat(v), flat(v_prev), idx, cnt, B, L, c, p)
    ctx.sync_check()
    return c, p


@pytest.mark.parametrize("model", ["tiny", "small"])
@pytest.mark.parametrize("L", [1, 100, 300])
@pytest.mark.parametrize("kind", ["none", "some", "all", "last", "mixed"])
def test_approx_attention_matches_oracle(model, L, kind):
    dims = synth.TINY if model == "tiny" else synth.SMALL_BF16
    run = synth.TINY_RUN if model == "tiny" else synth.SMALL_BF16_RUN
    B, H, hd = 2, dims.n_heads, dims.head_dim
    ctx, _ = make_context(dims, run, 2, 320)
    rng = np.random.default_rng(L * 31 + len(kind))
    shape = (B, L, H, hd)
    q, k, v = (O.store(rng.standard_normal(shape), dims.dtype) for _ in range(3))
    c_prev = O.store(rng.standard_normal(shape), dims.dtype)
    p_prev = _softmax_rows(rng, B, H, L)
    sets = _changed_sets(rng, kind, B, L)
    v_prev = v.copy()
    for b, s in enumerate(sets):
        v_prev[b, s] = O.store(v[b, s] + rng.standard_normal((len(s), H, hd)), dims.dtype)
    c, p = _run(ctx, dims, q, k, v, v_prev, c_prev, p_prev, sets, B, L)
    g_c, g_p = to_np(c).reshape(shape), to_np(p)
    for b, s in enumerate(sets):
        o_c, o_p = O.approx_contexts(q[b], k[b], v[b], v_prev[b], c_prev[b], p_prev[b], s)
        assert_parity(g_c[b], o_c, dims.dtype, f"contexts, sequence {b}")
        assert_parity(g_p[b], o_p, "f32", f"probabilities, sequence {b}")
        rest = np.setdiff1d(np.arange(L), s)
        assert np.array_equal(g_p[b][:, rest], p_prev[b][:, rest])   # unmoved rows untouched
        if len(s) == 0:
            assert np.array_equal(g_c[b], c_prev[b])                 # nothing moved: bit-identical
        else:
            assert np.allclose(g_p[b][:, s].sum(-1), 1.0, atol=1e-5)   # fresh rows are distributions
    ctx.close()


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_approx_attention_exact_when_queries_and_keys_stay(model):
    """Queries and keys unchanged, cached probabilities and contexts exact for
    the previous values, every moved value row listed: the update is exact for
    every row, so the result is full attention over the new values."""
    dims = synth.TINY if model == "tiny" else synth.SMALL_BF16
    run = synth.TINY_RUN if model == "tiny" else synth.SMALL_BF16_RUN
    B, L, H, hd = 2, 200, dims.n_heads, dims.head_dim
    ctx, _ = make_context(dims, run, 2, 256)
    rng = np.random.default_rng(5)
    shape = (B, L, H, hd)
    q, k, v_prev = (O.store(rng.standard_normal(shape), dims.dtype) for _ in range(3))
    sets = _changed_sets(rng, "some", B, L)
    v = v_prev.copy()
    for b, s in enumerate(sets):
        v[b, s] = O.store(rng.standard_normal((len(s), H, hd)), dims.dtype)
    p_prev = np.empty((B, H, L, L))
    c_prev = np.empty(shape)
    for b in range(B):
        sc = np.einsum("ihd,jhd->hij", q[b], k[b]) / math.sqrt(hd)
        e = np.exp(sc - sc.max(-1, keepdims=True))
        p_prev[b] = (e / e.sum(-1, keepdims=True)).astype(np.float32)
        c_prev[b] = O.store(O.attention(q[b], k[b], v_prev[b]), dims.dtype)
    c, _ = _run(ctx, dims, q, k, v, v_prev, c_prev, p_prev, sets, B, L)
    g_c = to_np(c).reshape(shape)
    for b in range(B):
        assert_parity(g_c[b], O.attention(q[b], k[b], v[b]), dims.dtype, f"sequence {b}")
    ctx.close()


def test_approx_attention_checks_its_lists():
    """A changed list out of order and a count above L are skipped on the
    device (no access outside the buffers) and reported as ESD_ERR_CHECK; the
    context keeps working. Bad host arguments are rejected before any launch."""
    import token_skipping_sparse_step_b200 as esd
    dims, run = synth.SMALL_BF16, synth.SMALL_BF16_RUN
    B, L = 2, 64
    ctx, _ = make_context(dims, run, 2, 128)
    x = torch.zeros((B * L, dims.d), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros_like(x)
    p = torch.zeros((B, dims.n_heads, L, L), dtype=torch.float32, device="cuda")
    idx = torch.tensor([[3, 2] + [-1] * (L - 2), [0, 1] + [-1] * (L - 2)], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([2, 2], dtype=torch.int32, device="cuda")
    ctx.approx_attention(x, x, x, x, idx, cnt, B, L, c, p)
    with pytest.raises(esd.EsdError) as err:
        ctx.sync_check()
    assert err.value.status == 6  # ESD_ERR_CHECK
    cnt_bad = torch.tensor([0, L + 1], dtype=torch.int32, device="cuda")
    ctx.approx_attention(x, x, x, x, idx, cnt_bad, B, L, c, p)
    with pytest.raises(esd.EsdError) as err:
        ctx.sync_check()
    assert err.value.status == 6
    idx_ok = torch.tensor([[0, 5] + [-1] * (L - 2), [1, 2] + [-1] * (L - 2)], dtype=torch.int32, device="cuda")
    ctx.approx_attention(x, x, x, x, idx_ok, cnt, B, L, c, p)
    ctx.sync_check()
    with pytest.raises(esd.EsdError):
        ctx.approx_attention(x, x, x, x, idx_ok, cnt, B, 200, c, p)      # L above max_len
    with pytest.raises(esd.EsdError):
        ctx.approx_attention(x, x, x, None, idx_ok, cnt, B, L, c, p)     # null pointer
    ctx.close()
