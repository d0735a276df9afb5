"""Context saliency on the GPU ("DyLLM: Efficient Diffusion LLM Inference via
Saliency-based Token Selection and Partial Attention", technical summary
sections 2.A and 2.B.1) against the oracle: the float32 cosine of every row's
attention context with the previous step's, and per sequence the rows below
the layer's threshold in ascending order.

The salient set is an integer decided by floating point, so it is compared
bit-exactly with the oracle's rule applied to the kernel's own float32
similarities (same precision, same decision), and with the oracle's float64
similarities on every row that is not within the float32 tolerance of tau.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import TOL, assert_parity, make_context, to_gpu, to_np

pytestmark = pytest.mark.gpu


def _contexts(rng, B, L, d, dtype):
    """Rows of every kind: unchanged, rescaled, slightly and strongly moved,
    fresh, zero, anti-parallel."""
    prev = rng.standard_normal((B * L, d))
    kind = rng.integers(0, 7, B * L)
    cur = prev.copy()
    cur[kind == 1] *= 2.5
    cur[kind == 2] += 0.05 * rng.standard_normal(((kind == 2).sum(), d))
    cur[kind == 3] += 0.8 * rng.standard_normal(((kind == 3).sum(), d))
    cur[kind == 4] = rng.standard_normal(((kind == 4).sum(), d))
    cur[kind == 5] = 0.0
    cur[kind == 6] *= -1.0
    return O.store(cur, dtype), O.store(prev, dtype), kind


def _check(ctx, cur, prev, B, L, tau, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sim = torch.empty(B * L, dtype=torch.float32, device="cuda")
    idx = torch.full((B * L,), 7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    ctx.context_saliency(to_gpu(cur, tdt), to_gpu(prev, tdt), B, L, tau, idx, cnt, sim_out=sim)
    ctx.sync_check()
    g_sim, g_idx, g_cnt = to_np(sim), to_np(idx).reshape(B, L), to_np(cnt)
    want = O.context_cosine(cur, prev)
    assert_parity(g_sim, want, "f32", "context cosine")
    for b in range(B):
        rows = slice(b * L, (b + 1) * L)
        own = O.salient_rows(g_sim[rows], tau)              # the kernel's similarities
        assert g_cnt[b] == len(own)
        assert np.array_equal(g_idx[b, :len(own)], own)
        assert np.all(g_idx[b, len(own):] == -1)
        ref = O.salient_rows(want[rows], tau)              # the oracle's similarities
        clear = np.abs(want[rows].astype(np.float64) - np.float32(tau)) > 2 * TOL["f32"]
        assert np.array_equal(np.isin(np.arange(L), own)[clear], np.isin(np.arange(L), ref)[clear])
    return g_sim


@pytest.mark.parametrize("model", ["tiny", "small"])
@pytest.mark.parametrize("B,L", [(1, 1), (3, 1000), (2, 128)])
def test_context_saliency_matches_oracle(model, B, L):
    dims = synth.TINY if model == "tiny" else synth.SMALL_BF16
    run = synth.TINY_RUN if model == "tiny" else synth.SMALL_BF16_RUN
    ctx, _ = make_context(dims, run, 3, 1024)
    rng = np.random.default_rng(B * 7919 + L)
    cur, prev, kind = _contexts(rng, B, L, dims.d, dims.dtype)
    for tau in (0.9, 0.5, 1.0, 1.01, -1.0):
        g_sim = _check(ctx, cur, prev, B, L, tau, dims.dtype)
    assert np.all(g_sim[kind == 0] == 1.0)      # unchanged rows: exactly 1, never salient for tau <= 1
    assert np.all(g_sim[kind == 5] == 0.0)      # zero rows: floored denominator
    ctx.close()


def test_context_saliency_microbenchmark_shape():
    """B 16, S 4096, d 4096 bf16 (the microbenchmark tensors: 10% of rows
    replaced by fresh draws): sampled rows against the oracle; the salient set
    against the kernel's own similarities; the fresh rows are the salient ones
    at tau 0.9."""
    import synth.gpu as sg
    import token_skipping_sparse_step_b200 as esd
    B, S, d = synth.MICRO["batch"], synth.MICRO["seq"], synth.MICRO["d"]
    dims = synth.ModelDims(2, d, 32, 128, 256, 1024, 1023, 5e5, 1e-6, "bf16")
    ctx = esd.Context(esd.make_dims(2, d, 32, 128, 256, 1024, 1023, 5e5, 1e-6, "bf16"),
                      sg.model_weights(dims), esd.make_run("es", 0.5, 0.5, 1, 0.25, 0, B, S))
    x, h, _ = sg.micro_inputs(B, S, d)
    sim = torch.empty(B * S, dtype=torch.float32, device="cuda")
    idx = torch.empty(B * S, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    ctx.context_saliency(x, h, B, S, 0.9, idx, cnt, sim_out=sim)
    ctx.sync_check()
    rows = np.array([0, 5, 4095, 4096, 30000, 65535])
    xr, hr, _ = synth.micro_rows(B, S, d, rows)
    assert_parity(to_np(sim)[rows], O.context_cosine(O.store(xr, "bf16"), O.store(hr, "bf16")), "f32", "cosine")
    g_sim, g_idx, g_cnt = to_np(sim).reshape(B, S), to_np(idx).reshape(B, S), to_np(cnt)
    for b in range(B):
        own = O.salient_rows(g_sim[b], 0.9)
        assert g_cnt[b] == len(own) and np.array_equal(g_idx[b, :len(own)], own)
        assert np.all(g_idx[b, len(own):] == -1)
    frac = g_cnt.sum() / (B * S)
    assert 0.05 < frac < 0.15, frac            # ~10% fresh rows, cosine ~0; the rest ~1
    ctx.close()
