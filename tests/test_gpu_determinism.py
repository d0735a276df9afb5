"""Run-twice bitwise determinism of the CUDA path (the stand-in for a race
detector, which is not available on the test machines): the same sparse
layer, or the same whole denoising step, run twice from byte-identical inputs
and caches must give byte-identical outputs and caches. The kernels that
combine partial results across CTAs (the cluster split-K GEMMs through
distributed shared memory, the stream-K fix-ups, the key-split attention's
last-ticket merge) add the partials in a fixed order, so any difference
means a race or an order that depends on timing.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import make_context, to_gpu

pytestmark = pytest.mark.gpu

FULL = dataclasses.replace(synth.M8B, n_layers=5, vocab=8192, mask_id=8191)  # 8B layer shapes
L = 768


@pytest.fixture(scope="module")
def full():
    import synth.gpu as sg
    import token_skipping_sparse_step_b200 as esd
    w = sg.model_weights(FULL)
    run = synth.M8B_RUN
    ctx = esd.Context(esd.make_dims(FULL.n_layers, FULL.d, FULL.n_heads, FULL.head_dim, FULL.ffn, FULL.vocab,
                                    FULL.mask_id, FULL.rope_theta, FULL.rms_eps, FULL.dtype),
                      w, esd.make_run(run.score_mode, run.alpha, run.lam, run.skip_layer, run.keep_ratio, 0, 1, L))
    yield ctx
    ctx.close()


@pytest.mark.parametrize("k", [192, 1, 37])
def test_8b_sparse_layer_twice_bit_identical(full, k):
    """Layer 4 of the 8B shapes on k selected rows of L = 768 (k = 192: the
    benchmark's row count; k = 1: one query, attention split over the keys),
    twice from the same inputs and K/V cache: every output byte and every
    cache byte equal."""
    ctx = full
    rng = np.random.default_rng(40 + k)
    ls = synth.M8B_RUN.skip_layer
    x = to_gpu(O.store(rng.standard_normal((k, FULL.d)) * 0.5, "bf16"), torch.bfloat16)
    kc = to_gpu(O.store(rng.standard_normal((1, L, FULL.d)), "bf16"), torch.bfloat16)
    vc = to_gpu(O.store(rng.standard_normal((1, L, FULL.d)), "bf16"), torch.bfloat16)
    idx = to_gpu(np.sort(rng.choice(L, k, replace=False)).astype(np.int32), torch.int32)
    v = ctx.state(1, L)
    outs = []
    for _ in range(2):
        v["k_cache"][0].copy_(kc.view_as(v["k_cache"][0]))
        v["v_cache"][0].copy_(vc.view_as(v["v_cache"][0]))
        xs = x.clone()
        ctx.sparse_layers_forward(ls, ls + 1, idx, 1, L, k, xs)
        ctx.sync_check()
        outs.append((xs.clone(), v["k_cache"][0].clone(), v["v_cache"][0].clone()))
    for a, b, what in zip(outs[0], outs[1], ("output rows", "K cache", "V cache")):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), what


def _snapshot(v):
    return {k_: (x.clone() if torch.is_tensor(x) else [y.clone() for y in x]) for k_, x in v.items()
            if k_ in ("h_cache", "k_cache", "v_cache", "conf_cache", "tok_cache")}


def _restore(v, snap):
    for k_, x in snap.items():
        if torch.is_tensor(x):
            v[k_].copy_(x)
        else:
            for a, b in zip(v[k_], x):
                a.copy_(b)


def test_8b_sparse_denoise_step_twice_bit_identical(full):
    """A whole early-skipping step (dense early layers, score, top-k, gather,
    the sparse layer, head, remask) at L = 768, twice from the caches a dense
    step left: every cache byte and the tokens equal."""
    ctx = full
    P, blk = 736, 32
    tok = torch.full((1, L), FULL.mask_id, dtype=torch.int32, device="cuda")
    tok[:, :P] = torch.from_numpy(synth.prompt_ids(FULL, 1, P)).cuda()
    msk = torch.zeros((1, L), dtype=torch.uint8, device="cuda")
    msk[:, P:] = 1
    ctx.denoise_step(tok, msk, P, P + blk, 1, force_dense=True)
    ctx.sync_check()
    v = ctx.state(1, L)
    snap = _snapshot(v)
    t0, m0 = tok.clone(), msk.clone()
    res = []
    for _ in range(2):
        _restore(v, snap)
        t, m = t0.clone(), m0.clone()
        ctx.denoise_step(t, m, P, P + blk, 1, force_dense=False)
        ctx.sync_check()
        res.append((t, m, _snapshot(v)))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    for k_ in res[0][2]:
        a, b = res[0][2][k_], res[1][2][k_]
        if torch.is_tensor(a):
            assert torch.equal(a, b), k_
        else:
            for i, (x, y) in enumerate(zip(a, b)):
                assert torch.equal(x, y), (k_, i)


def test_small_block_scope_step_twice_bit_identical():
    """The block-scoped step (every layer on the block's rows, K/V scattered
    into every layer's cache) twice from the same caches."""
    dims = synth.SMALL_BF16
    run = dataclasses.replace(synth.SMALL_BF16_RUN, scope="block")
    B, P, G = 2, 96, 64
    ctx, _ = make_context(dims, run, B, P + G)
    tok = torch.full((B, P + G), dims.mask_id, dtype=torch.int32, device="cuda")
    tok[:, :P] = torch.from_numpy(synth.prompt_ids(dims, B, P)).cuda()
    msk = torch.zeros((B, P + G), dtype=torch.uint8, device="cuda")
    msk[:, P:] = 1
    ctx.denoise_step(tok, msk, P, P + 32, 2, force_dense=True)
    v = ctx.state(B, P + G)
    snap = _snapshot(v)
    res = []
    for _ in range(2):
        _restore(v, snap)
        t, m = tok.clone(), msk.clone()
        ctx.denoise_step(t, m, P, P + 32, 2, force_dense=False)
        ctx.sync_check()
        res.append((t, _snapshot(v)))
    assert torch.equal(res[0][0], res[1][0])
    for k_ in res[0][1]:
        a, b = res[0][1][k_], res[1][1][k_]
        pairs = [(a, b)] if torch.is_tensor(a) else list(zip(a, b))
        for x, y in pairs:
            assert torch.equal(x, y), k_
    ctx.close()
