"""The DyLLM token-selection layers as CUDA graphs ("DyLLM: Efficient
Diffusion LLM Inference via Saliency-based Token Selection and Partial
Attention", technical summary sections 2.A, 2.B.1 and 2.B.2).

A non-refresh call picks the row capacity of its output projection and SwiGLU
block (and, with the approximate attention, of its moved rows) on the device,
in a switch node of a graph. These tests check that side of it:
* salient counts on both sides of every kind of capacity edge (none, one,
  16 and 17, 256 and 257, all rows) against the oracle, from the same layer
  state each time;
* a graph replayed from the cache gives, bit for bit, what a freshly captured
  one gives, and device-side counts equal the host-side ones.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import assert_parity, make_context, to_gpu, to_np

pytestmark = pytest.mark.gpu


def _peaked_weights(dims):
    # larger query and key weights: peaked attention, so that the contexts of
    # different rows move by different amounts
    w32 = synth.model_weights_f32(dims)
    for lw in w32["layers"]:
        lw["wq"] = lw["wq"] * 4.0
        lw["wk"] = lw["wk"] * 4.0
    return w32


def test_dyllm_salient_counts_at_capacity_edges():
    """One bf16 layer over 300 rows (capacities 16, 32, ..., 256 on the
    swapped-operand GEMMs, then 300 on the SM-pair GEMMs). For each target
    count m the layer is refreshed with x0, probed with x1 and nothing salient
    (to read the similarities), refreshed again (the same state, bit for bit),
    and run with x1 and a threshold that makes exactly the m least similar
    rows salient. The salient rows must match the oracle's layer with that
    salient set; the others keep the refresh's outputs bit for bit."""
    dims, run = synth.SMALL_BF16, synth.SMALL_BF16_RUN
    B, L = 1, 300
    ctx, w = make_context(dims, run, 1, L, w32=_peaked_weights(dims))
    rng = np.random.default_rng(47)
    x0 = O.store(rng.standard_normal((L, dims.d)), "bf16")
    x1 = O.store(x0 + np.linspace(0.0, 1.0, L)[:, None] * rng.standard_normal((L, dims.d)), "bf16")
    tr0 = {}
    out0, c0, _, _ = O.dyllm_layer(x0, w["layers"][0], dims, None, None, 0.0, True, trace=tr0)
    sim = torch.empty(B * L, dtype=torch.float32, device="cuda")
    probe = None
    for m in (0, 1, 15, 16, 17, 255, 256, 257, 299, 300):
        xr = to_gpu(x0, torch.bfloat16)
        ctx.dyllm_layers_forward(0, 1, xr, B, L, refresh=True)
        if probe is None:
            refreshed = xr.clone()
            xp = to_gpu(x1, torch.bfloat16)
            counts = ctx.dyllm_layers_forward(0, 1, xp, B, L, [-2.0], refresh=False, sim_out=sim)
            assert counts.sum() == 0
            probe = sim.clone()
            ctx.dyllm_layers_forward(0, 1, to_gpu(x0, torch.bfloat16), B, L, refresh=True)
        else:
            assert torch.equal(xr, refreshed)
        srt = np.sort(to_np(probe))
        assert len(np.unique(srt)) == L, "tied similarities: pick another seed"
        tau = -2.0 if m == 0 else (2.0 if m == L else float(0.5 * (srt[m - 1] + srt[m])))
        xg = to_gpu(x1, torch.bfloat16)
        counts = ctx.dyllm_layers_forward(0, 1, xg, B, L, [tau], refresh=False, sim_out=sim)
        ctx.sync_check()
        assert torch.equal(sim, probe), m
        assert counts[0, 0] == m
        g_set = O.salient_rows(to_np(sim), tau)
        assert len(g_set) == m
        tr = {}
        want, _, _, _ = O.dyllm_layer(x1, w["layers"][0], dims, c0, out0, tau, False, salient=g_set, trace=tr)
        got = to_np(xg)
        terms = tr0["salient_terms"].copy()
        if m:
            terms[g_set] = tr["salient_terms"]
        assert_parity(got, want, "bf16", f"{m} salient rows", terms=terms)
        others = np.setdiff1d(np.arange(L), g_set)
        assert np.array_equal(got[others], to_np(refreshed)[others]), m
    ctx.close()


@pytest.mark.parametrize("approx", [False, True])
def test_dyllm_graph_replay_and_device_counts(approx):
    """Two contexts, the same calls: a refresh, then eight steps whose input
    alternates between two tensors (every 3rd row differs), with per-layer
    thresholds at the median similarity. Context A passes a new sim_out
    tensor every step, so each step captures a new graph, and reads the
    counts into host memory; context B passes the same sim_out and reads the
    counts into device memory, so from its third step on the graphs come from
    its cache. Every output, similarity and count must agree bit for bit."""
    dims, run = synth.SMALL_BF16, synth.SMALL_BF16_RUN
    B, L = 2, 100
    n = dims.n_layers
    w32 = _peaked_weights(dims)
    ctx_a, _ = make_context(dims, run, B, 128, w32=w32)
    ctx_b, _ = make_context(dims, run, B, 128, w32=w32)
    rng = np.random.default_rng(53)
    x0 = to_gpu(O.store(rng.standard_normal((B * L, dims.d)), "bf16"), torch.bfloat16)
    x1 = x0.clone()
    x1[::3] = to_gpu(O.store(rng.standard_normal((len(range(0, B * L, 3)), dims.d)), "bf16"), torch.bfloat16)
    xa, xb = x0.clone(), x0.clone()
    ctx_a.dyllm_layers_forward(0, n, xa, B, L, refresh=True, approx=approx)
    ctx_b.dyllm_layers_forward(0, n, xb, B, L, refresh=True, approx=approx)
    # thresholds: the median similarity of a step to x1 with every row salient
    probe = torch.empty(n * B * L, dtype=torch.float32, device="cuda")
    xa.copy_(x1)
    xb.copy_(x1)
    ctx_a.dyllm_layers_forward(0, n, xa, B, L, [2.0] * n, refresh=False, sim_out=probe, approx=approx)
    ctx_b.dyllm_layers_forward(0, n, xb, B, L, [2.0] * n, refresh=False, approx=approx)
    assert torch.equal(xa, xb)
    taus = [float(torch.median(probe[l * B * L:(l + 1) * B * L])) for l in range(n)]
    sims_a = [torch.empty(n * B * L, dtype=torch.float32, device="cuda") for _ in range(8)]
    sim_b = torch.empty(n * B * L, dtype=torch.float32, device="cuda")
    cnt_b = torch.zeros((n, B), dtype=torch.int32, device="cuda")
    total = 0
    for i in range(8):
        src = x0 if i % 2 == 0 else x1
        xa.copy_(src)
        xb.copy_(src)
        ca = ctx_a.dyllm_layers_forward(0, n, xa, B, L, taus, refresh=False, sim_out=sims_a[i], approx=approx)
        ctx_b.dyllm_layers_forward(0, n, xb, B, L, taus, refresh=False, sim_out=sim_b, approx=approx,
                                   counts_out=cnt_b)
        ctx_a.sync_check()
        ctx_b.sync_check()
        assert np.array_equal(ca, cnt_b.cpu().numpy()), i
        assert torch.equal(sims_a[i], sim_b), i
        assert torch.equal(xa, xb), i
        total += int(ca.sum())
    assert 0 < total < 8 * n * B * L
    ctx_a.close()
    ctx_b.close()
