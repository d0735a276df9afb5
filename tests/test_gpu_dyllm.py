"""DyLLM token-selection layers on the GPU ("DyLLM: Efficient Diffusion LLM
Inference via Saliency-based Token Selection and Partial Attention", technical
summary sections 2.A and 2.B.1) against the oracle's dyllm_layer.

Three calls on the same context: a refresh (every row recomputed; equals the
dense layers), a step whose input moved, every row by a different amount
(contexts compared with the refresh's under per-layer thresholds that split
the rows about in half, the salient rows recomputed, the others from the
output cache), and a step with that same input again (every context repeats,
so nothing is salient and the output repeats bit for bit). The salient sets are
integers decided by floating point: the oracle takes the GPU's sets
(teacher-forced, derived from the GPU's float32 similarities with the same
rule) to compare hidden states, and the GPU's decisions are checked against
the oracle's own similarities wherever those are clear of tau.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import TOL, assert_parity, make_context, to_gpu, to_np

pytestmark = pytest.mark.gpu


def _oracle_layers(w, dims, x, l0, l1, caches, taus, refresh, salient=None):
    """x [B, L, d] through layers [l0, l1) of the oracle, per sequence;
    caches[(l, b)] = (context, output). Returns (x, sims, salient sets)."""
    B = x.shape[0]
    x = x.copy()
    sims, sets = {}, {}
    for li, l in enumerate(range(l0, l1)):
        for b in range(B):
            c_prev, out_prev = caches.get((l, b), (None, None))
            forced = None if salient is None else salient[(l, b)]
            out, c, sal, sim = O.dyllm_layer(x[b], w["layers"][l], dims, c_prev, out_prev,
                                             0.0 if taus is None else taus[li], refresh, forced)
            caches[(l, b)] = (c, out)
            x[b] = out
            sims[(l, b)], sets[(l, b)] = sim, sal
    return x, sims, sets


def _median_taus(w, dims, x, l0, l1, caches):
    """Per layer, a threshold between the two middle similarities of the
    oracle's own step (so that about half of the rows are salient and none
    sits on tau), found layer by layer on a copy of the caches."""
    caches = dict(caches)
    x = x.copy()
    taus = []
    for l in range(l0, l1):
        sims = [O.dyllm_layer(x[b], w["layers"][l], dims, *caches[(l, b)], -2.0, False)[3]
                for b in range(x.shape[0])]
        srt = np.sort(np.concatenate(sims).astype(np.float64))
        taus.append(float(0.5 * (srt[len(srt) // 2 - 1] + srt[len(srt) // 2])))
        for b in range(x.shape[0]):
            out, c, _, _ = O.dyllm_layer(x[b], w["layers"][l], dims, *caches[(l, b)], taus[-1], False)
            caches[(l, b)] = (c, out)
            x[b] = out
    return taus


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_dyllm_layers_refresh_step_and_repeat(model):
    """Layer by layer, each GPU call fed the oracle's input of that layer
    (teacher forcing at the layer boundaries, so that bf16 rounding flips of
    one layer are not compounded by the next): a refresh, a step whose input
    moved, and the same step again."""
    dims = synth.TINY if model == "tiny" else synth.SMALL_BF16
    run = synth.TINY_RUN if model == "tiny" else synth.SMALL_BF16_RUN
    B, L = 2, 100
    # larger query and key weights: peaked attention, so that the contexts of
    # different rows move by different amounts (x 4 in bf16, whose rounding of
    # q and k would otherwise dominate the softmax of very large logits)
    scale = 20.0 if dims.dtype == "f32" else 4.0
    w32 = synth.model_weights_f32(dims)
    for lw in w32["layers"]:
        lw["wq"] = lw["wq"] * scale
        lw["wk"] = lw["wk"] * scale
    ctx, w = make_context(dims, run, 2, 128, w32=w32)
    tdt = torch.bfloat16 if dims.dtype == "bf16" else torch.float32
    l0, l1 = 0, dims.n_layers
    rng = np.random.default_rng(31)
    x0 = O.store(rng.standard_normal((B, L, dims.d)), dims.dtype)
    caches = {}
    terms = {}  # (layer, seq) -> per-element scale of the cached output rows

    # refresh: every row recomputed = the dense layers
    x_in = x0.copy()
    for l in range(l0, l1):
        xg = to_gpu(x_in.reshape(B * L, dims.d), tdt)
        counts = ctx.dyllm_layers_forward(l, l + 1, xg, B, L, refresh=True)
        ctx.sync_check()
        assert np.all(counts == L)
        want = np.empty_like(x_in)
        for b in range(B):
            tr = {}
            out, c, _, _ = O.dyllm_layer(x_in[b], w["layers"][l], dims, None, None, 0.0, True, trace=tr)
            dense_tr = {}
            assert np.array_equal(out, O.dense_layer(x_in[b], w["layers"][l], dims, trace=dense_tr)[0])
            caches[(l, b)] = (c, out)
            terms[(l, b)] = tr["salient_terms"]
            want[b] = out
        assert_parity(to_np(xg).reshape(B, L, dims.d), want, dims.dtype, f"refresh output layer {l}",
                      terms=np.stack([terms[(l, b)] for b in range(B)]))
        x_in = want

    # a step whose input moved: every row by a different amount
    x1 = O.store(x0 + np.linspace(0.0, 1.0, L)[None, :, None] * rng.standard_normal((B, L, dims.d)),
                 dims.dtype)
    taus = _median_taus(w, dims, x1, l0, l1, caches)
    tol = TOL[dims.dtype]
    sim = torch.empty(B * L, dtype=torch.float32, device="cuda")
    x_in = x1.copy()
    inputs, outs = [], []
    n_salient = 0
    for l in range(l0, l1):
        xg = to_gpu(x_in.reshape(B * L, dims.d), tdt)
        counts = ctx.dyllm_layers_forward(l, l + 1, xg, B, L, [taus[l - l0]], refresh=False, sim_out=sim)
        ctx.sync_check()
        g_sim = to_np(sim).reshape(B, L)
        want = np.empty_like(x_in)
        for b in range(B):
            g_set = O.salient_rows(g_sim[b], taus[l - l0])
            assert counts[0, b] == len(g_set)
            n_salient += len(g_set)
            c_prev, out_prev = caches[(l, b)]
            tr = {}
            out, c, _, s = O.dyllm_layer(x_in[b], w["layers"][l], dims, c_prev, out_prev, taus[l - l0], False,
                                         salient=g_set, trace=tr)
            # similarities, and the GPU's decisions against the oracle's wherever clear of tau
            assert_parity(g_sim[b], s, dims.dtype, f"similarity layer {l}")
            clear = np.abs(s.astype(np.float64) - np.float32(taus[l - l0])) > 2 * tol
            mine = np.isin(np.arange(L), g_set)
            theirs = np.isin(np.arange(L), O.salient_rows(s, taus[l - l0]))
            assert np.array_equal(mine[clear], theirs[clear]), (l, b)
            caches[(l, b)] = (c, out)
            tm = terms[(l, b)].copy()
            if len(g_set):
                tm[g_set] = tr["salient_terms"]
            terms[(l, b)] = tm
            want[b] = out
        got = to_np(xg).reshape(B, L, dims.d)
        assert_parity(got, want, dims.dtype, f"step output layer {l} (teacher-forced salient sets)",
                      terms=np.stack([terms[(l, b)] for b in range(B)]))
        inputs.append(x_in.copy())
        outs.append(xg.clone())
        x_in = want
    assert 0 < n_salient < B * L * (l1 - l0)

    # the same inputs again: every context repeats exactly, nothing is salient
    for l in range(l0, l1):
        xg2 = to_gpu(inputs[l - l0].reshape(B * L, dims.d), tdt)
        counts = ctx.dyllm_layers_forward(l, l + 1, xg2, B, L, [taus[l - l0]], refresh=False, sim_out=sim)
        ctx.sync_check()
        assert np.all(to_np(sim) == 1.0)
        assert np.all(counts == 0)
        assert torch.equal(xg2, outs[l - l0])
    ctx.close()


def test_dyllm_layers_argument_errors():
    import token_skipping_sparse_step_b200 as esd
    ctx, _ = make_context(synth.SMALL_BF16, synth.SMALL_BF16_RUN, 2, 128)
    x = torch.zeros((2 * 64, synth.SMALL_BF16.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(esd.EsdError):   # no refresh yet
        ctx.dyllm_layers_forward(0, 2, x, 2, 64, [0.9, 0.9], refresh=False)
    ctx.dyllm_layers_forward(0, 2, x, 2, 64, refresh=True)
    with pytest.raises(esd.EsdError):   # other shape than the refresh
        ctx.dyllm_layers_forward(0, 2, x, 1, 64, [0.9, 0.9], refresh=False)
    with pytest.raises(esd.EsdError):   # layers outside the model
        ctx.dyllm_layers_forward(0, 9, x, 2, 64, refresh=True)
    ctx.close()


def _copy_caches(caches):
    return {key: {k_: np.array(v_, copy=True) for k_, v_ in c.items()} for key, c in caches.items()}


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_dyllm_approx_layers_refresh_step_and_repeat(model):
    """The token-selection layers with the saliency-aware approximate attention
    ("DyLLM", technical summary section 2.B.2) against the oracle's
    dyllm_layer_approx, layer by layer from the oracle's input of each layer:
    a refresh (every row exact), a step whose input moved on 30 rows of each
    sequence (the moved rows get exact rows, the others the cached
    probabilities' update; salient sets teacher-forced from the GPU's own
    similarities; moved sets follow from the inputs), and the same inputs
    again (nothing moves, nothing is salient, the output repeats)."""
    dims = synth.TINY if model == "tiny" else synth.SMALL_BF16
    run = synth.TINY_RUN if model == "tiny" else synth.SMALL_BF16_RUN
    B, L = 2, 100
    scale = 20.0 if dims.dtype == "f32" else 4.0
    w32 = synth.model_weights_f32(dims)
    for lw in w32["layers"]:
        lw["wq"] = lw["wq"] * scale
        lw["wk"] = lw["wk"] * scale
    ctx, w = make_context(dims, run, 2, 128, w32=w32)
    tdt = torch.bfloat16 if dims.dtype == "bf16" else torch.float32
    l0, l1 = 0, dims.n_layers
    rng = np.random.default_rng(41)
    x0 = O.store(rng.standard_normal((B, L, dims.d)), dims.dtype)
    caches = {(l, b): {} for l in range(l0, l1) for b in range(B)}
    terms = {}

    x_in = x0.copy()
    for l in range(l0, l1):
        xg = to_gpu(x_in.reshape(B * L, dims.d), tdt)
        counts = ctx.dyllm_layers_forward(l, l + 1, xg, B, L, refresh=True, approx=True)
        ctx.sync_check()
        assert np.all(counts == L)
        want = np.empty_like(x_in)
        for b in range(B):
            tr = {}
            want[b] = O.dyllm_layer_approx(x_in[b], w["layers"][l], dims, caches[(l, b)], 0.0, True, trace=tr)[0]
            terms[(l, b)] = tr["salient_terms"]
        assert_parity(to_np(xg).reshape(B, L, dims.d), want, dims.dtype, f"approx refresh layer {l}",
                      terms=np.stack([terms[(l, b)] for b in range(B)]))
        x_in = want

    # a step whose input moved on 30 rows of each sequence
    x1 = x0.copy()
    moved0 = np.sort(rng.choice(L, 30, replace=False))
    x1[:, moved0] = O.store(x0[:, moved0] + rng.standard_normal((B, len(moved0), dims.d)), dims.dtype)
    # per layer, a threshold between the two middle similarities of the oracle's own step
    taus, probe, xp = [], _copy_caches(caches), x1.copy()
    for l in range(l0, l1):
        sims = [O.dyllm_layer_approx(xp[b], w["layers"][l], dims, _copy_caches({0: probe[(l, b)]})[0], -2.0,
                                     False)[3] for b in range(B)]
        srt = np.sort(np.concatenate(sims).astype(np.float64))
        taus.append(float(0.5 * (srt[len(srt) // 2 - 1] + srt[len(srt) // 2])))
        for b in range(B):
            xp[b] = O.dyllm_layer_approx(xp[b], w["layers"][l], dims, probe[(l, b)], taus[-1], False)[0]
    tol = TOL[dims.dtype]
    sim = torch.empty(B * L, dtype=torch.float32, device="cuda")
    x_in = x1.copy()
    inputs, outs = [], []
    n_salient = 0
    for l in range(l0, l1):
        xg = to_gpu(x_in.reshape(B * L, dims.d), tdt)
        counts = ctx.dyllm_layers_forward(l, l + 1, xg, B, L, [taus[l - l0]], refresh=False, sim_out=sim,
                                          approx=True)
        ctx.sync_check()
        g_sim = to_np(sim).reshape(B, L)
        want = np.empty_like(x_in)
        for b in range(B):
            g_set = O.salient_rows(g_sim[b], taus[l - l0])
            assert counts[0, b] == len(g_set)
            n_salient += len(g_set)
            tr = {}
            out, a, _, s, mv = O.dyllm_layer_approx(x_in[b], w["layers"][l], dims, caches[(l, b)], taus[l - l0],
                                                    False, salient=g_set, trace=tr)
            if l == l0:
                assert np.array_equal(mv, moved0)
            assert_parity(g_sim[b], s, dims.dtype, f"approx similarity layer {l}")
            clear = np.abs(s.astype(np.float64) - np.float32(taus[l - l0])) > 2 * tol
            mine = np.isin(np.arange(L), g_set)
            theirs = np.isin(np.arange(L), O.salient_rows(s, taus[l - l0]))
            assert np.array_equal(mine[clear], theirs[clear]), (l, b)
            tm = terms[(l, b)].copy()
            if len(g_set):
                tm[g_set] = tr["salient_terms"]
            terms[(l, b)] = tm
            want[b] = out
        assert_parity(to_np(xg).reshape(B, L, dims.d), want, dims.dtype, f"approx step output layer {l}",
                      terms=np.stack([terms[(l, b)] for b in range(B)]))
        inputs.append(x_in.copy())
        outs.append(xg.clone())
        x_in = want
    assert 0 < n_salient < B * L * (l1 - l0)

    # the same inputs again: nothing moved, every context repeats, nothing salient
    for l in range(l0, l1):
        xg2 = to_gpu(inputs[l - l0].reshape(B * L, dims.d), tdt)
        counts = ctx.dyllm_layers_forward(l, l + 1, xg2, B, L, [taus[l - l0]], refresh=False, sim_out=sim,
                                          approx=True)
        ctx.sync_check()
        assert np.all(to_np(sim) == 1.0)
        assert np.all(counts == 0)
        assert torch.equal(xg2, outs[l - l0])
    ctx.close()
