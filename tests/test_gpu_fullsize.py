"""Parity at full size: the 8B-class layer shapes in the launch configuration
the benchmark times (B = 1, L = 768, k = 192), the head over the full 126464-id
vocabulary, and the microbenchmark's tensors (B = 16, S = 4096, d = 4096).

Weights and microbenchmark tensors are drawn on the device by the seeded
generator's CUDA twin (synth/csrc/synth.cu); the oracle receives copies of
those inputs, and a few rows are re-drawn on the host to check that both
generators agree. Expected values come from the oracle only; where it would be
too slow on every output it computes sampled rows.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import TOL, assert_parity, to_gpu, to_np

pytestmark = pytest.mark.gpu

FULL = dataclasses.replace(synth.M8B, n_layers=5, vocab=8192, mask_id=8191)  # 8B layer shapes
RUN = synth.M8B_RUN  # skip layer 4, keep 25%: one cached (sparse) layer
L, K = 768, 192


def _ctx(dims, max_batch, max_len):
    import synth.gpu as sg
    import token_skipping_sparse_step_b200 as esd
    w = sg.model_weights(dims)
    ed = esd.make_dims(dims.n_layers, dims.d, dims.n_heads, dims.head_dim, dims.ffn, dims.vocab,
                       dims.mask_id, dims.rope_theta, dims.rms_eps, dims.dtype)
    er = esd.make_run(RUN.score_mode, RUN.alpha, RUN.lam, RUN.skip_layer, RUN.keep_ratio, 0,
                      max_batch, max_len)
    return esd.Context(ed, w, er), w


@pytest.fixture(scope="module")
def full():
    ctx, w = _ctx(FULL, 1, L)
    yield ctx, w
    ctx.close()


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)  # bf16 values, exact


def _layer_host(w, layer, dims):
    lw = {k: _host(v) for k, v in w["layers"][layer].items()}
    # the device generator agrees with the host generator on sampled rows
    lay = {(n, l): (shape, off) for n, l, shape, off in synth.weight_layout(dims)}
    for name in ("wq", "wd"):
        shape, off = lay[(name, layer)]
        rows = [0, shape[0] // 2, shape[0] - 1]
        ref = O.store(synth.weight_rows_f32(synth.SEED_WEIGHTS, off, shape, rows).astype(np.float64), "bf16")
        assert np.array_equal(lw[name][rows], ref), name
    return lw


def test_8b_sparse_layer_at_benchmark_shape(full):
    """Layer 4 of the 8B shapes on k = 192 selected rows of L = 768: QKV GEMM with
    RoPE and K/V scatter, partial attention over the whole cache, O, SwiGLU,
    down - every output row and the scattered K rows against the oracle."""
    ctx, w = full
    rng = np.random.default_rng(8)
    ls = RUN.skip_layer
    x = O.store(rng.standard_normal((L, FULL.d)) * 0.5, "bf16")
    kc = O.store(rng.standard_normal((L, FULL.n_heads, FULL.head_dim)), "bf16")
    vc = O.store(rng.standard_normal((L, FULL.n_heads, FULL.head_dim)), "bf16")
    idx = np.sort(rng.choice(L, K, replace=False)).astype(np.int32)
    v = ctx.state(1, L)
    v["k_cache"][0].copy_(to_gpu(kc[None], torch.bfloat16))
    v["v_cache"][0].copy_(to_gpu(vc[None], torch.bfloat16))
    xs = to_gpu(x[idx], torch.bfloat16)
    ctx.sparse_layers_forward(ls, ls + 1, to_gpu(idx, torch.int32), 1, L, K, xs)
    ctx.sync_check()
    lw = _layer_host(w, ls, FULL)
    kb, vb = kc.copy(), vc.copy()
    tr = {}
    want = O.sparse_layer(x[idx], idx, kb, vb, lw, FULL, trace=tr)
    assert_parity(to_np(xs), want, "bf16", "8B sparse layer output", terms=tr["residual_terms"])
    gk = to_np(v["k_cache"][0])[0]
    assert_parity(gk[idx], kb[idx], "bf16", "scattered K")
    rest = np.setdiff1d(np.arange(L), idx)
    assert np.array_equal(gk[rest], kc[rest])


def test_8b_dense_layer_at_benchmark_shape(full):
    """Layer 0 of the 8B shapes on all L = 768 rows (the dense early layers and
    the refresh step: two-SM 256x256 tiles)."""
    ctx, w = full
    rng = np.random.default_rng(9)
    x = O.store(rng.standard_normal((L, FULL.d)) * 0.5, "bf16")
    xg = to_gpu(x, torch.bfloat16)
    ctx.sparse_layers_forward(0, 1, None, 1, L, L, xg)
    ctx.sync_check()
    tr = {}
    want, _, _ = O.dense_layer(x, _layer_host(w, 0, FULL), FULL, trace=tr)
    assert_parity(to_np(xg), want, "bf16", "8B dense layer output", terms=tr["residual_terms"])


def test_8b_dyllm_layer_graph_at_benchmark_shape(full):
    """DyLLM token-selection layer 0 of the 8B shapes over L = 768 rows, as the
    non-refresh call runs it (a CUDA graph whose switch node picks the GEMMs'
    row capacity from the salient count on the device): a refresh with x0,
    a probe step with x1 (every 4th row redrawn) and nothing salient to read
    the similarities, the same refresh again, then x1 with a threshold that
    makes the 150 least similar rows salient (capacity 160 on the
    swapped-operand GEMMs). The salient rows' outputs against the oracle's
    layer with that salient set; every other row keeps the refresh's output
    bit for bit."""
    ctx, w = full
    rng = np.random.default_rng(11)
    x0 = O.store(rng.standard_normal((L, FULL.d)) * 0.5, "bf16")
    x1 = x0.copy()
    x1[::4] = O.store(rng.standard_normal((L // 4, FULL.d)) * 0.5, "bf16")
    sim = torch.empty(L, dtype=torch.float32, device="cuda")
    xr = to_gpu(x0, torch.bfloat16)
    ctx.dyllm_layers_forward(0, 1, xr, 1, L, refresh=True)
    counts = ctx.dyllm_layers_forward(0, 1, to_gpu(x1, torch.bfloat16), 1, L, [-2.0], refresh=False,
                                      sim_out=sim)
    assert counts.sum() == 0
    probe = to_np(sim)
    xr2 = to_gpu(x0, torch.bfloat16)
    ctx.dyllm_layers_forward(0, 1, xr2, 1, L, refresh=True)
    assert torch.equal(xr2, xr)
    m = 150
    srt = np.sort(probe)
    assert srt[m - 1] < srt[m]
    tau = float(0.5 * (srt[m - 1] + srt[m]))
    xg = to_gpu(x1, torch.bfloat16)
    counts = ctx.dyllm_layers_forward(0, 1, xg, 1, L, [tau], refresh=False, sim_out=sim)
    ctx.sync_check()
    assert counts[0, 0] == m
    assert np.array_equal(to_np(sim), probe)
    g_set = O.salient_rows(to_np(sim), tau)
    assert len(g_set) == m
    lw = _layer_host(w, 0, FULL)
    tr = {}
    zeros = np.zeros_like(x1)
    want, _, _, _ = O.dyllm_layer(x1, lw, FULL, zeros, zeros, tau, False, salient=g_set, trace=tr)
    got = to_np(xg)
    assert_parity(got[g_set], want[g_set], "bf16", "8B DyLLM salient rows", terms=tr["salient_terms"])
    others = np.setdiff1d(np.arange(L), g_set)
    assert np.array_equal(got[others], to_np(xr)[others])


def test_8b_head_full_vocabulary_sampled_rows():
    """The fused head over all 126464 ids for the 192 selected rows; the oracle
    computes 6 sampled rows over the whole vocabulary."""
    dims = dataclasses.replace(synth.M8B, n_layers=5)
    ctx, w = _ctx(dims, 1, L)
    rng = np.random.default_rng(10)
    x = O.store(rng.standard_normal((K, dims.d)), "bf16")
    conf = torch.empty(K, dtype=torch.float32, device="cuda")
    tok = torch.empty(K, dtype=torch.int32, device="cuda")
    ctx.confidence_argmax(to_gpu(x, torch.bfloat16), None, 1, K, K, conf, tok)
    ctx.sync_check()
    rows = [0, 1, 63, 100, 150, 191]
    xr = x[rows]
    h = xr * O.rms_inv(xr, dims.rms_eps)[:, None]
    lg = np.empty((len(rows), dims.vocab))
    for c0 in range(0, dims.vocab, 16384):
        c1 = min(dims.vocab, c0 + 16384)
        lg[:, c0:c1] = h @ _host(w["w_out"][c0:c1]).T
    lg[:, dims.mask_id] = -np.inf
    m = lg.max(axis=1)
    want_conf = 1.0 / np.exp(lg - m[:, None]).sum(axis=1)
    lg32 = lg.astype(np.float32)
    want_tok = np.argmax(lg32, axis=1)
    srt = np.sort(lg32, axis=1)
    margin = srt[:, -1].astype(np.float64) - srt[:, -2]
    scale = np.abs(np.where(np.isfinite(lg), lg, 0)).max(axis=1)
    assert_parity(to_np(conf)[rows], want_conf, "bf16", "confidence")
    got_tok = to_np(tok)[rows]
    near = margin < 2 * TOL["bf16"] * scale
    assert np.all((got_tok == want_tok) | near), (got_tok, want_tok, margin)
    assert np.all(to_np(tok) != dims.mask_id)
    ctx.close()


@pytest.mark.parametrize("k", [64, 256, 1024])
def test_micro_scores_selection_gather_full_size(k):
    """Microbenchmark shapes (B 16, S 4096, d 4096, bf16): scores of sampled rows
    against the oracle; the selection is a valid top-k of the kernel's own
    scores under (score desc, index asc); the gather is exact. (Selection fed
    the oracle's scores at this size is bit-exact in test_gpu_parity.py.)"""
    import synth.gpu as sg
    import token_skipping_sparse_step_b200 as esd
    B, S, d = synth.MICRO["batch"], synth.MICRO["seq"], synth.MICRO["d"]
    ed = esd.make_dims(2, d, 32, 128, 256, 1024, 1023, 5e5, 1e-6, "bf16")
    dims = synth.ModelDims(2, d, 32, 128, 256, 1024, 1023, 5e5, 1e-6, "bf16")
    w = sg.model_weights(dims)
    ctx = esd.Context(ed, w, esd.make_run("es", 0.5, 0.5, 1, 0.25, 0, B, S))
    x, h, conf = sg.micro_inputs(B, S, d)
    sc = torch.empty(B * S, dtype=torch.float32, device="cuda")
    idx = torch.empty(B * k, dtype=torch.int32, device="cuda")
    ctx.importance_select(x, h, conf, B, S, k, idx, scores_out=sc)
    xs = torch.empty((B * k, d), dtype=torch.bfloat16, device="cuda")
    ctx.gather_rows(x, idx, B, S, k, xs, None)
    ctx.sync_check()
    rows = np.array([0, 5, 4095, 4096, 30000, 65535])
    xr, hr, cr = synth.micro_rows(B, S, d, rows)
    want = O.importance_es(O.store(xr, "bf16"), O.store(hr, "bf16"), cr.astype(np.float64), 0.5)
    assert_parity(to_np(sc)[rows], want, "f32", "scores")
    gi = to_np(idx).reshape(B, k)
    gs = to_np(sc).reshape(B, S)
    for b in range(B):
        assert np.all(np.diff(gi[b]) > 0)
        sel = np.zeros(S, bool)
        sel[gi[b]] = True
        # every selected row outranks every skipped row under (score desc, index asc)
        lo = gs[b][sel].min()
        hi = gs[b][~sel].max() if (~sel).any() else -np.inf
        assert lo >= hi
        if lo == hi:
            assert np.flatnonzero(sel & (gs[b] == lo)).max() < np.flatnonzero(~sel & (gs[b] == hi)).min()
    assert torch.equal(xs, x.view(B, S, d)[torch.arange(B, device="cuda")[:, None], idx.view(B, k).long()].reshape(B * k, d))
    ctx.close()


def test_micro_partial_attention_full_size():
    """k = 256 selected queries per sequence over S = 4096 keys, 32 heads x 128,
    B = 16: sampled query rows against the oracle's attention over the whole K/V
    of their sequence."""
    import synth.gpu as sg
    import token_skipping_sparse_step_b200 as esd
    B, S, d, k = 16, 4096, 4096, 256
    H, hd = 32, 128
    dims = synth.ModelDims(2, d, H, hd, 256, 1024, 1023, 5e5, 1e-6, "bf16")
    ctx = esd.Context(esd.make_dims(2, d, H, hd, 256, 1024, 1023, 5e5, 1e-6, "bf16"),
                      sg.model_weights(dims), esd.make_run("es", 0.5, 0.5, 1, 0.25, 0, B, S))
    q = torch.empty((B * k, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.empty((B * S, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty((B * S, d), dtype=torch.bfloat16, device="cuda")
    sg.fill_normal(q, 21, 0)
    sg.fill_normal(kc, 22, 0)
    sg.fill_normal(vc, 23, 0)
    out = torch.empty_like(q)
    ctx.partial_attention(q, kc, vc, B, S, k, out)
    ctx.sync_check()
    for r in (0, 255, 256 * 7 + 100, B * k - 1):
        b = r // k
        qr = _host(q[r:r + 1]).reshape(1, H, hd)
        kb = _host(kc[b * S:(b + 1) * S]).reshape(S, H, hd)
        vb = _host(vc[b * S:(b + 1) * S]).reshape(S, H, hd)
        want = O.attention(qr, kb, vb).reshape(d)
        assert_parity(to_np(out[r]), want, "bf16", f"attention row {r}")
    ctx.close()


# (B, R, L, growing, H): heads x 128. Pair-tiles of 256 queries; the keys,
# in chunks of 128, are split over 2 pairs of a cluster when the pair-tiles
# leave SMs idle (e.g. (1, 192, 768), (1, 130, 1024)), over 3 or 4 with few
# heads ((1, 250, 700, 4): 3 splits of 2 chunks; (1, 100, 1000, 4): 4 splits;
# (2, 300, 333, 4): two pair-tiles, 3 splits of one chunk), over one pair
# otherwise; one-key tails, a second pair-tile. Up to 64 queries per sequence
# ((3, 1, 5), (8, 37, 1000), (40, 1, 5)) run the 64-query mma.sync kernel,
# with the keys split across CTAs where its query tiles are few.
# "growing" scales key l by 1 + l / 40 so that the row maximum keeps rising
# across key chunks (running-max rescales of the accumulated O).
ATTN_CASES = [(1, 192, 768, False, 32), (3, 1, 5, False, 32), (5, 200, 333, False, 32),
              (8, 37, 1000, False, 32), (6, 129, 129, False, 32), (40, 1, 5, False, 32),
              (6, 128, 640, True, 32), (1, 130, 1024, True, 32), (1, 250, 700, True, 4),
              (1, 100, 1000, False, 4), (2, 300, 333, True, 4), (1, 768, 768, False, 32)]


@pytest.mark.parametrize("B,R,Lk,growing,H", ATTN_CASES)
def test_partial_attention_ragged_shapes(B, R, Lk, growing, H):
    """Every output row against the oracle's attention over its sequence's
    whole K/V, on ragged query and key counts (partial tiles, one-key tails,
    one query per sequence) and on scores that rise along the keys."""
    import token_skipping_sparse_step_b200 as esd
    import synth.gpu as sg
    hd = 128
    d = H * hd
    dims = synth.ModelDims(2, d, H, hd, 256, 1024, 1023, 5e5, 1e-6, "bf16")
    ctx = esd.Context(esd.make_dims(2, d, H, hd, 256, 1024, 1023, 5e5, 1e-6, "bf16"),
                      sg.model_weights(dims), esd.make_run("es", 0.5, 0.5, 1, 0.25, 0, 40, 1024))
    rng = np.random.default_rng(B * 100003 + R * 1009 + Lk)
    q = O.store(rng.standard_normal((B, R, H, hd)), "bf16")
    kc = rng.standard_normal((B, Lk, H, hd))
    if growing:
        kc *= (1.0 + np.arange(Lk) / 40.0)[None, :, None, None]
    kc = O.store(kc, "bf16")
    vc = O.store(rng.standard_normal((B, Lk, H, hd)), "bf16")
    out = torch.empty((B * R, d), dtype=torch.bfloat16, device="cuda")
    ctx.partial_attention(to_gpu(q.reshape(B * R, d), torch.bfloat16), to_gpu(kc.reshape(B * Lk, d), torch.bfloat16),
                          to_gpu(vc.reshape(B * Lk, d), torch.bfloat16), B, Lk, R, out)
    ctx.sync_check()
    got = to_np(out).reshape(B, R, H, hd)
    for b in range(B):
        want = O.attention(q[b], kc[b], vc[b])
        assert_parity(got[b], want, "bf16", f"attention sequence {b}")
    ctx.close()
