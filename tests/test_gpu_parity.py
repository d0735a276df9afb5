"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Every input is seeded and synthetic (``synth``); every expected value comes from
``oracle``. Tolerances: float32 models 1e-4, bf16 models 2e-2, asserted both normwise
(max|g - o| / max|o|) and element-wise (|g - o| <= tol * max(1, |o|)) by
tests/helpers.py. Integer and
index results are compared exactly, except decisions whose oracle margin is a
near-tie (then both answers are correct up to rounding).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import TOL, assert_parity, make_context, near_tie_ok, parity_error, parity_ok, to_gpu, to_np

pytestmark = pytest.mark.gpu

_CTX = {}


def ctx_for(name):
    if name not in _CTX:
        if name == "tiny":
            _CTX[name] = make_context(synth.TINY, synth.TINY_RUN, 3, 256)
        elif name == "small":
            _CTX[name] = make_context(synth.SMALL_BF16, synth.SMALL_BF16_RUN, 3, 256)
        else:
            raise KeyError(name)
    return _CTX[name]


def dims_run(name):
    return {"tiny": (synth.TINY, synth.TINY_RUN), "small": (synth.SMALL_BF16, synth.SMALL_BF16_RUN)}[name]


def tdt(dims):
    return torch.bfloat16 if dims.dtype == "bf16" else torch.float32


# ----------------------------------------------------------------------------- selection
@pytest.mark.parametrize("model", ["tiny", "small"])
@pytest.mark.parametrize("mode", ["es", "cos"])
def test_importance_scores_and_selection(model, mode):
    ctx, _ = ctx_for(model)
    dims, run = dims_run(model)
    run = dataclasses.replace(run, score_mode=mode)
    B, L = 3, 200
    k = O.keep_count(0.25, L)
    x, hc, conf = synth.micro_inputs(B, L, dims.d, seed=11)
    xo, ho = O.store(x, dims.dtype), O.store(hc, dims.dtype)
    conf = conf.astype(np.float32)
    want = np.stack([O.importance(xo[b], ho[b], conf[b].astype(np.float64), run) for b in range(B)])
    # the context's score mode is fixed at create: build one for this mode
    from helpers import make_context as mk
    c2, _ = mk(dims, run, 3, 256) if mode != dims_run(model)[1].score_mode else (ctx, None)
    xg, hg = to_gpu(xo, tdt(dims)), to_gpu(ho, tdt(dims))
    cg = to_gpu(conf, torch.float32)
    sc = torch.empty(B * L, dtype=torch.float32, device="cuda")
    idx = torch.empty(B * k, dtype=torch.int32, device="cuda")
    c2.importance_select(xg, hg, cg, B, L, k, idx, scores_out=sc)
    c2.sync_check()
    got = to_np(sc).reshape(B, L)
    assert_parity(got, want, "f32", "importance score")
    gi = to_np(idx).reshape(B, k)
    for b in range(B):
        # the GPU's indices are exactly the top-k of its own float32 scores
        assert np.array_equal(gi[b], O.topk_select(got[b], k)), b
        oi = O.topk_select(want[b], k)
        if np.array_equal(gi[b], oi):
            continue
        # otherwise the sets may differ only among rows whose oracle score
        # lies within the score error band around the oracle's k-th score
        kth = float(np.sort(want[b])[::-1][k - 1])
        band = 2 * TOL["f32"] * max(1.0, abs(kth))
        diff = np.setxor1d(gi[b], oi)
        assert np.all(np.abs(want[b][diff] - kth) <= band), (b, diff, want[b][diff], kth)


def _topk_cases(rng):
    yield "random", rng.standard_normal((3, 300)).astype(np.float32), 77
    yield "ties", rng.choice([0.0, -0.0, 0.5, 1.0, 0.5, -2.0], size=(2, 513)).astype(np.float32), 100
    yield "all_equal", np.full((2, 64), 0.25, np.float32), 10
    yield "k1", rng.standard_normal((1, 1000)).astype(np.float32), 1
    yield "kL", rng.standard_normal((2, 130)).astype(np.float32), 130
    yield "L1", np.array([[3.0]], np.float32), 1
    s = rng.standard_normal((2, 257)).astype(np.float32)
    s[0, ::7] = np.nan
    s[1, ::5] = -np.inf
    yield "nan_inf", s, 200
    yield "max_len", rng.standard_normal((16, 4096)).astype(np.float32), 1024
    yield "neg_zero", np.where(rng.uniform(size=(1, 300)) < 0.5, 0.0, -0.0).astype(np.float32), 150


@pytest.mark.parametrize("case", [c[0] for c in _topk_cases(np.random.default_rng(0))])
def test_topk_bit_exact_from_oracle_scores(case):
    rng = np.random.default_rng(5)
    name, s, k = next(c for c in _topk_cases(rng) if c[0] == case)
    B, L = s.shape
    ctx, _ = make_context(synth.TINY, synth.TINY_RUN, B, max(L, 128)) if L > 256 or B > 3 else ctx_for("tiny")
    idx = torch.full((B * k,), -1, dtype=torch.int32, device="cuda")
    ctx.topk_select(to_gpu(s, torch.float32), B, L, k, idx)
    ctx.sync_check()
    got = to_np(idx).reshape(B, k)
    for b in range(B):
        assert np.array_equal(got[b], O.topk_select(s[b], k)), (name, b)


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_gather_rows_and_h_cache_scatter_exact(model):
    ctx, _ = ctx_for(model)
    dims, _ = dims_run(model)
    B, L, k = 3, 150, 37
    rng = np.random.default_rng(3)
    x = O.store(rng.standard_normal((B * L, dims.d)), dims.dtype)
    h0 = O.store(rng.standard_normal((B * L, dims.d)), dims.dtype)
    idx = np.stack([np.sort(rng.choice(L, k, replace=False)) for _ in range(B)]).astype(np.int32)
    xg, hg = to_gpu(x, tdt(dims)), to_gpu(h0, tdt(dims))
    xs = torch.empty((B * k, dims.d), dtype=tdt(dims), device="cuda")
    ctx.gather_rows(xg, to_gpu(idx, torch.int32), B, L, k, xs, hg)
    ctx.sync_check()
    rows = (np.arange(B)[:, None] * L + idx).reshape(-1)
    assert np.array_equal(to_np(xs), x[rows])
    want_h = h0.copy()
    want_h[rows] = x[rows]
    assert np.array_equal(to_np(hg), want_h)


def test_remask_exact():
    ctx, _ = ctx_for("tiny")
    rng = np.random.default_rng(9)
    B, L = 3, 200
    for trial in range(5):
        masked = (rng.uniform(size=(B, L)) < 0.5).astype(np.uint8)
        conf = rng.choice([0.1, 0.3, 0.3, 0.9], size=(B, L)).astype(np.float32)
        tok_c = rng.integers(0, 1000, size=(B, L)).astype(np.int32)
        tok = rng.integers(0, 1000, size=(B, L)).astype(np.int32)
        b0, b1, n = 40, 104, int(rng.integers(1, 6))
        tg, mg = to_gpu(tok, torch.int32), to_gpu(masked, torch.uint8)
        ctx.remask(tg, mg, to_gpu(conf, torch.float32), to_gpu(tok_c, torch.int32), B, L, b0, b1, n)
        ctx.sync_check()
        for b in range(B):
            O.remask(tok[b], masked[b], conf[b], tok_c[b], b0, b1, n)
        assert np.array_equal(to_np(tg), tok) and np.array_equal(to_np(mg), masked)


# ----------------------------------------------------------------------------- the model
def _state_for(dims, run, B, prompt_len, gen, seed=1):
    prompt = synth.prompt_ids(dims, B, prompt_len, seed=seed)
    L = prompt_len + gen
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :prompt_len] = prompt
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, prompt_len:] = 1
    return O.new_state(dims, run, tok, masked)


def _upload_state(ctx, st, dims):
    B, L = st.tok.shape
    v = ctx.state(B, L)
    dt = tdt(dims)
    v["h_cache"].copy_(to_gpu(st.hc, dt))
    for i in range(len(st.kc)):
        v["k_cache"][i].copy_(to_gpu(st.kc[i], dt))
        v["v_cache"][i].copy_(to_gpu(st.vc[i], dt))
    v["conf_cache"].copy_(to_gpu(st.conf_c, torch.float32))
    v["tok_cache"].copy_(to_gpu(st.tok_c, torch.int32))
    return v


def _compare_state(v, st, dims, rows=None):
    pairs = {"h": (to_np(v["h_cache"]), st.hc), "conf": (to_np(v["conf_cache"]), st.conf_c)}
    for i in range(len(st.kc)):
        pairs[f"k{i}"] = (to_np(v["k_cache"][i]), st.kc[i])
        pairs[f"v{i}"] = (to_np(v["v_cache"][i]), st.vc[i])
    errs = {k_: parity_ok(g, o, dims.dtype) for k_, (g, o) in pairs.items()}
    for k_, (ok, n, e) in errs.items():
        assert ok, (k_, n, e, errs)
    return errs


def _check_predictions(g_tok, o_tok, info, idx, dims):
    """Predictions of the recomputed rows match, except near-ties: rows whose
    oracle top-2 logit margin is below 2 * tol * (the row's largest |logit|),
    the accuracy the hidden states carry into the logits."""
    tol = TOL[dims.dtype]
    for b in range(o_tok.shape[0]):
        rows = np.arange(o_tok.shape[1]) if idx is None else idx[b]
        near = info["row_margin"][b] < 2 * tol * info["row_scale"][b]
        bad = (g_tok[b][rows] != o_tok[b][rows]) & ~near
        assert not bad.any(), f"{int(bad.sum())} predictions differ outside near-ties"


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_dense_step_matches_oracle(model):
    ctx, w = ctx_for(model)
    dims, run = dims_run(model)
    B, P, G = 2, 96, 64
    st = _state_for(dims, run, B, P, G)
    tg, mg = to_gpu(st.tok, torch.int32), to_gpu(st.masked, torch.uint8)
    info = O.dense_step(w, dims, run, st, P, P + 32, 2)
    ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=True)
    ctx.sync_check()
    v = ctx.state(B, P + G)
    _compare_state(v, st, dims)
    _check_predictions(to_np(v["tok_cache"]), st.tok_c, info, None, dims)


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_sparse_step_teacher_forced(model):
    """From the oracle's state after a dense step, the sparse-step pieces
    (embed + dense early layers, score, selection fed the oracle's indices,
    gather + H scatter, sparse layers with K/V scatter and partial attention,
    head with the confidence scatter) match the oracle's sparse step."""
    ctx, w = ctx_for(model)
    dims, run = dims_run(model)
    B, P, G = 2, 96, 64
    L = P + G
    st = _state_for(dims, run, B, P, G)
    O.dense_step(w, dims, run, st, P, P + 32, 2)
    _upload_state(ctx, st, dims)
    before = st.copy()
    info = O.sparse_step(w, dims, run, st, P, P + 32, 2)
    k = O.keep_count(run.keep_ratio, L)
    dt = tdt(dims)
    tg = to_gpu(before.tok, torch.int32)
    x = torch.empty((B * L, dims.d), dtype=dt, device="cuda")
    ctx.embed(tg, x)
    ctx.sparse_layers_forward(0, run.skip_layer, None, B, L, L, x)
    v = ctx.state(B, L)
    assert_parity(to_np(x).reshape(B, L, dims.d), np.stack(info["x_ls"]), dims.dtype, "skip-layer input")
    sc = torch.empty(B * L, dtype=torch.float32, device="cuda")
    idx = torch.empty(B * k, dtype=torch.int32, device="cuda")
    ctx.importance_select(x, v["h_cache"], v["conf_cache"], B, L, k, idx, scores_out=sc)
    assert_parity(to_np(sc).reshape(B, L), np.stack(info["scores"]), "f32" if dims.dtype == "f32" else "bf16", "scores")
    oidx = np.stack(info["idx"]).astype(np.int32)
    n_sel_diff = int((to_np(idx).reshape(B, k) != oidx).sum())
    ig = to_gpu(oidx, torch.int32)          # teacher forcing: the oracle's selection
    # teacher forcing of the skip-layer input too (the oracle's x at l_s)
    x_or = to_gpu(np.stack(info["x_ls"]).reshape(B * L, dims.d), dt)
    xs = torch.empty((B * k, dims.d), dtype=dt, device="cuda")
    ctx.gather_rows(x_or, ig, B, L, k, xs, v["h_cache"])
    ctx.sparse_layers_forward(run.skip_layer, dims.n_layers, ig, B, L, k, xs)
    assert_parity(to_np(xs).reshape(B, k, dims.d), np.stack(info["xs_out"]), dims.dtype, "sparse rows out")
    ctx.confidence_argmax(xs, ig, B, L, k, v["conf_cache"], v["tok_cache"])
    ctx.sync_check()
    _compare_state(v, st, dims)
    g_tok = to_np(v["tok_cache"])
    _check_predictions(g_tok, st.tok_c, info, oidx, dims)
    # skipped rows of every cache are byte-identical to the state before the step
    for b in range(B):
        skip = np.setdiff1d(np.arange(L), oidx[b])
        assert np.array_equal(to_np(v["conf_cache"])[b][skip], before.conf_c[b][skip].astype(np.float32))
        for i in range(len(st.kc)):
            assert np.array_equal(to_np(v["k_cache"][i])[b][skip], before.kc[i][b][skip])
    print(f"selection differences vs oracle (GPU scores): {n_sel_diff}")


def test_tiny_generation_tokens_identical():
    ctx, w = ctx_for("tiny")
    dims, run = synth.TINY, synth.TINY_RUN
    seq = synth.TINY_SEQ
    prompt = synth.prompt_ids(dims, seq["batch"], seq["prompt"])
    want, log = O.generate(w, dims, run, prompt, seq["gen"], seq["block"], seq["n_unmask"])
    got = ctx.generate(torch.from_numpy(prompt), seq["gen"], seq["block"], seq["n_unmask"])
    got = got.cpu().numpy()
    tk = min(m for l in log if not l["dense"] for m in l["topk_margin"])
    rm = min(m for l in log for m in l["remask_margin"])
    print(f"smallest top-k margin {tk:.3e}, smallest remask margin {rm:.3e}")
    assert np.array_equal(got, want), f"{int((got != want).sum())} tokens differ (margins {tk:.2e}/{rm:.2e})"


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_keep_all_sparse_step_equals_dense_step_on_gpu(model):
    ctx, w = ctx_for(model)
    dims, run = dims_run(model)
    B, P, G = 2, 64, 64
    L = P + G
    st = _state_for(dims, run, B, P, G)
    tg, mg = to_gpu(st.tok, torch.int32), to_gpu(st.masked, torch.uint8)
    ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=True)
    v = ctx.state(B, L)
    snap = {k_: (x.clone() if torch.is_tensor(x) else [y.clone() for y in x]) for k_, x in v.items()}
    t1, m1 = tg.clone(), mg.clone()
    ctx.denoise_step(t1, m1, P, P + 32, 2, force_dense=True)
    dense = {k_: (x.clone() if torch.is_tensor(x) else [y.clone() for y in x]) for k_, x in v.items()}
    for k_, x in snap.items():  # restore, then a sparse step with k = L through the pieces
        if torch.is_tensor(x):
            v[k_].copy_(x)
        else:
            for a, b in zip(v[k_], x):
                a.copy_(b)
    dt = tdt(dims)
    x = torch.empty((B * L, dims.d), dtype=dt, device="cuda")
    ctx.embed(tg, x)
    ctx.sparse_layers_forward(0, run.skip_layer, None, B, L, L, x)
    idx = torch.empty(B * L, dtype=torch.int32, device="cuda")
    ctx.importance_select(x, v["h_cache"], v["conf_cache"], B, L, L, idx)
    assert np.array_equal(to_np(idx).reshape(B, L), np.tile(np.arange(L), (B, 1)))
    xs = torch.empty_like(x)
    ctx.gather_rows(x, idx, B, L, L, xs, v["h_cache"])
    ctx.sparse_layers_forward(run.skip_layer, dims.n_layers, idx, B, L, L, xs)
    ctx.confidence_argmax(xs, idx, B, L, L, v["conf_cache"], v["tok_cache"])
    ctx.sync_check()
    for k_, x in dense.items():
        if torch.is_tensor(x):
            assert torch.equal(v[k_], x), k_
        else:
            for a, b in zip(v[k_], x):
                assert torch.equal(a, b), k_


@pytest.mark.parametrize("model", ["tiny", "small"])
def test_logits_and_head_match_oracle(model):
    ctx, w = ctx_for(model)
    dims, _ = dims_run(model)
    rng = np.random.default_rng(21)
    rows = 150
    x = O.store(rng.standard_normal((rows, dims.d)) * 0.3, dims.dtype)
    xg = to_gpu(x, tdt(dims))
    lg = torch.empty((rows, dims.vocab), dtype=torch.float32, device="cuda")
    ctx.logits(xg, rows, lg)
    conf = torch.empty(rows, dtype=torch.float32, device="cuda")
    tok = torch.empty(rows, dtype=torch.int32, device="cuda")
    ctx.confidence_argmax(xg, None, 1, rows, rows, conf, tok)
    ctx.sync_check()
    want = O.logits(x, w["w_out"], dims)
    g = to_np(lg)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(g), fin)
    assert_parity(g[fin], want[fin], dims.dtype, "logits")
    oc, ot, om = O.head(x, w["w_out"], dims)
    assert_parity(to_np(conf), oc, dims.dtype, "confidence")
    ok, nbad = near_tie_ok(to_np(tok), ot, om, 1e-3 if dims.dtype == "bf16" else 1e-5)
    assert ok, f"{nbad} argmax mismatches outside near-ties"


@pytest.mark.parametrize("B,k", [(1, 1), (1, 37), (2, 64), (1, 129), (2, 100), (1, 256), (3, 86), (2, 160)])
def test_one_sparse_layer_across_row_counts(B, k):
    """One layer on B*k selected rows (1 .. 320: every tensor-core tile shape,
    split-K and not) against the oracle's sparse layer from the same cache."""
    ctx, w = ctx_for("small")
    dims, run = dims_run("small")
    L = 160
    k = min(k, L)
    rng = np.random.default_rng(100 + B * k)
    ls = run.skip_layer
    x = O.store(rng.standard_normal((B, L, dims.d)) * 0.5, dims.dtype)
    idx = np.stack([np.sort(rng.choice(L, k, replace=False)) for _ in range(B)]).astype(np.int32)
    kc = O.store(rng.standard_normal((B, L, dims.n_heads, dims.head_dim)), dims.dtype)
    vc = O.store(rng.standard_normal((B, L, dims.n_heads, dims.head_dim)), dims.dtype)
    v = ctx.state(B, L)
    v["k_cache"][0].copy_(to_gpu(kc, torch.bfloat16))
    v["v_cache"][0].copy_(to_gpu(vc, torch.bfloat16))
    xs = to_gpu(np.stack([x[b][idx[b]] for b in range(B)]).reshape(B * k, dims.d), torch.bfloat16)
    ctx.sparse_layers_forward(ls, ls + 1, to_gpu(idx, torch.int32), B, L, k, xs)
    ctx.sync_check()
    want = []
    for b in range(B):
        kb, vb = kc[b].copy(), vc[b].copy()
        want.append(O.sparse_layer(x[b][idx[b]], idx[b], kb, vb, w["layers"][ls], dims))
        # the K/V scatter: selected rows fresh, the others untouched
        gk = to_np(v["k_cache"][0])[b]
        assert_parity(gk[idx[b]], kb[idx[b]], "bf16", "scattered K")
        rest = np.setdiff1d(np.arange(L), idx[b])
        assert np.array_equal(gk[rest], kc[b][rest])
    assert_parity(to_np(xs).reshape(B, k, dims.d), np.stack(want), "bf16", "layer output")


# ----------------------------------------------------------------------------- dense baseline
def test_tiny_vanilla_generation_tokens_identical():
    """The dense every-token baseline (every step a full refresh,
    ``esd_generate(..., vanilla=1)``) on the float32 tiny model gives the
    oracle's vanilla generation token for token."""
    ctx, w = ctx_for("tiny")
    dims, run = synth.TINY, synth.TINY_RUN
    seq = synth.TINY_SEQ
    prompt = synth.prompt_ids(dims, seq["batch"], seq["prompt"])
    want, log = O.generate(w, dims, run, prompt, seq["gen"], seq["block"], seq["n_unmask"], vanilla=True)
    assert all(l["dense"] for l in log)
    got = ctx.generate(torch.from_numpy(prompt), seq["gen"], seq["block"], seq["n_unmask"], vanilla=True)
    got = got.cpu().numpy()
    rm = min(m for l in log for m in l["remask_margin"])
    assert np.array_equal(got, want), f"{int((got != want).sum())} tokens differ (remask margin {rm:.2e})"


def test_small_bf16_vanilla_generation_is_dense_steps_matching_oracle():
    """bf16 dense baseline: the vanilla generation equals, bit for bit, the same
    number of dense steps driven one by one; every one of those steps matches
    the oracle's dense step on the same tokens (caches within tolerance,
    predictions outside near-ties, the unmasked positions where the oracle's
    remask margin is clear)."""
    ctx, w = ctx_for("small")
    dims, run = synth.SMALL_BF16, synth.SMALL_BF16_RUN
    B, P, G, blk, nu = 2, 96, 64, 32, 8
    L = P + G
    prompt = synth.prompt_ids(dims, B, P, seed=3)
    got = ctx.generate(torch.from_numpy(prompt).cuda(), G, blk, nu, vanilla=True).cpu().numpy()
    st = _state_for(dims, run, B, P, G, seed=3)
    tg, mg = to_gpu(st.tok, torch.int32), to_gpu(st.masked, torch.uint8)
    for b0 in range(P, L, blk):
        for _ in range(blk // nu):
            tok_before, mask_before = to_np(tg), to_np(mg)
            ctx.denoise_step(tg, mg, b0, b0 + blk, nu, force_dense=True)
            ctx.sync_check()
            o = O.new_state(dims, run, tok_before.copy(), mask_before.copy())
            info = O.dense_step(w, dims, run, o, b0, b0 + blk, nu)
            v = ctx.state(B, L)
            _compare_state(v, o, dims)
            _check_predictions(to_np(v["tok_cache"]), o.tok_c, info, None, dims)
            g_tok, g_msk = to_np(tg), to_np(mg)
            for b in range(B):
                g_pick = np.sort(np.nonzero(mask_before[b].astype(bool) & ~g_msk[b].astype(bool))[0])
                scale = float(np.max(o.conf_c[b][b0:b0 + blk]))
                if info["remask_margin"][b] > 2 * TOL["bf16"] * scale:
                    assert np.array_equal(g_pick, np.sort(info["unmasked"][b])), (b0, b)
                # the GPU wrote its own cached predictions at its own picks
                assert np.array_equal(g_tok[b][g_pick], to_np(v["tok_cache"])[b][g_pick])
    assert np.array_equal(got, to_np(tg)[:, P:]), "vanilla generation differs from the dense steps"
