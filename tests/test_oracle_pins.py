"""Pins of the CPU oracle against things other than itself.

Closed forms, hand-evaluated cases of the importance equation ("ES-dLLM:
Efficient Inference for Diffusion Large Language Models by Early-Skipping",
technical summary section 2.A), library routines (torch CPU float64: rms_norm,
scaled_dot_product_attention, softmax, argmax, sort), invariants and brute
force on tiny inputs. Each test is built so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
RoPE pairing, a wrong tie-break) fails it.
"""
import dataclasses
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
import synth

HERE = os.path.dirname(os.path.abspath(__file__))
RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- bf16 rounding
def test_round_bf16_matches_torch_float32_conversion():
    # float32 inputs across the whole range, subnormals included
    bits = RNG.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.astype(np.float64))
    fin = np.isfinite(want)
    assert np.array_equal(got[fin], want[fin])
    assert np.array_equal(np.isinf(got), np.isinf(want))


def test_round_bf16_hand_values():
    u = 2.0 ** -7  # bf16 ulp at 1
    assert O.round_bf16(1.0 + u / 2)[()] == 1.0               # tie -> even (1.0)
    assert O.round_bf16(1.0 + 3 * u / 2)[()] == 1.0 + 2 * u   # tie -> even (1 + 2u)
    assert O.round_bf16(1.0 + u / 2 + 1e-12)[()] == 1.0 + u   # above the tie
    assert O.round_bf16(-3.0)[()] == -3.0
    assert O.round_bf16(2.0 ** -140)[()] == 0.0 or abs(O.round_bf16(2.0 ** -140)[()]) <= 2.0 ** -133
    assert np.isinf(O.round_bf16(3.5e38)[()])


def test_store_f32_is_float32_rounding():
    x = RNG.standard_normal(1000)
    assert np.array_equal(O.store(x, "f32"), x.astype(np.float32).astype(np.float64))
    assert np.array_equal(O.store(x, "f64"), x)


# ---------------------------------------------------------------- RMSNorm
def test_rms_inv_constant_vector_closed_form():
    for c in (0.5, -2.0, 3e-3):
        x = np.full((1, 64), c)
        eps = 1e-6
        assert math.isclose(O.rms_inv(x, eps)[0], 1.0 / math.sqrt(c * c + eps), rel_tol=1e-14)
        h = x * O.rms_inv(x, eps)[:, None]
        assert np.allclose(h, np.sign(c) / math.sqrt(1 + eps / (c * c)), rtol=1e-14)


def test_rms_inv_matches_torch_rms_norm():
    x = RNG.standard_normal((7, 96))
    h = x * O.rms_inv(x, 1e-6)[:, None]
    ref = F.rms_norm(torch.from_numpy(x), (96,), eps=1e-6).numpy()
    assert np.allclose(h, ref, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- RoPE
def _rope_complex(x, pos, theta):
    """Rotate-half RoPE written as a complex rotation: (x_j + i x_{j+h}) * e^{i p w_j}."""
    hd = x.shape[-1]
    h = hd // 2
    xt = torch.from_numpy(x)
    z = torch.complex(xt[..., :h], xt[..., h:])
    w = torch.tensor([theta ** (-(2.0 * j) / hd) for j in range(h)], dtype=torch.float64)
    ang = torch.from_numpy(np.asarray(pos, dtype=np.float64))[:, None] * w[None, :]
    r = z * torch.polar(torch.ones_like(ang), ang)[:, None, :]
    return torch.cat([r.real, r.imag], dim=-1).numpy()


def test_rope_matches_complex_rotation():
    x = RNG.standard_normal((9, 3, 16))
    pos = np.array([0, 1, 2, 5, 17, 100, 511, 1000, 4095])
    assert np.allclose(O.rope(x, pos, 10000.0), _rope_complex(x, pos, 10000.0), rtol=1e-12, atol=1e-12)
    assert np.allclose(O.rope(x, pos, 5e5), _rope_complex(x, pos, 5e5), rtol=1e-12, atol=1e-12)


def test_rope_identity_at_zero_norm_preserving_and_relative():
    x = RNG.standard_normal((4, 2, 8))
    assert np.array_equal(O.rope(x, np.zeros(4), 1e4), x)
    y = O.rope(x, np.array([3, 7, 11, 100]), 1e4)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # q(m).k(n) depends only on m - n
    q = RNG.standard_normal((1, 1, 8))
    k = RNG.standard_normal((1, 1, 8))
    d1 = (O.rope(q, [5], 1e4) * O.rope(k, [2], 1e4)).sum()
    d2 = (O.rope(q, [45], 1e4) * O.rope(k, [42], 1e4)).sum()
    assert math.isclose(d1, d2, rel_tol=1e-10)
    # hd = 2: one pair rotated by exactly pos radians
    v = np.array([[[1.0, 0.0]]])
    assert np.allclose(O.rope(v, [1.0], 1e4)[0, 0], [math.cos(1.0), math.sin(1.0)], rtol=1e-14)


# ---------------------------------------------------------------- attention
def test_attention_matches_torch_sdpa():
    q = RNG.standard_normal((5, 3, 16))
    k = RNG.standard_normal((11, 3, 16))
    v = RNG.standard_normal((11, 3, 16))
    ref = F.scaled_dot_product_attention(
        torch.from_numpy(q).permute(1, 0, 2), torch.from_numpy(k).permute(1, 0, 2),
        torch.from_numpy(v).permute(1, 0, 2)).permute(1, 0, 2).numpy()
    assert np.allclose(O.attention(q, k, v), ref, rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    v = RNG.standard_normal((1, 2, 4))
    q = RNG.standard_normal((3, 2, 4))
    k = RNG.standard_normal((1, 2, 4))
    assert np.allclose(O.attention(q, k, v), np.broadcast_to(v, (3, 2, 4)))  # one key
    k6 = np.repeat(k, 6, axis=0)
    v6 = RNG.standard_normal((6, 2, 4))
    assert np.allclose(O.attention(q, k6, v6), v6.mean(axis=0, keepdims=True).repeat(3, 0))
    # permuting keys and values together changes nothing
    kk = RNG.standard_normal((6, 2, 4))
    p = RNG.permutation(6)
    assert np.allclose(O.attention(q, kk, v6), O.attention(q, kk[p], v6[p]), rtol=1e-13)


# ---------------------------------------------------------------- one layer
def _torch_layer(x, lw, dims, pos):
    """The layer of the model statement from torch library routines (float64)."""
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    X = t(x)
    R, H, hd = x.shape[0], dims.n_heads, dims.head_dim
    h = F.rms_norm(X, (dims.d,), eps=dims.rms_eps)
    q = F.linear(h, t(lw["wq"])).reshape(R, H, hd).numpy()
    k = F.linear(h, t(lw["wk"])).reshape(R, H, hd).numpy()
    v = F.linear(h, t(lw["wv"])).reshape(R, H, hd)
    q = t(_rope_complex(q, pos, dims.rope_theta)).permute(1, 0, 2)
    k = t(_rope_complex(k, pos, dims.rope_theta)).permute(1, 0, 2)
    a = F.scaled_dot_product_attention(q, k, v.permute(1, 0, 2)).permute(1, 0, 2).reshape(R, dims.d)
    X = X + F.linear(a, t(lw["wo"]))
    h2 = F.rms_norm(X, (dims.d,), eps=dims.rms_eps)
    X = X + F.linear(F.silu(F.linear(h2, t(lw["wg"]))) * F.linear(h2, t(lw["wu"])), t(lw["wd"]))
    return X.numpy()


DIMS64 = synth.ModelDims(n_layers=2, d=32, n_heads=2, head_dim=16, ffn=48, vocab=50,
                         mask_id=49, rope_theta=1e4, dtype="f64")


def _rand_layer(dims, scale=0.2):
    s = synth.layer_shapes(dims)
    return {n: scale * RNG.standard_normal(s[n]) for n in synth.LAYER_MATS}


def test_dense_layer_matches_torch_composition():
    lw = _rand_layer(DIMS64)
    x = RNG.standard_normal((13, 32))
    got, _, _ = O.dense_layer(x, lw, DIMS64)
    assert np.allclose(got, _torch_layer(x, lw, DIMS64, np.arange(13)), rtol=1e-11, atol=1e-12)


def test_layer_zero_output_projections_is_identity():
    lw = _rand_layer(DIMS64)
    lw["wo"] = np.zeros_like(lw["wo"])
    lw["wd"] = np.zeros_like(lw["wd"])
    x = RNG.standard_normal((5, 32))
    got, _, _ = O.dense_layer(x, lw, DIMS64)
    assert np.array_equal(got, x)


def test_partial_attention_equals_full_attention_rows():
    """A sparse layer on rows idx, over a cache holding stale K/V at idx and the
    dense K/V elsewhere, equals the dense layer restricted to idx."""
    lw = _rand_layer(DIMS64)
    x = RNG.standard_normal((12, 32))
    full, k, v = O.dense_layer(x, lw, DIMS64)
    idx = np.array([1, 4, 5, 11])
    kc, vc = k.copy(), v.copy()
    kc[idx] = 99.0
    vc[idx] = -99.0
    out = O.sparse_layer(x[idx], idx, kc, vc, lw, DIMS64)
    assert np.array_equal(out, full[idx])
    assert np.array_equal(kc, k) and np.array_equal(vc, v)


# ---------------------------------------------------------------- head
def test_head_matches_torch_softmax_max_and_argmax():
    d = DIMS64
    x = RNG.standard_normal((9, d.d))
    w = RNG.standard_normal((d.vocab, d.d))
    conf, tok, margin = O.head(x, w, d)
    lg = F.linear(F.rms_norm(torch.from_numpy(x), (d.d,), eps=d.rms_eps), torch.from_numpy(w))
    lg = torch.cat([lg[:, :d.mask_id], lg[:, d.mask_id + 1:]], dim=1)  # drop the mask column
    p = torch.softmax(lg, dim=1)
    assert np.allclose(conf, p.max(dim=1).values.float().double().numpy(), rtol=1e-6)
    am = torch.argmax(lg.float(), dim=1).numpy()
    am = am + (am >= d.mask_id)
    assert np.array_equal(tok, am)
    assert np.all(tok != d.mask_id)
    assert np.all(margin >= 0)


def test_head_equal_logits_and_mask_exclusion():
    d = dataclasses.replace(DIMS64, mask_id=0)
    x = np.ones((2, d.d))
    w = np.zeros((d.vocab, d.d))
    conf, tok, _ = O.head(x, w, d)
    assert np.allclose(conf, 1.0 / (d.vocab - 1), rtol=1e-7)
    assert np.array_equal(tok, [1, 1])          # lowest id that is not the mask
    w[0] = 50.0                                  # a huge logit on the mask id is ignored
    conf, tok, _ = O.head(x, w, d)
    assert np.array_equal(tok, [1, 1])
    assert np.allclose(conf, 1.0 / (d.vocab - 1), rtol=1e-7)
    w[7] = 10.0
    conf, tok, _ = O.head(x, w, d)
    assert np.array_equal(tok, [7, 7]) and np.all(conf > 0.99)


# ---------------------------------------------------------------- importance
def test_importance_hand_cases():
    g = json.load(open(os.path.join(HERE, "golden", "importance_hand.json")))
    for c in g["es"]:
        s = O.importance_es(np.array([c["x"]]), np.array([c["h"]]), np.array([c["conf"]]), c["alpha"])
        assert s[0] == np.float32(c["score"]), c
    for c in g["cos"]:
        s = O.importance_cos(np.array([c["x"]]), np.array([c["h"]]), np.array([c["conf"]]), c["lam"])
        assert s[0] == np.float32(c["score"]), c


def test_importance_unchanged_cache_and_limits():
    x = RNG.standard_normal((50, 64))
    conf = RNG.uniform(size=50)
    # unchanged cache: zero variation exactly
    assert np.array_equal(O.importance_es(x, x, conf, 0.5), O.store(0.5 * conf, "f32"))
    assert np.array_equal(O.importance_cos(x, x, conf, 0.5), O.store(0.5 * (1 - conf), "f32"))
    h = x + 0.3 * RNG.standard_normal((50, 64))
    # alpha = 1: pure confidence ranking; alpha = 0: pure variation ranking
    s1 = O.importance_es(x, h, conf, 1.0)
    assert np.array_equal(np.argsort(-s1, kind="stable"), np.argsort(-O.store(conf, "f32"), kind="stable"))
    s0 = O.importance_es(x, h, conf, 0.0)
    var = np.abs(x - h).sum(1) / (8.0 * np.linalg.norm(h, axis=1))
    assert np.allclose(s0, var, rtol=1e-6)
    # the variation term is scale invariant: scaling x and H together changes nothing
    assert np.allclose(O.importance_es(3 * x, 3 * h, conf, 0.5), O.importance_es(x, h, conf, 0.5), rtol=1e-6)
    # zero cache row: the floor keeps the score finite
    z = np.zeros((1, 64))
    assert np.isfinite(O.importance_es(x[:1], z, conf[:1], 0.5)).all()
    assert np.isfinite(O.importance_cos(x[:1], z, conf[:1], 0.5)).all()


# ---------------------------------------------------------------- top-k
def _brute_topk(s, k):
    """The k-subset whose every member outranks every non-member, found by
    enumerating all subsets (rank: NaN last, score descending, index ascending)."""
    L = len(s)
    vals = [0.0 if (v == 0 or math.isnan(v)) else float(v) for v in s]
    nan = [math.isnan(v) for v in s]

    def better(i, j):
        if nan[i] != nan[j]:
            return not nan[i]
        if vals[i] != vals[j]:
            return vals[i] > vals[j]
        return i < j

    for sub in itertools.combinations(range(L), k):
        rest = [j for j in range(L) if j not in sub]
        if all(better(i, j) for i in sub for j in rest):
            return list(sub)
    raise AssertionError("no valid subset")


def test_topk_matches_brute_force_with_ties():
    for trial in range(300):
        L = int(RNG.integers(1, 9))
        k = int(RNG.integers(1, L + 1))
        s = RNG.choice([0.0, -0.0, 0.5, 0.25, -1.0, 0.5, 2.0, np.nan], size=L).astype(np.float32)
        assert list(O.topk_select(s, k)) == _brute_topk(list(s), k), (s, k)


def test_topk_edge_cases_and_sort_reference():
    s = np.zeros(10, dtype=np.float32)
    assert list(O.topk_select(s, 3)) == [0, 1, 2]                     # all equal -> first k
    s = np.array([-0.0, 0.0, -0.0], dtype=np.float32)
    assert list(O.topk_select(s, 2)) == [0, 1]                        # -0 == +0
    s = RNG.standard_normal(300).astype(np.float32)
    assert list(O.topk_select(s, 300)) == list(range(300))             # k = L
    assert list(O.topk_select(s, 1)) == [int(np.argmax(s))]            # k = 1
    ref = sorted(range(300), key=lambda i: (-float(s[i]), i))[:37]
    assert list(O.topk_select(s, 37)) == sorted(ref)
    assert O.topk_margin(s, 37) == float(s[ref[36]]) - float(s[sorted(range(300), key=lambda i: (-float(s[i]), i))[37]])


def test_keep_count():
    assert O.keep_count(0.25, 768) == 192
    assert O.keep_count(0.20, 512) == 103
    assert O.keep_count(0.10, 1536) == 154
    assert O.keep_count(0.25, 1536) == 384
    assert O.keep_count(0.50, 1536) == 768
    assert O.keep_count(0.25, 128) == 32
    assert O.keep_count(1.0, 77) == 77
    assert O.keep_count(0.0, 77) == 1


# ---------------------------------------------------------------- remask
def test_remask_brute_force():
    for trial in range(200):
        L = 16
        b0, b1 = 4, 12
        masked = (RNG.uniform(size=L) < 0.6).astype(np.uint8)
        conf = RNG.choice([0.1, 0.2, 0.2, 0.7, 0.9], size=L).astype(np.float32)
        tok_c = RNG.integers(0, 100, size=L).astype(np.int32)
        tok = np.full(L, 99, dtype=np.int32)
        n = int(RNG.integers(1, 5))
        t0, m0 = tok.copy(), masked.copy()
        pick, _ = O.remask(tok, masked, conf, tok_c, b0, b1, n)
        cand = [i for i in range(b0, b1) if m0[i]]
        want = sorted(sorted(cand, key=lambda i: (-float(conf[i]), i))[:n])
        assert list(pick) == want
        assert m0.sum() - masked.sum() == min(n, len(cand))
        for i in range(L):
            if i in want:
                assert tok[i] == tok_c[i] and masked[i] == 0
            else:
                assert tok[i] == t0[i] and masked[i] == m0[i]


# ---------------------------------------------------------------- the step
TINY = synth.TINY
TINY_W = None


def _tiny():
    global TINY_W
    if TINY_W is None:
        TINY_W = O.prepare_weights(synth.model_weights_f32(TINY), TINY)
    return TINY_W


def _tiny_state_after_refresh():
    w = _tiny()
    run = synth.TINY_RUN
    prompt = synth.prompt_ids(TINY, 1, 64)
    tok = np.full((1, 128), TINY.mask_id, dtype=np.int32)
    tok[:, :64] = prompt
    masked = np.zeros((1, 128), dtype=np.uint8)
    masked[:, 64:] = 1
    st = O.new_state(TINY, run, tok, masked)
    O.dense_step(w, TINY, run, st, 64, 96, 4)
    return w, run, st


def test_sparse_step_with_all_rows_equals_dense_step():
    w, run, st = _tiny_state_after_refresh()
    a, b = st.copy(), st.copy()
    O.dense_step(w, TINY, run, a, 64, 96, 4)
    O.sparse_step(w, TINY, run, b, 64, 96, 4, k=128)
    for f in ("tok", "masked", "hc", "conf_c", "tok_c"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    for i in range(len(a.kc)):
        assert np.array_equal(a.kc[i], b.kc[i]) and np.array_equal(a.vc[i], b.vc[i])


def test_sparse_step_cache_semantics():
    w, run, st = _tiny_state_after_refresh()
    before = st.copy()
    info = O.sparse_step(w, TINY, run, st, 64, 96, 4)
    idx = info["idx"][0]
    assert len(idx) == 32 and np.all(np.diff(idx) > 0)
    skip = np.setdiff1d(np.arange(128), idx)
    # skipped rows: byte-identical caches
    assert np.array_equal(st.hc[0][skip], before.hc[0][skip])
    for i in range(len(st.kc)):
        assert np.array_equal(st.kc[i][0][skip], before.kc[i][0][skip])
        assert np.array_equal(st.vc[i][0][skip], before.vc[i][0][skip])
    assert np.array_equal(st.conf_c[0][skip], before.conf_c[0][skip])
    assert np.array_equal(st.tok_c[0][skip], before.tok_c[0][skip])
    # selected rows: the H cache holds this step's skip-layer input, and the
    # layer-l_s K/V cache holds a fresh projection of it
    assert np.array_equal(st.hc[0][idx], info["x_ls"][0][idx])
    lw = w["layers"][run.skip_layer]
    _, k, v = O.dense_layer(info["x_ls"][0], lw, TINY)
    assert np.array_equal(st.kc[0][0][idx], k[idx]) and np.array_equal(st.vc[0][0][idx], v[idx])
    # exactly n unmasked in the block; the prompt never changes
    assert before.masked[0].sum() - st.masked[0].sum() == 4
    assert np.array_equal(st.tok[0][:64], before.tok[0][:64])


def test_generate_keep_all_equals_vanilla_and_fills_blocks():
    w = _tiny()
    run = synth.TINY_RUN
    prompt = synth.prompt_ids(TINY, 1, 64)
    a, log_a = O.generate(w, TINY, run, prompt, 64, 32, 4, k=128)
    b, _ = O.generate(w, TINY, run, prompt, 64, 32, 4, vanilla=True)
    assert np.array_equal(a, b)
    assert np.all(a != TINY.mask_id)
    assert len(log_a) == 16 and sum(l["dense"] for l in log_a) == 2
    c, log_c = O.generate(w, TINY, run, prompt, 64, 32, 4)
    assert np.all(c != TINY.mask_id)
    assert all(len(l["unmasked"][0]) == 4 for l in log_c)


# ------------------------------------------------------- DyLLM context saliency
def test_context_cosine_closed_forms():
    """"DyLLM", technical summary section 2.A: identical, scaled, orthogonal,
    anti-parallel and zero contexts, and a hand-evaluated pair."""
    a = RNG.standard_normal((1, 64))
    ortho = np.zeros((1, 64)); ortho[0, 0] = 1.0
    e1 = np.zeros((1, 64)); e1[0, 1] = 2.0
    cur = np.concatenate([a, a, ortho, a, np.zeros((1, 64)), np.array([[1.0, 0.0] + [0.0] * 62])])
    prev = np.concatenate([a, 3.0 * a, e1, -a, a, np.array([[1.0, 1.0] + [0.0] * 62])])
    s = O.context_cosine(cur, prev)
    assert s.dtype == np.float32 or s.dtype == np.float64
    np.testing.assert_allclose(s[:2], [1.0, 1.0], atol=1e-7)      # unchanged, scale-invariant
    assert s[2] == 0.0                                             # orthogonal
    np.testing.assert_allclose(s[3], -1.0, atol=1e-7)              # anti-parallel
    assert s[4] == 0.0                                             # zero row: floored, no NaN
    np.testing.assert_allclose(s[5], np.float32(1.0 / math.sqrt(2.0)), rtol=0, atol=0)  # hand value


def test_context_cosine_matches_torch_cosine_similarity():
    cur = RNG.standard_normal((37, 96))
    prev = cur + 0.3 * RNG.standard_normal((37, 96))
    want = F.cosine_similarity(torch.from_numpy(cur), torch.from_numpy(prev), dim=-1, eps=1e-12).numpy()
    np.testing.assert_allclose(O.context_cosine(cur, prev), want.astype(np.float32), rtol=0, atol=1e-7)


def test_salient_rows_brute_force():
    """Ascending indices of the rows below tau, compared in float32; values
    equal to tau are not salient; NaN never is."""
    sim = np.array([0.5, 0.9, 0.2, np.nan, 0.7, 0.7, 1.0, -0.3], dtype=np.float32)
    assert O.salient_rows(sim, 0.7).tolist() == [0, 2, 7]
    assert O.salient_rows(sim, 1.1).tolist() == [0, 1, 2, 4, 5, 6, 7]
    assert O.salient_rows(sim, -1.0).tolist() == []
    for _ in range(20):
        s = RNG.choice(np.linspace(-1, 1, 9), 50).astype(np.float32)
        tau = float(RNG.choice(np.linspace(-1, 1, 9)))
        brute = [i for i in range(50) if float(s[i]) < float(np.float32(tau))]
        assert O.salient_rows(s, tau).tolist() == brute


def test_dyllm_layer_against_the_dense_layer():
    """"DyLLM", technical summary section 2.B.1: salient rows equal a fresh
    dense layer, the others keep their cached output; a refresh is the dense
    layer; an unchanged context selects nothing; tau above 1 selects every
    finite row, below -1 none."""
    dims = dataclasses.replace(synth.SMALL_BF16, n_layers=1, d=256, n_heads=2, ffn=512, vocab=64, mask_id=63)
    w = O.prepare_weights(synth.model_weights_f32(dims), dims)
    lw = w["layers"][0]
    L = 24
    x = O.store(RNG.standard_normal((L, dims.d)), "bf16")
    dense, _, _ = O.dense_layer(x, lw, dims)
    out0, c0, sal0, _ = O.dyllm_layer(x, lw, dims, None, None, 0.5, refresh=True)
    assert np.array_equal(out0, dense) and sal0.tolist() == list(range(L))
    # unchanged input: the context repeats, cosine exactly 1, nothing recomputed
    out1, c1, sal1, sim1 = O.dyllm_layer(x, lw, dims, c0, out0, 0.999, refresh=False)
    assert np.all(sim1 == 1.0) and len(sal1) == 0 and np.array_equal(out1, out0)
    # moved rows: the salient ones equal the dense layer of the new input
    x2 = x.copy()
    x2[[3, 10]] = O.store(RNG.standard_normal((2, dims.d)), "bf16")
    dense2, _, _ = O.dense_layer(x2, lw, dims)
    stale = O.store(RNG.standard_normal((L, dims.d)), "bf16")
    out2, _, sal2, sim2 = O.dyllm_layer(x2, lw, dims, c0, stale, 0.95, refresh=False)
    assert {3, 10} <= set(sal2.tolist())
    assert np.array_equal(out2[sal2], dense2[sal2])
    rest = np.setdiff1d(np.arange(L), sal2)
    assert np.array_equal(out2[rest], stale[rest])
    assert np.array_equal(O.dyllm_layer(x2, lw, dims, c0, stale, 1.5, refresh=False)[2], np.arange(L))
    assert len(O.dyllm_layer(x2, lw, dims, c0, stale, -1.5, refresh=False)[2]) == 0


def test_two_skip_points_reduce_to_one():
    """"ES-dLLM", technical summary section 2.B (skip points at early layers,
    k = (1 - r_l)|S| over the tokens that reach the layer): keeping every row
    at the second point is the single-skip step; keeping every row at the first
    point and skipping at l_s2 is the single-skip step at l_s2."""
    dims = dataclasses.replace(synth.TINY, n_layers=4)
    w = O.prepare_weights(synth.model_weights_f32(dims), dims)
    B, P, G = 2, 24, 16
    L = P + G
    prompt = synth.prompt_ids(dims, B, P)
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = prompt
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    one = dataclasses.replace(synth.TINY_RUN, skip_layer=1, keep_ratio=0.5)
    two = dataclasses.replace(one, skip_layer2=3, keep_ratio2=1.0)
    sa, sb = O.new_state(dims, one, tok, masked), O.new_state(dims, two, tok, masked)
    O.dense_step(w, dims, one, sa, P, P + 8, 2)
    O.dense_step(w, dims, two, sb, P, P + 8, 2)
    O.sparse_step(w, dims, one, sa, P, P + 8, 2)
    info = O.sparse_step(w, dims, two, sb, P, P + 8, 2)
    assert np.array_equal(info["idx2"][0], info["idx"][0])
    for f in ("tok", "masked", "hc", "conf_c", "tok_c"):
        assert np.array_equal(getattr(sa, f), getattr(sb, f)), f
    for i in range(len(sa.kc)):
        assert np.array_equal(sa.kc[i], sb.kc[i]) and np.array_equal(sa.vc[i], sb.vc[i])
    # keep all at l_s = 1, skip at 3 with 50%  ==  a single skip point at 3
    full = dataclasses.replace(one, keep_ratio=1.0, skip_layer2=3, keep_ratio2=0.5)
    at3 = dataclasses.replace(one, skip_layer=3, keep_ratio=0.5)
    sc, sd = O.new_state(dims, full, tok, masked), O.new_state(dims, at3, tok, masked)
    O.dense_step(w, dims, full, sc, P, P + 8, 2)
    O.dense_step(w, dims, at3, sd, P, P + 8, 2)
    info_c = O.sparse_step(w, dims, full, sc, P, P + 8, 2)
    info_d = O.sparse_step(w, dims, at3, sd, P, P + 8, 2)
    for b in range(B):
        assert np.array_equal(info_c["idx2"][b], info_d["idx"][b])
    for f in ("tok", "masked", "conf_c", "tok_c"):
        assert np.array_equal(getattr(sc, f), getattr(sd, f)), f
    assert np.array_equal(sc.hc2, sd.hc)
    for i in range(len(sd.kc)):   # layers >= 3: cache index 2 + i in the two-point state
        assert np.array_equal(sc.kc[2 + i], sd.kc[i]) and np.array_equal(sc.vc[2 + i], sd.vc[i])


def test_score_on_keys_matches_the_dense_layers_keys():
    """"ES-dLLM", technical summary section 2.A (the variation of an
    intermediate tensor): scoring on K uses the skip layer's keys, which the
    separately written dense layer also returns (and likewise V)."""
    dims = dataclasses.replace(synth.TINY, n_layers=3)
    w = O.prepare_weights(synth.model_weights_f32(dims), dims)
    B, P, G = 1, 24, 16
    L = P + G
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = synth.prompt_ids(dims, B, P)
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    for tensor in ("k", "v"):
        run = dataclasses.replace(synth.TINY_RUN, score_mode="es", alpha=0.5, skip_layer=1, keep_ratio=0.5,
                                  score_tensor=tensor)
        st = O.new_state(dims, run, tok, masked)
        O.dense_step(w, dims, run, st, P, P + 8, 2)
        before = st.copy()
        info = O.sparse_step(w, dims, run, st, P, P + 8, 2)
        x = O.embed(before.tok[0], w)
        x, _, _ = O.dense_layer(x, w["layers"][0], dims)
        _, k1, v1 = O.dense_layer(x, w["layers"][1], dims)
        fresh = (k1 if tensor == "k" else v1).reshape(L, dims.d)
        cache = (before.kc[0] if tensor == "k" else before.vc[0])[0].reshape(L, dims.d)
        want = np.float32(0.5) * before.conf_c[0] + 0.5 * np.abs(fresh - cache).sum(-1) / np.maximum(
            math.sqrt(dims.d) * np.sqrt((cache * cache).sum(-1)), 1e-12)
        np.testing.assert_allclose(info["scores"][0], want.astype(np.float32), rtol=1e-6, atol=1e-7)


def test_block_scope():
    """Selection scoped to the current block ("ES-dLLM", technical summary
    section 2.B, refresh of "the prompt or the current block"): over the whole
    sequence it is the step over all positions (the early layers with their
    caches compute what the dense early layers compute); over a block, every
    row outside it keeps every cache byte for byte."""
    dims = dataclasses.replace(synth.TINY, n_layers=3)
    w = O.prepare_weights(synth.model_weights_f32(dims), dims)
    B, P, G = 2, 24, 16
    L = P + G
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = synth.prompt_ids(dims, B, P)
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    allrun = dataclasses.replace(synth.TINY_RUN, skip_layer=1, keep_ratio=0.5)
    blkrun = dataclasses.replace(allrun, scope="block")
    sa, sb = O.new_state(dims, allrun, tok, masked), O.new_state(dims, blkrun, tok, masked)
    assert len(sb.kc) == dims.n_layers and len(sa.kc) == dims.n_layers - 1
    O.dense_step(w, dims, allrun, sa, 0, L, 2)
    O.dense_step(w, dims, blkrun, sb, 0, L, 2)
    ia = O.sparse_step(w, dims, allrun, sa, 0, L, 2)
    ib = O.sparse_step(w, dims, blkrun, sb, 0, L, 2)
    for b in range(B):
        assert np.array_equal(ia["idx"][b], ib["idx"][b])
    for f in ("tok", "masked", "hc", "conf_c", "tok_c"):
        assert np.array_equal(getattr(sa, f), getattr(sb, f)), f
    for i in range(len(sa.kc)):
        assert np.array_equal(sa.kc[i], sb.kc[i + 1]) and np.array_equal(sa.vc[i], sb.vc[i + 1])
    # a block: the rows outside it keep every cache
    before = sb.copy()
    info = O.sparse_step(w, dims, blkrun, sb, P, P + 8, 2)
    out = np.r_[0:P, P + 8:L]
    for b in range(B):
        assert np.all((info["idx"][b] >= P) & (info["idx"][b] < P + 8)) and len(info["idx"][b]) == 4
        for i in range(len(sb.kc)):
            assert np.array_equal(sb.kc[i][b][out], before.kc[i][b][out])
        assert np.array_equal(sb.hc[b][out], before.hc[b][out])
        assert np.array_equal(sb.conf_c[b][out], before.conf_c[b][out])


def test_approx_contexts_exact_limits():
    """"DyLLM", technical summary section 2.B.2: with queries and keys
    unchanged the update of the stable rows by the salient rows' change of
    values is exact (attention is linear in V), so the result equals exact
    attention with the new values; every row salient is exact attention; no
    row salient keeps the cached contexts."""
    L, H, hd = 40, 3, 16
    q = RNG.standard_normal((L, H, hd))
    k = RNG.standard_normal((L, H, hd))
    v_prev = RNG.standard_normal((L, H, hd))
    s = np.einsum("ihd,jhd->hij", q, k) / math.sqrt(hd)
    e = np.exp(s - s.max(-1, keepdims=True))
    p_prev = e / e.sum(-1, keepdims=True)
    c_prev = O.attention(q, k, v_prev)
    changed = np.array([2, 7, 19, 33])
    v = v_prev.copy()
    v[changed] = RNG.standard_normal((len(changed), H, hd))
    want = O.attention(q, k, v)
    c, p = O.approx_contexts(q, k, v, v_prev, c_prev, p_prev, changed)
    np.testing.assert_allclose(c, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(p, p_prev, rtol=0, atol=1e-13)
    c_all, _ = O.approx_contexts(q, k, v, v_prev, c_prev, p_prev, np.arange(L))
    np.testing.assert_allclose(c_all, want, rtol=0, atol=1e-12)
    c_none, p_none = O.approx_contexts(q, k, v, v_prev, c_prev, p_prev, [])
    assert np.array_equal(c_none, c_prev) and np.array_equal(p_none, p_prev)
    # moved keys: the stable rows keep the stale probabilities (an approximation)
    k2 = k.copy()
    k2[changed] += 0.5 * RNG.standard_normal((len(changed), H, hd))
    c2, _ = O.approx_contexts(q, k2, v, v_prev, c_prev, p_prev, changed)
    exact2 = O.attention(q, k2, v)
    np.testing.assert_allclose(c2[changed], exact2[changed], rtol=0, atol=1e-12)
    stable = np.setdiff1d(np.arange(L), changed)
    assert np.abs(c2[stable] - exact2[stable]).max() > 1e-6


def test_approx_contexts_hand_cases_with_moved_keys():
    """"DyLLM", technical summary section 2.B.2, on hand-evaluated cases where
    the keys moved since the cached probabilities were taken
    (tests/golden/approx_moved_keys.json): the stable rows must be updated with
    their cached probabilities P_prev[i, j] (row i, column j of the moved row),
    the moved rows get exact softmax rows over the new keys, and only the
    moved rows' probabilities are rewritten."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "approx_moved_keys.json")) as f:
        g = json.load(f)
    cm = g["common"]
    q = np.array(cm["q"])[:, None, :]
    k = np.array(cm["k"])[:, None, :]
    v_prev = np.array(cm["v_prev"])[:, None, :]
    c_prev = np.array(cm["c_prev"])[:, None, :]
    p_prev = np.array(cm["p_prev"])[None]
    for case in g["cases"]:
        v = np.array(case["v"])[:, None, :]
        c, p = O.approx_contexts(q, k, v, v_prev, c_prev, p_prev, case["changed"])
        np.testing.assert_allclose(c[:, 0, :], np.array(case["c"]), rtol=0, atol=1e-12, err_msg=case["name"])
        np.testing.assert_allclose(p[0], np.array(case["p"]), rtol=0, atol=1e-12, err_msg=case["name"])


def _tiny_state(dims, run, B, P, G):
    L = P + G
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = synth.prompt_ids(dims, B, P)
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    return O.new_state(dims, run, tok, masked)


def test_response_only_scope():
    """Response-only steps ("DyLLM", technical summary section 2.B.3: only the
    response tokens are processed; the whole context only at intervals):
    (1) with no prompt the response is the whole sequence and the step is the
    step over all positions; (2) right after a full step, with the tokens
    unchanged and every response row kept, a response-only step reproduces the
    full step on every response row (the prompt's cached K/V are then exact)
    and leaves every prompt row's caches byte for byte; (3) when the response
    is one block, it is the block-scoped step."""
    dims = dataclasses.replace(synth.TINY, n_layers=3)
    w = O.prepare_weights(synth.model_weights_f32(dims), dims)
    base = dataclasses.replace(synth.TINY_RUN, skip_layer=1, keep_ratio=0.5)
    resp = dataclasses.replace(base, scope="response")
    B, G = 2, 16
    # (1) no prompt
    sa, sr = _tiny_state(dims, base, B, 0, G), _tiny_state(dims, resp, B, 0, G)
    O.dense_step(w, dims, base, sa, 0, 8, 2)
    O.dense_step(w, dims, resp, sr, 0, 8, 2)
    ia = O.sparse_step(w, dims, base, sa, 0, 8, 2)
    ir = O.sparse_step(w, dims, resp, sr, 0, 8, 2, region=(0, G))
    for b in range(B):
        assert np.array_equal(ia["idx"][b], ir["idx"][b])
    for f in ("tok", "masked", "hc", "conf_c", "tok_c"):
        assert np.array_equal(getattr(sa, f), getattr(sr, f)), f
    for i in range(len(sa.kc)):
        assert np.array_equal(sa.kc[i], sr.kc[i + 1]) and np.array_equal(sa.vc[i], sr.vc[i + 1])
    # (2) after a full step, unchanged tokens, keep every row: = the full step
    P = 24
    L = P + G
    keep1 = dataclasses.replace(resp, keep_ratio=1.0)
    st = _tiny_state(dims, keep1, B, P, G)
    O.dense_step(w, dims, keep1, st, 0, 8, 2)   # block inside the prompt: nothing unmasked
    full = st.copy()
    O.dense_step(w, dims, keep1, full, 0, 8, 2)
    before = st.copy()
    info = O.sparse_step(w, dims, keep1, st, 0, 8, 2, region=(P, L))
    for b in range(B):
        assert np.array_equal(info["idx"][b], np.arange(P, L))
        for i in range(len(st.kc)):
            assert np.array_equal(st.kc[i][b][P:], full.kc[i][b][P:])
            assert np.array_equal(st.vc[i][b][P:], full.vc[i][b][P:])
            assert np.array_equal(st.kc[i][b][:P], before.kc[i][b][:P])
        assert np.array_equal(st.hc[b][P:], full.hc[b][P:]) and np.array_equal(st.hc[b][:P], before.hc[b][:P])
        assert np.array_equal(st.conf_c[b], full.conf_c[b]) and np.array_equal(st.tok_c[b], full.tok_c[b])
    assert np.array_equal(st.tok, before.tok)
    # (3) a one-block response: the block-scoped step
    blk = dataclasses.replace(base, scope="block")
    s1, s2 = _tiny_state(dims, resp, B, P, G), _tiny_state(dims, blk, B, P, G)
    O.dense_step(w, dims, resp, s1, P, L, 2)
    O.dense_step(w, dims, blk, s2, P, L, 2)
    i1 = O.sparse_step(w, dims, resp, s1, P, L, 2, region=(P, L))
    i2 = O.sparse_step(w, dims, blk, s2, P, L, 2)
    for b in range(B):
        assert np.array_equal(i1["idx"][b], i2["idx"][b])
    for f in ("tok", "masked", "hc", "conf_c", "tok_c"):
        assert np.array_equal(getattr(s1, f), getattr(s2, f)), f
    for i in range(len(s1.kc)):
        assert np.array_equal(s1.kc[i], s2.kc[i]) and np.array_equal(s1.vc[i], s2.vc[i])


def test_response_only_generation_refreshes_every_interval():
    """A response-only generation takes a full step at the start of every
    block and every refresh_interval steps; in between the prompt rows'
    caches never change; the prompt itself is never rewritten."""
    dims = dataclasses.replace(synth.TINY, n_layers=3)
    w = O.prepare_weights(synth.model_weights_f32(dims), dims)
    run = dataclasses.replace(synth.TINY_RUN, skip_layer=1, keep_ratio=0.5, scope="response", refresh_interval=4)
    prompt = synth.prompt_ids(dims, 1, 24)
    out, log = O.generate(w, dims, run, prompt, 32, 16, 2)
    dense = [l["dense"] for l in log]
    assert dense == [j % 8 in (0, 4) for j in range(16)]
    assert out.shape == (1, 32) and not np.any(out == dims.mask_id)
    for l in log:
        if not l["dense"]:
            assert all(np.all(ix >= 24) for ix in l["idx"])


def test_dyllm_layer_approx_limits():
    """The DyLLM layer with the approximate attention ("DyLLM", technical
    summary section 2.B.2): a refresh is the exact DyLLM layer; a call whose
    input moved on every row is the exact layer (every row exact); a call
    whose input did not move reuses every cached context, so nothing is
    salient and the cached output comes back; with some rows moved, the moved
    rows' contexts are exact and the others follow approx_contexts."""
    dims = dataclasses.replace(synth.SMALL_BF16, n_layers=2)
    w = O.prepare_weights(synth.model_weights_f32(dims), dims)
    lw = w["layers"][0]
    L = 24
    rng = np.random.default_rng(77)
    x0 = O.store(rng.standard_normal((L, dims.d)), "bf16")
    cache = {}
    out0, a0, sal0, sim0, mv0 = O.dyllm_layer_approx(x0, lw, dims, cache, 0.9, True)
    want0, c0, _, _ = O.dyllm_layer(x0, lw, dims, None, None, 0.9, True)
    assert np.array_equal(out0, want0) and np.array_equal(a0, c0) and len(mv0) == L and sim0 is None
    # nothing moved: every context repeats, nothing salient, cached output
    c_saved = {k_: np.array(v_, copy=True) for k_, v_ in cache.items()}
    out1, a1, sal1, sim1, mv1 = O.dyllm_layer_approx(x0, lw, dims, cache, 0.9, False)
    assert len(mv1) == 0 and np.array_equal(a1, c_saved["c"]) and np.all(sim1 == 1.0) and len(sal1) == 0
    assert np.array_equal(out1, c_saved["out"])
    # every row moved: the exact layer (the same salient decisions)
    x2 = O.store(x0 + rng.standard_normal((L, dims.d)), "bf16")
    out2, a2, sal2, sim2, mv2 = O.dyllm_layer_approx(x2, lw, dims, cache, 0.99, False)
    want2, c2, sal_w, sim_w = O.dyllm_layer(x2, lw, dims, a1, out1, 0.99, False)
    assert len(mv2) == L and np.array_equal(a2, c2) and np.array_equal(sal2, sal_w) and np.array_equal(out2, want2)
    # some rows moved: exact contexts for them, approx_contexts for the rest
    x3 = x2.copy()
    moved = np.array([3, 10, 17])
    x3[moved] = O.store(x3[moved] + rng.standard_normal((3, dims.d)), "bf16")
    before = {k_: np.array(v_, copy=True) for k_, v_ in cache.items()}
    out3, a3, sal3, sim3, mv3 = O.dyllm_layer_approx(x3, lw, dims, cache, 0.9, False)
    assert np.array_equal(mv3, moved)
    from oracle.model import _qkv
    q, k, v = _qkv(x3, np.arange(L), lw, dims)
    H, hd = dims.n_heads, dims.head_dim
    c_want, p_want = O.approx_contexts(q, k, v, before["v"], before["c"].reshape(L, H, hd), before["p"], moved)
    assert np.array_equal(a3, O.store(c_want, "bf16").reshape(L, dims.d))
    exact = O.store(O.attention(q, k, v), "bf16").reshape(L, dims.d)
    assert np.array_equal(a3[moved], exact[moved])
    assert np.allclose(cache["p"][:, moved, :], O.attention_probs(q[moved], k), rtol=0, atol=1e-14)
    stable = np.setdiff1d(np.arange(L), moved)
    assert np.array_equal(cache["p"][:, stable, :], before["p"][:, stable, :])
