"""Two skip points ("ES-dLLM: Efficient Inference for Diffusion Large Language
Models by Early-Skipping", technical summary section 2.B: skipping at early
layers such as 4 and 8 of 32, k = (1 - r_l)|S| over the tokens that reach
each point) on the GPU: a float32 generation with two skip points equals the
oracle's token for token, a second point that keeps every row reproduces the
single-point step bit for bit, and the refresh-interval variant (ES-dLLM*)
the scores on the skip layer's keys or values (section 2.A) and the
selection scoped to the current block (section 2.B, refresh of "the prompt or
the current block") generate the oracle's tokens too.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import assert_parity, make_context, to_gpu, to_np

pytestmark = pytest.mark.gpu


def _generate_both(dims, run, seq):
    ctx, w = make_context(dims, run, seq["batch"], seq["prompt"] + seq["gen"])
    prompt = synth.prompt_ids(dims, seq["batch"], seq["prompt"])
    want, log = O.generate(w, dims, run, prompt, seq["gen"], seq["block"], seq["n_unmask"])
    got = ctx.generate(torch.from_numpy(prompt), seq["gen"], seq["block"], seq["n_unmask"]).cpu().numpy()
    ctx.close()
    tk = min((m for l in log if not l["dense"] for m in l["topk_margin"]), default=np.inf)
    rm = min(m for l in log for m in l["remask_margin"])
    return got, want, tk, rm


def test_tiny_generation_two_skip_points():
    """4 float32 layers, skip points 1 (keep 50%) and 3 (keep 50% of those)."""
    dims = dataclasses.replace(synth.TINY, n_layers=4)
    run = dataclasses.replace(synth.TINY_RUN, skip_layer=1, keep_ratio=0.5, skip_layer2=3, keep_ratio2=0.5)
    got, want, tk, rm = _generate_both(dims, run, synth.TINY_SEQ)
    print(f"smallest top-k margin {tk:.3e}, smallest remask margin {rm:.3e}")
    assert np.array_equal(got, want), f"{int((got != want).sum())} tokens differ"


def test_tiny_generation_refresh_interval():
    """ES-dLLM*: a dense refresh every 3 steps of a block as well."""
    run = dataclasses.replace(synth.TINY_RUN, refresh_interval=3)
    got, want, tk, rm = _generate_both(synth.TINY, run, synth.TINY_SEQ)
    assert np.array_equal(got, want), f"{int((got != want).sum())} tokens differ"


@pytest.mark.parametrize("tensor", ["k", "v"])
def test_tiny_generation_score_on_keys_or_values(tensor):
    run = dataclasses.replace(synth.TINY_RUN, score_tensor=tensor)
    got, want, tk, rm = _generate_both(synth.TINY, run, synth.TINY_SEQ)
    print(f"score on {tensor}: smallest top-k margin {tk:.3e}, smallest remask margin {rm:.3e}")
    assert np.array_equal(got, want), f"{int((got != want).sum())} tokens differ"


def test_tiny_generation_block_scope():
    """Every layer recomputes only the current block's rows over cached K/V;
    k = 50% of the block (16 of 32)."""
    dims = dataclasses.replace(synth.TINY, n_layers=3)
    run = dataclasses.replace(synth.TINY_RUN, skip_layer=1, keep_ratio=0.5, scope="block")
    got, want, tk, rm = _generate_both(dims, run, synth.TINY_SEQ)
    print(f"block scope: smallest top-k margin {tk:.3e}, smallest remask margin {rm:.3e}")
    assert np.array_equal(got, want), f"{int((got != want).sum())} tokens differ"


def test_block_scope_keeps_other_rows_caches():
    """bf16: after a block-scoped sparse step, every row outside the block has
    byte-identical caches at every layer, and the block's selected rows moved."""
    dims = synth.SMALL_BF16
    run = dataclasses.replace(synth.SMALL_BF16_RUN, skip_layer=2, keep_ratio=0.5, scope="block")
    B, P, G = 2, 64, 64
    L = P + G
    ctx, _ = make_context(dims, run, B, L)
    prompt = synth.prompt_ids(dims, B, P)
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = prompt
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    tg, mg = to_gpu(tok, torch.int32), to_gpu(masked, torch.uint8)
    ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=True)
    v = ctx.state(B, L)
    assert len(v["k_cache"]) == dims.n_layers
    before = {"h": to_np(v["h_cache"]).copy(), "conf": to_np(v["conf_cache"]).copy(),
              "k": [to_np(t).copy() for t in v["k_cache"]], "v": [to_np(t).copy() for t in v["v_cache"]]}
    ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=False)
    ctx.sync_check()
    out = np.r_[0:P, P + 32:L]
    after_k = [to_np(t) for t in v["k_cache"]]
    for b in range(B):
        assert np.array_equal(to_np(v["h_cache"])[b][out], before["h"][b][out])
        assert np.array_equal(to_np(v["conf_cache"])[b][out], before["conf"][b][out])
        for i in range(dims.n_layers):
            assert np.array_equal(after_k[i][b][out], before["k"][i][b][out]), i
            assert np.array_equal(to_np(v["v_cache"][i])[b][out], before["v"][i][b][out]), i
        # the early layers recomputed every row of the block (their K moved: the
        # block's tokens changed by the remask of the dense step)
        assert not np.array_equal(after_k[0][b][P:P + 32], before["k"][0][b][P:P + 32])
    ctx.close()


def test_tiny_generation_response_only_steps():
    """Response-only steps ("DyLLM", technical summary section 2.B.3): every
    layer recomputes only the rows after the prompt over the prompt's cached
    K/V, a full step at the start of every block and every 4 steps; k = 50% of
    the response rows; token-identical to the oracle's generation."""
    dims = dataclasses.replace(synth.TINY, n_layers=3)
    run = dataclasses.replace(synth.TINY_RUN, skip_layer=1, keep_ratio=0.5, scope="response", refresh_interval=4)
    got, want, tk, rm = _generate_both(dims, run, synth.TINY_SEQ)
    print(f"response-only: smallest top-k margin {tk:.3e}, smallest remask margin {rm:.3e}")
    assert np.array_equal(got, want), f"{int((got != want).sum())} tokens differ"


def test_response_only_step_keeps_prompt_caches_and_matches_oracle():
    """bf16: a response-only sparse step after a full step leaves every prompt
    row's caches byte for byte, recomputes the response rows in every layer,
    and (teacher-forced: the oracle gets the GPU's state after the full step)
    matches the oracle's response-only step on every cache."""
    dims = synth.SMALL_BF16
    run = dataclasses.replace(synth.SMALL_BF16_RUN, skip_layer=2, keep_ratio=0.5, scope="response")
    B, P, G = 2, 64, 64
    L = P + G
    ctx, w = make_context(dims, run, B, L)
    prompt = synth.prompt_ids(dims, B, P)
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = prompt
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    tg, mg = to_gpu(tok, torch.int32), to_gpu(masked, torch.uint8)
    ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=True)
    with pytest.raises(Exception):   # a sparse response-only step needs its region
        ctx.denoise_step(tg.clone(), mg.clone(), P, P + 32, 2, force_dense=False)
    ctx.sync_check()
    v = ctx.state(B, L)
    assert len(v["k_cache"]) == dims.n_layers
    st = O.new_state(dims, run, to_np(tg), to_np(mg))
    st.hc = to_np(v["h_cache"]).copy()
    st.kc = [to_np(t).copy() for t in v["k_cache"]]
    st.vc = [to_np(t).copy() for t in v["v_cache"]]
    st.conf_c = to_np(v["conf_cache"]).astype(np.float32).copy()
    st.tok_c = to_np(v["tok_cache"]).copy()
    before = st.copy()
    info = O.sparse_step(w, dims, run, st, P, P + 32, 2, region=(P, L))
    ctx.denoise_step_region(tg, mg, P, L, P, P + 32, 2, force_dense=False)
    ctx.sync_check()
    after_k = [to_np(t) for t in v["k_cache"]]
    for b in range(B):
        assert np.array_equal(to_np(v["h_cache"])[b][:P], before.hc[b][:P])
        assert np.array_equal(to_np(v["conf_cache"])[b][:P], before.conf_c[b][:P])
        for i in range(dims.n_layers):
            assert np.array_equal(after_k[i][b][:P], before.kc[i][b][:P]), i
            assert np.array_equal(to_np(v["v_cache"][i])[b][:P], before.vc[i][b][:P]), i
        # layer 0 recomputed the whole response (its tokens changed by the remask)
        assert not np.array_equal(after_k[0][b][P:], before.kc[0][b][P:])
    # teacher-forced against the oracle (same state after the full step): the
    # layers below the skip point recompute every response row, whatever the
    # selection, so their K/V rows of the response compare element by element
    for i in range(run.skip_layer):
        assert_parity(after_k[i][:, P:], st.kc[i][:, P:], "bf16", f"response K layer {i}")
        assert_parity(to_np(v["v_cache"][i])[:, P:], st.vc[i][:, P:], "bf16", f"response V layer {i}")
    assert len(info["idx"][0]) == O.keep_count(run.keep_ratio, G)
    ctx.close()


def test_second_point_keeping_every_row_is_the_single_point_step():
    """bf16: the same dense and sparse step on two contexts, one with a single
    skip point at 1, one with a second point at 3 that keeps every row; every
    cache the two share is bit-identical afterwards."""
    dims = synth.SMALL_BF16
    one = dataclasses.replace(synth.SMALL_BF16_RUN, skip_layer=1, keep_ratio=0.5)
    two = dataclasses.replace(one, skip_layer2=3, keep_ratio2=1.0)
    B, P, G = 2, 64, 64
    L = P + G
    ca, _ = make_context(dims, one, B, L)
    cb, _ = make_context(dims, two, B, L)
    prompt = synth.prompt_ids(dims, B, P)
    tok = np.full((B, L), dims.mask_id, dtype=np.int32)
    tok[:, :P] = prompt
    masked = np.zeros((B, L), dtype=np.uint8)
    masked[:, P:] = 1
    outs = []
    for ctx in (ca, cb):
        tg, mg = to_gpu(tok, torch.int32), to_gpu(masked, torch.uint8)
        ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=True)
        ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=False)
        ctx.sync_check()
        v = ctx.state(B, L)
        outs.append({"tok": to_np(tg), "masked": to_np(mg), "h": to_np(v["h_cache"]),
                     "conf": to_np(v["conf_cache"]), "pred": to_np(v["tok_cache"]),
                     "k": [to_np(t) for t in v["k_cache"]], "v": [to_np(t) for t in v["v_cache"]]})
    a, b = outs
    for f in ("tok", "masked", "h", "conf", "pred"):
        assert np.array_equal(a[f], b[f]), f
    for i in range(len(a["k"])):
        assert np.array_equal(a["k"][i], b["k"][i]) and np.array_equal(a["v"][i], b["v"][i]), i
    ca.close()
    cb.close()


def test_second_skip_point_arguments():
    import token_skipping_sparse_step_b200 as esd
    dims = synth.SMALL_BF16
    for skip2, keep2 in ((1, 0.5), (dims.n_layers, 0.5), (3, 0.0), (3, 1.5)):
        run = dataclasses.replace(synth.SMALL_BF16_RUN, skip_layer=1, skip_layer2=skip2, keep_ratio2=keep2)
        with pytest.raises(esd.EsdError):
            make_context(dims, run, 1, 64)
