"""The allocation-free head (esd_confidence_argmax_noalloc) through the C ABI:
against the context head (esd_confidence_argmax) and against the oracle's
head, on two calls in a row, with 128-row and 256-row tensor-core tiles.

The allocation-free call exists for callers that cannot allocate device memory
(a pool or allocator that must not be bypassed, a host that forbids cudaMalloc
after start-up, a fully reserved device): it takes its workspace from a fixed
array inside the library. Collected last on purpose: if it fails, a run that
stops at the first failure has already run every other test. It also passes
alone in a fresh process (its first call sets the device up).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import TOL, assert_parity, make_context, near_tie_ok, to_gpu, to_np

pytestmark = pytest.mark.gpu


def _inputs(dims, rows, seed):
    rng = np.random.default_rng(seed)
    x = O.store(rng.standard_normal((rows, dims.d)) * 0.3, dims.dtype)
    return x, to_gpu(x, torch.bfloat16)


@pytest.mark.parametrize("B,k", [(2, 40), (2, 150)])  # 80 rows: 128-row tiles; 300 rows: 256-row tiles
def test_noalloc_head_matches_context_head_and_oracle_twice(B, k):
    import token_skipping_sparse_step_b200 as esd

    dims, run = synth.SMALL_BF16, synth.SMALL_BF16_RUN
    L = 160
    ctx, w = make_context(dims, run, B, max(L, B * k))
    w_out = ctx._keep["w_out"]
    idx = np.stack([np.sort(np.random.default_rng(b).choice(L, k, replace=False)) for b in range(B)])
    ig = to_gpu(idx.astype(np.int32), torch.int32)
    for call, seed in enumerate((1, 2)):  # two calls in a row, different inputs
        xo, x = _inputs(dims, B * k, seed)
        # rows written in place (idx = NULL)
        c_ref = torch.full((B * k,), -1.0, device="cuda")
        t_ref = torch.full((B * k,), -1, dtype=torch.int32, device="cuda")
        ctx.confidence_argmax(x, None, 1, B * k, B * k, c_ref, t_ref)
        c_new = torch.full((B * k,), -1.0, device="cuda")
        t_new = torch.full((B * k,), -1, dtype=torch.int32, device="cuda")
        esd.confidence_argmax_noalloc(x, B * k, w_out, dims.d, dims.vocab, dims.mask_id,
                                      dims.rms_eps, None, 0, 0, c_new, t_new)
        esd.noalloc_check()
        # scattered through idx into [B*L] caches
        cc_ref = torch.zeros(B * L, device="cuda")
        tc_ref = torch.zeros(B * L, dtype=torch.int32, device="cuda")
        ctx.confidence_argmax(x, ig, B, L, k, cc_ref, tc_ref)
        cc_new = torch.zeros(B * L, device="cuda")
        tc_new = torch.zeros(B * L, dtype=torch.int32, device="cuda")
        esd.confidence_argmax_noalloc(x, B * k, w_out, dims.d, dims.vocab, dims.mask_id,
                                      dims.rms_eps, ig, L, k, cc_new, tc_new)
        esd.noalloc_check()
        ctx.sync_check()
        # the same kernels on the same inputs as the context head
        assert torch.equal(c_new, c_ref) and torch.equal(t_new, t_ref), call
        assert torch.equal(cc_new, cc_ref) and torch.equal(tc_new, tc_ref), call
        # and the oracle's head: confidence within the bf16 tolerance, argmax
        # equal outside near-ties
        oc, ot, om = O.head(xo, w["w_out"], dims)
        assert_parity(to_np(c_new), oc, "bf16", f"noalloc confidence, call {call}")
        ok, nbad = near_tie_ok(to_np(t_new), ot, om, 2 * TOL["bf16"] * O.logit_scale(xo, w["w_out"], dims))
        assert ok, f"{nbad} argmax mismatches outside near-ties, call {call}"
        scat = np.zeros(B * L)
        scat[(np.arange(B)[:, None] * L + idx).reshape(-1)] = 1
        assert np.all(to_np(tc_new)[scat == 0] == 0)
    ctx.close()


def test_noalloc_head_reports_an_expired_wait_then_recovers():
    """A bounded wait on the allocation-free head's status word runs out (no
    fault); esd_noalloc_check reports ESD_ERR_TIMEOUT; the next head call
    clears the word and its results are valid again."""
    import token_skipping_sparse_step_b200 as esd

    dims = synth.SMALL_BF16
    esd.noalloc_selftest_wait_timeout(1 << 12)
    with pytest.raises(esd.EsdError) as e:
        esd.noalloc_check()
    assert e.value.status == esd.ESD_ERR_TIMEOUT
    w32 = synth.model_weights_f32(dims)
    w_out = to_gpu(w32["w_out"], torch.bfloat16)
    xo, x = _inputs(dims, 64, 7)
    conf = torch.zeros(64, device="cuda")
    tok = torch.zeros(64, dtype=torch.int32, device="cuda")
    esd.confidence_argmax_noalloc(x, 64, w_out, dims.d, dims.vocab, dims.mask_id, dims.rms_eps,
                                  None, 0, 0, conf, tok)
    esd.noalloc_check()
    oc, _, _ = O.head(xo, O.store(w32["w_out"].astype(np.float64), "bf16"), dims)
    assert_parity(to_np(conf), oc, "bf16", "confidence after recovery")


def test_noalloc_head_rejects_requests_beyond_its_scratch():
    import token_skipping_sparse_step_b200 as esd

    dims = synth.SMALL_BF16
    x = torch.zeros((8, dims.d), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((dims.vocab, dims.d), dtype=torch.bfloat16, device="cuda")
    conf = torch.zeros(8, device="cuda")
    tok = torch.zeros(8, dtype=torch.int32, device="cuda")
    tiles = (dims.vocab + 127) // 128

    def need(rows):
        return 256 + (4 * rows + 255) // 256 * 256 + 12 * rows * tiles

    rows = esd.NOALLOC_SCRATCH_BYTES // (4 + 12 * tiles)
    while need(rows) > esd.NOALLOC_SCRATCH_BYTES:
        rows -= 1
    too_many = rows + 1
    with pytest.raises(esd.EsdError) as e:
        esd.confidence_argmax_noalloc(x, too_many, w, dims.d, dims.vocab, dims.mask_id,
                                      dims.rms_eps, None, 0, 0, conf, tok)
    assert e.value.status == 1  # ESD_ERR_INVALID_ARG, before any device work
