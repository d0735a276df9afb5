"""The allocation-free head (esd_confidence_argmax_noalloc) against the context
head (esd_confidence_argmax), through the C ABI.

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
from helpers import TOL, make_context, parity_error, to_gpu, to_np

pytestmark = pytest.mark.gpu


def _inputs(dims, rows, seed):
    rng = np.random.default_rng(seed)
    return to_gpu(O.store(rng.standard_normal((rows, dims.d)) * 0.3, dims.dtype), torch.bfloat16)


def test_noalloc_head_matches_context_head_twice():
    import token_skipping_sparse_step_b200 as esd

    dims, run = synth.SMALL_BF16, synth.SMALL_BF16_RUN
    B, L, k = 2, 160, 40
    ctx, _ = make_context(dims, run, B, L)
    w_out = ctx._keep["w_out"]
    idx = np.stack([np.sort(np.random.default_rng(b).choice(L, k, replace=False)) for b in range(B)])
    ig = to_gpu(idx.astype(np.int32), torch.int32)
    for call, seed in enumerate((1, 2)):  # two calls in a row, different inputs
        x = _inputs(dims, B * k, seed)
        # rows written in place (idx = NULL)
        c_ref = torch.full((B * k,), -1.0, device="cuda")
        t_ref = torch.full((B * k,), -1, dtype=torch.int32, device="cuda")
        ctx.confidence_argmax(x, None, 1, B * k, B * k, c_ref, t_ref)
        c_new = torch.full((B * k,), -1.0, device="cuda")
        t_new = torch.full((B * k,), -1, dtype=torch.int32, device="cuda")
        esd.confidence_argmax_noalloc(x, B * k, w_out, dims.d, dims.vocab, dims.mask_id,
                                      dims.rms_eps, None, 0, 0, c_new, t_new)
        # scattered through idx into [B*L] caches
        cc_ref = torch.zeros(B * L, device="cuda")
        tc_ref = torch.zeros(B * L, dtype=torch.int32, device="cuda")
        ctx.confidence_argmax(x, ig, B, L, k, cc_ref, tc_ref)
        cc_new = torch.zeros(B * L, device="cuda")
        tc_new = torch.zeros(B * L, dtype=torch.int32, device="cuda")
        esd.confidence_argmax_noalloc(x, B * k, w_out, dims.d, dims.vocab, dims.mask_id,
                                      dims.rms_eps, ig, L, k, cc_new, tc_new)
        torch.cuda.synchronize()
        ctx.sync_check()
        assert parity_error(to_np(c_new), to_np(c_ref)) <= TOL["bf16"], call
        assert torch.equal(t_new, t_ref), call
        assert parity_error(to_np(cc_new), to_np(cc_ref)) <= TOL["bf16"], call
        assert torch.equal(tc_new, tc_ref), call
    ctx.close()


def test_noalloc_head_rejects_requests_beyond_its_scratch():
    import token_skipping_sparse_step_b200 as esd

    dims = synth.SMALL_BF16
    x = torch.zeros((8, dims.d), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((dims.vocab, dims.d), dtype=torch.bfloat16, device="cuda")
    conf = torch.zeros(8, device="cuda")
    tok = torch.zeros(8, dtype=torch.int32, device="cuda")
    per_row = 4 + 12 * ((dims.vocab + 127) // 128)
    too_many = esd.NOALLOC_SCRATCH_BYTES // per_row + 1
    with pytest.raises(esd.EsdError) as e:
        esd.confidence_argmax_noalloc(x, too_many, w, dims.d, dims.vocab, dims.mask_id,
                                      dims.rms_eps, None, 0, 0, conf, tok)
    assert e.value.status == 1  # ESD_ERR_INVALID_ARG, before any device work
