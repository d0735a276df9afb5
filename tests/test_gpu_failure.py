"""Failure detection without a GPU fault: a bounded device wait that expires
(a barrier phase that nothing completes) records ESD_ERR_TIMEOUT on the
context's flag, the host reads it from esd_sync_check, and the context keeps
working afterwards."""
import numpy as np
import pytest
import torch

import synth
from helpers import make_context, to_gpu

pytestmark = pytest.mark.gpu


def test_expired_device_wait_reports_timeout_and_context_stays_usable():
    import token_skipping_sparse_step_b200 as esd
    dims, run = synth.SMALL_BF16, synth.SMALL_BF16_RUN
    ctx, _ = make_context(dims, run, 1, 128)
    ctx.selftest_wait_timeout(1 << 16)
    with pytest.raises(esd.EsdError) as err:
        ctx.sync_check()
    assert err.value.status == 5  # ESD_ERR_TIMEOUT
    ctx.sync_check()  # the flag was cleared by the report
    P, G = 96, 32
    tok = np.full((1, P + G), dims.mask_id, dtype=np.int32)
    tok[:, :P] = synth.prompt_ids(dims, 1, P)
    masked = np.zeros((1, P + G), dtype=np.uint8)
    masked[:, P:] = 1
    tg, mg = to_gpu(tok, torch.int32), to_gpu(masked, torch.uint8)
    ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=True)
    ctx.denoise_step(tg, mg, P, P + 32, 2, force_dense=False)
    ctx.sync_check()
    assert int((tg[:, P:] != dims.mask_id).sum()) == 4
    with pytest.raises(esd.EsdError):
        ctx.selftest_wait_timeout(0)
    ctx.close()
