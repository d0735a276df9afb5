"""Shared test utilities: build a GPU context and the oracle's weights from the
same seeded float32 draws, convert between torch and the oracle's float64
arrays, and the tolerance rule of the parity tests."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import synth


def torch_dtype(dims):
    return torch.bfloat16 if dims.dtype == "bf16" else torch.float32


def gpu_weights(dims, w32: dict) -> dict:
    dt = torch_dtype(dims)
    cv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dt).contiguous()
    return {"embed": cv(w32["embed"]), "w_out": cv(w32["w_out"]),
            "layers": [{k: cv(v) for k, v in lw.items()} for lw in w32["layers"]]}


def make_context(dims, run, max_batch, max_len, w32=None):
    import token_skipping_sparse_step_b200 as esd
    if w32 is None:
        w32 = synth.model_weights_f32(dims)
    tw = gpu_weights(dims, w32)
    ed = esd.make_dims(dims.n_layers, dims.d, dims.n_heads, dims.head_dim, dims.ffn, dims.vocab,
                       dims.mask_id, dims.rope_theta, dims.rms_eps, dims.dtype)
    er = esd.make_run(run.score_mode, run.alpha, run.lam, run.skip_layer, run.keep_ratio,
                      run.refresh_interval, max_batch, max_len, run.skip_layer2, run.keep_ratio2,
                      run.score_tensor, run.scope)
    ctx = esd.Context(ed, tw, er)
    return ctx, O.prepare_weights(w32, dims)


def to_gpu(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).to("cuda").contiguous()


def to_np(t) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy() if t.dtype.is_floating_point \
        else t.detach().cpu().numpy()


TOL = {"f32": 1e-4, "bf16": 2e-2}


def parity_error(g: np.ndarray, o: np.ndarray) -> float:
    """Max-abs error relative to the reference's largest magnitude:
    max |g - o| / max |o| (the normwise half of the parity rule)."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if not o.size:
        return 0.0
    return float(np.max(np.abs(g - o)) / max(np.max(np.abs(o)), 1e-30))


def c14_error(g: np.ndarray, o: np.ndarray, terms=None) -> float:
    """The element-wise half of the parity rule: max over elements of
    |g - o| / max(1, |o|), i.e. absolute error where |o| <= 1 and relative
    error above. A tensor passes at tolerance tol iff this is <= tol.

    ``terms``: for a bf16 residual-stream output o = bf16(x + act Wd^T), the
    oracle's per-element 2-norm of the terms of that last sum,
    sqrt(x^2 + sum_j (act_j Wd_ij)^2). Its stored operands carry bf16 rounding
    (a relative 2^-9 each) that moves the sum by an amount proportional to
    this norm, not to |o|; the denominator is then max(1, |o|, norm).
    """
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if not o.size:
        return 0.0
    den = np.maximum(1.0, np.abs(o))
    if terms is not None:
        den = np.maximum(den, np.asarray(terms, dtype=np.float64).reshape(o.shape))
    return float(np.max(np.abs(g - o) / den))


def elementwise_error(g: np.ndarray, o: np.ndarray) -> float:
    """Diagnostic: max |g - o| / (|o| + rms(o)), the per-element relative error
    floored at the tensor's RMS (reported, not asserted)."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    scale = np.sqrt(np.mean(o * o)) if o.size else 1.0
    return float(np.max(np.abs(g - o) / (np.abs(o) + scale))) if o.size else 0.0


def parity_ok(g, o, dtype: str, terms=None) -> tuple:
    """Both halves of the parity rule at the tolerance of ``dtype``:
    normwise max|g - o| / max|o| <= tol, and element-wise
    |g - o| <= tol * max(1, |o|) for every element (c14_error; ``terms`` for
    residual-stream outputs)."""
    n, e = parity_error(g, o), c14_error(g, o, terms)
    return (n <= TOL[dtype] and e <= TOL[dtype]), n, e


def assert_parity(g, o, dtype: str, what: str = "", terms=None):
    ok, n, e = parity_ok(g, o, dtype, terms)
    assert ok, (f"{what}: normwise {n:.3e}, element-wise {e:.3e} (limit {TOL[dtype]}; "
                f"RMS-floored {elementwise_error(g, o):.3e})")
    return n


def near_tie_ok(g_tok, o_tok, margins, thresh):
    """Token decisions match except where the oracle's top-2 margin is below
    ``thresh`` (a near-tie: both answers are correct up to rounding)."""
    bad = (np.asarray(g_tok) != np.asarray(o_tok)) & (np.asarray(margins) >= thresh)
    return not bad.any(), int((np.asarray(g_tok) != np.asarray(o_tok)).sum())
