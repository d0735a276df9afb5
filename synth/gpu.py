"""GPU twin of the seeded generator (``synth/csrc/synth.cu``) for tensors too
large to draw on the host. Bit-identical to ``synth`` up to the rare float64
last-place difference of the device's log1p/cos, which vanishes after the
rounding to float32/bf16 except with probability ~1e-13 per bf16 element."""
from __future__ import annotations

import ctypes
import os

import torch

from . import SEED_MICRO, SEED_WEIGHTS, WEIGHT_STD, ModelDims, uniform, weight_layout

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} missing: run python token_skipping_sparse_step_b200/build.py")
        _lib = ctypes.CDLL(LIB_PATH)
        _lib.synth_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                           ctypes.c_uint64, ctypes.c_double, ctypes.c_double,
                                           ctypes.c_int, ctypes.c_void_p]
        _lib.synth_fill_normal.restype = ctypes.c_int
        _lib.synth_fill_micro.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
                                          ctypes.c_int, ctypes.c_void_p]
        _lib.synth_fill_micro.restype = ctypes.c_int
    return _lib


def fill_normal(t: torch.Tensor, seed: int, start: int, scale: float = 1.0, shift: float = 0.0):
    """t (contiguous float32 or bf16 CUDA tensor) <- shift + scale * normal(start + i)."""
    assert t.is_cuda and t.is_contiguous() and t.dtype in (torch.float32, torch.bfloat16)
    st = torch.cuda.current_stream().cuda_stream
    rc = _load().synth_fill_normal(t.data_ptr(), t.numel(), seed, start, scale, shift,
                                   int(t.dtype == torch.bfloat16), st)
    if rc != 0:
        raise RuntimeError(f"synth_fill_normal failed ({rc})")
    return t


def model_weights(dims: ModelDims, seed: int = SEED_WEIGHTS) -> dict:
    """All model weights drawn on the current CUDA device in the storage type."""
    dt = torch.bfloat16 if dims.dtype == "bf16" else torch.float32
    w = {"layers": [dict() for _ in range(dims.n_layers)]}
    for name, layer, shape, off in weight_layout(dims):
        t = torch.empty(shape, dtype=dt, device="cuda")
        fill_normal(t, seed, off, WEIGHT_STD)
        if layer is None:
            w[name] = t
        else:
            w["layers"][layer][name] = t
    return w


def micro_inputs(batch: int, seq: int, d: int, seed: int = SEED_MICRO, dtype=torch.bfloat16,
                 changed_frac: float = 0.1):
    """synth.micro_inputs drawn on the device: x, h_cache [B*S, d] in `dtype`,
    conf [B*S] float32 (the confidences are drawn on the host: B*S values)."""
    rows = batch * seq
    x = torch.empty((rows, d), dtype=dtype, device="cuda")
    h = torch.empty((rows, d), dtype=dtype, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    rc = _load().synth_fill_micro(x.data_ptr(), h.data_ptr(), rows, d, seed, changed_frac,
                                  int(dtype == torch.bfloat16), st)
    if rc != 0:
        raise RuntimeError(f"synth_fill_micro failed ({rc})")
    conf = torch.from_numpy((uniform(seed + 2, 0, rows) ** 0.2).astype("float32")).to("cuda")
    return x, h, conf
