"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module draws random numbers and lays them out; it holds none of the
early-skipping method's arithmetic. Both the CPU oracle and the CUDA path take
their inputs from here, so that the two sides see bit-identical weights,
prompts and hidden states.

Generator (counter based, so any element can be drawn on its own):

* ``splitmix64``: the i-th raw 64-bit draw of stream ``seed`` is
  ``mix(seed + (i + 1) * 0x9E3779B97F4A7C15 mod 2**64)`` with Steele, Lea and
  Flood's finaliser ``mix`` (SplitMix64, OOPSLA 2014).
* Uniforms take the top 53 bits: ``u = (r >> 11) * 2**-53`` in [0, 1).
* Normal number j uses raw draws 2j and 2j+1 and the cosine branch of the
  Box-Muller transform in float64:
  ``z = sqrt(-2 ln(1 - u_a)) * cos(2 pi u_b)``.
* Model weights are ``float32(0.02 * z)``; the bf16 models round that float32
  to bf16 (round to nearest even). The weight stream is one stream of seed 0,
  drawn in the order E, then per layer Wq, Wk, Wv, Wo, Wg, Wu, Wd, then W_out,
  every matrix stored [out, in] row-major.
* Prompt ids (seed 1): raw draw mod (V - 1), then ids >= mask_id shift up by one,
  so the mask id is never drawn.
* Microbenchmark tensors (seed 2): x ~ N(0, 1); the cached state is
  x + N(0, 0.01^2) on rows kept by a Bernoulli(0.9) draw and an independent
  N(0, 1) row otherwise; confidences are Beta(5, 1) = U^(1/5).

The same definitions are implemented in CUDA in ``synth/csrc/synth.cu`` for the
models too large to draw on the host.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

SEED_WEIGHTS = 0
SEED_PROMPT = 1
SEED_MICRO = 2

_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def raw_u64(seed: int, start: int, n: int) -> np.ndarray:
    """Raw draws ``start .. start+n-1`` of stream ``seed`` (uint64)."""
    with np.errstate(over="ignore"):
        ctr = np.arange(start + 1, start + 1 + n, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + ctr * GOLDEN
        return _mix(z)


def raw_u64_at(seed: int, counters: np.ndarray) -> np.ndarray:
    """Raw draws at arbitrary (0-based) counters."""
    with np.errstate(over="ignore"):
        ctr = np.asarray(counters, dtype=np.uint64) + np.uint64(1)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + ctr * GOLDEN
        return _mix(z)


def _u53(r: np.ndarray) -> np.ndarray:
    return (r >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_at(seed: int, j: np.ndarray) -> np.ndarray:
    """Standard normals number ``j`` (array of normal indices) of stream ``seed``."""
    j = np.asarray(j, dtype=np.uint64)
    ua = _u53(raw_u64_at(seed, j * np.uint64(2)))
    ub = _u53(raw_u64_at(seed, j * np.uint64(2) + np.uint64(1)))
    return np.sqrt(-2.0 * np.log1p(-ua)) * np.cos(2.0 * math.pi * ub)


def normal(seed: int, start: int, n: int) -> np.ndarray:
    """``n`` consecutive standard normals from normal index ``start`` (float64)."""
    out = np.empty(n, dtype=np.float64)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        out[c0:c1] = normal_at(seed, np.arange(start + c0, start + c1, dtype=np.uint64))
    return out


def uniform(seed: int, start: int, n: int) -> np.ndarray:
    return _u53(raw_u64(seed, start, n))


# --------------------------------------------------------------------------
# model shapes and the weight stream
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class ModelDims:
    n_layers: int
    d: int
    n_heads: int
    head_dim: int
    ffn: int
    vocab: int
    mask_id: int
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    dtype: str = "f32"  # storage type: "f32" or "bf16"


@dataclasses.dataclass(frozen=True)
class RunConfig:
    score_mode: str = "es"      # "es" or "cos"
    alpha: float = 0.5          # ES weight of the confidence term
    lam: float = 0.5            # COS weight of (1 - confidence)
    skip_layer: int = 1
    keep_ratio: float = 0.25
    refresh_interval: int = 0   # 0: refresh only at the first step of each block
    skip_layer2: int = 0        # second skip point (0: none); skip_layer < skip_layer2 < n_layers
    keep_ratio2: float = 1.0    # of the rows that reach the second skip point
    score_tensor: str = "h"     # the score's variation on "h" (skip-layer input), "k" or "v" (of the skip layer)
    scope: str = "all"          # selection set S: "all" positions, the current "block", or the
                                # "response" (every position after the prompt); with "block" and
                                # "response" every layer recomputes only that region's rows and the
                                # other rows use cached K/V


LAYER_MATS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")


def layer_shapes(dims: ModelDims) -> dict:
    d, f = dims.d, dims.ffn
    return {"wq": (d, d), "wk": (d, d), "wv": (d, d), "wo": (d, d),
            "wg": (f, d), "wu": (f, d), "wd": (d, f)}


def weight_layout(dims: ModelDims):
    """[(name, layer or None, shape, normal offset)] in stream order."""
    out = []
    off = 0
    out.append(("embed", None, (dims.vocab, dims.d), off))
    off += dims.vocab * dims.d
    shapes = layer_shapes(dims)
    for layer in range(dims.n_layers):
        for name in LAYER_MATS:
            shp = shapes[name]
            out.append((name, layer, shp, off))
            off += shp[0] * shp[1]
    out.append(("w_out", None, (dims.vocab, dims.d), off))
    off += dims.vocab * dims.d
    return out


WEIGHT_STD = 0.02


def weight_f32(seed: int, offset: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return (WEIGHT_STD * normal(seed, offset, n)).astype(np.float32).reshape(shape)


def weight_rows_f32(seed: int, offset: int, shape, rows) -> np.ndarray:
    """Selected rows of one weight matrix, drawn without drawing the rest."""
    rows = np.asarray(rows, dtype=np.int64)
    cols = shape[1]
    j = (np.uint64(offset) + rows.astype(np.uint64)[:, None] * np.uint64(cols)
         + np.arange(cols, dtype=np.uint64)[None, :])
    return (WEIGHT_STD * normal_at(seed, j.reshape(-1))).astype(np.float32).reshape(len(rows), cols)


def model_weights_f32(dims: ModelDims, seed: int = SEED_WEIGHTS) -> dict:
    """All weights as float32 arrays: {"embed", "w_out", "layers": [{wq..wd}]}."""
    w = {"layers": [dict() for _ in range(dims.n_layers)]}
    for name, layer, shape, off in weight_layout(dims):
        arr = weight_f32(seed, off, shape)
        if layer is None:
            w[name] = arr
        else:
            w["layers"][layer][name] = arr
    return w


def prompt_ids(dims: ModelDims, batch: int, length: int, seed: int = SEED_PROMPT) -> np.ndarray:
    r = raw_u64(seed, 0, batch * length)
    ids = (r % np.uint64(dims.vocab - 1)).astype(np.int64)
    ids = ids + (ids >= dims.mask_id)
    return ids.astype(np.int32).reshape(batch, length)


# --------------------------------------------------------------------------
# microbenchmark tensors
# --------------------------------------------------------------------------
def micro_inputs(batch: int, seq: int, d: int, seed: int = SEED_MICRO,
                 changed_frac: float = 0.1):
    """x [B,S,d], h_cache [B,S,d] (float32) and conf [B,S] (float32)."""
    n = batch * seq * d
    x = normal(seed, 0, n).reshape(batch, seq, d)
    noise = normal(seed, n, n).reshape(batch, seq, d)
    fresh = normal(seed, 2 * n, n).reshape(batch, seq, d)
    changed = uniform(seed + 1, 0, batch * seq).reshape(batch, seq) < changed_frac
    hc = np.where(changed[..., None], fresh, x + 0.01 * noise)
    conf = uniform(seed + 2, 0, batch * seq).reshape(batch, seq) ** 0.2
    return x.astype(np.float32), hc.astype(np.float32), conf.astype(np.float32)


def micro_rows(batch: int, seq: int, d: int, rows, seed: int = SEED_MICRO,
               changed_frac: float = 0.1):
    """Rows (flat indices b*seq + i) of micro_inputs, drawn without the rest."""
    rows = np.asarray(rows, dtype=np.int64)
    n = batch * seq * d
    j = (rows.astype(np.uint64)[:, None] * np.uint64(d) + np.arange(d, dtype=np.uint64)[None, :])
    x = normal_at(seed, j)
    noise = normal_at(seed, j + np.uint64(n))
    fresh = normal_at(seed, j + np.uint64(2 * n))
    changed = _u53(raw_u64_at(seed + 1, rows.astype(np.uint64))) < changed_frac
    hc = np.where(changed[:, None], fresh, x + 0.01 * noise)
    conf = _u53(raw_u64_at(seed + 2, rows.astype(np.uint64))) ** 0.2
    return x.astype(np.float32), hc.astype(np.float32), conf.astype(np.float32)


# --------------------------------------------------------------------------
# the workloads
# --------------------------------------------------------------------------
TINY = ModelDims(n_layers=2, d=256, n_heads=4, head_dim=64, ffn=688, vocab=1024,
                 mask_id=1023, rope_theta=10000.0, dtype="f32")
TINY_RUN = RunConfig(score_mode="cos", lam=0.5, skip_layer=1, keep_ratio=0.25)
TINY_SEQ = dict(batch=1, prompt=64, gen=64, block=32, n_unmask=4)

M1B = ModelDims(n_layers=16, d=2048, n_heads=16, head_dim=128, ffn=5632, vocab=32000,
                mask_id=31999, rope_theta=10000.0, dtype="bf16")
M1B_RUN = RunConfig(score_mode="es", alpha=0.5, skip_layer=4, keep_ratio=0.20)
M1B_SEQ = dict(batch=1, prompt=256, gen=256, block=32, n_unmask=1)

M8B = ModelDims(n_layers=32, d=4096, n_heads=32, head_dim=128, ffn=12288, vocab=126464,
                mask_id=126336, rope_theta=500000.0, dtype="bf16")
M8B_RUN = RunConfig(score_mode="es", alpha=0.5, skip_layer=4, keep_ratio=0.25)
M8B_SEQ = dict(batch=1, prompt=512, gen=256, block=32, n_unmask=1)
M8B32_SEQ = dict(batch=32, prompt=1024, gen=512, block=64, n_unmask=2)

# a small bf16 model with the 1B/8B head geometry (head_dim 128), used for
# whole-step bf16 parity where the full models are too slow for the oracle
SMALL_BF16 = ModelDims(n_layers=4, d=512, n_heads=4, head_dim=128, ffn=1408, vocab=4096,
                       mask_id=4095, rope_theta=10000.0, dtype="bf16")
SMALL_BF16_RUN = RunConfig(score_mode="es", alpha=0.5, skip_layer=2, keep_ratio=0.25)
SMALL_BF16_SEQ = dict(batch=2, prompt=96, gen=64, block=32, n_unmask=2)

MICRO = dict(batch=16, seq=4096, d=4096, n_heads=32, head_dim=128, ks=(64, 256, 1024))

