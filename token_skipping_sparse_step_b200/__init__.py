"""Python binding of ``libesd.so``, the early-skipping sparse denoising step for
masked-diffusion transformers on NVIDIA B200 (sm_100a).

Argument marshalling only: every step of the method runs in the library's CUDA
kernels. PyTorch provides device memory and streams. Names follow the C ABI in
``include/esd.h`` without the ``esd_`` prefix. There is no CPU fallback: if the
library is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libesd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python token_skipping_sparse_step_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

ESD_OK = 0
ESD_ERR_INVALID_ARG, ESD_ERR_CUDA, ESD_ERR_OOM, ESD_ERR_UNSUPPORTED, ESD_ERR_TIMEOUT, ESD_ERR_CHECK = 1, 2, 3, 4, 5, 6
STATUS_NAMES = {0: "ESD_OK", 1: "ESD_ERR_INVALID_ARG", 2: "ESD_ERR_CUDA", 3: "ESD_ERR_OOM",
                4: "ESD_ERR_UNSUPPORTED", 5: "ESD_ERR_TIMEOUT", 6: "ESD_ERR_CHECK"}
DTYPE_F32, DTYPE_BF16 = 0, 1
SCORE_ES, SCORE_COS = 0, 1

# every symbol include/esd.h declares
EXPORTS = ("esd_create", "esd_destroy", "esd_last_error", "esd_keep_count", "esd_state",
           "esd_embed", "esd_importance_select", "esd_topk_select", "esd_gather_rows",
           "esd_sparse_layers_forward", "esd_confidence_argmax", "esd_logits", "esd_remask",
           "esd_denoise_step", "esd_denoise_step_region", "esd_generate", "esd_sync_check", "esd_launch_count",
           "esd_profile_enable", "esd_profile_read", "esd_confidence_argmax_noalloc",
           "esd_partial_attention", "esd_context_saliency", "esd_dyllm_layers_forward",
           "esd_dyllm_layers_forward_approx",
           "esd_selftest_wait_timeout", "esd_approx_attention", "esd_noalloc_check",
           "esd_noalloc_selftest_wait_timeout")
K_GEMM_QKV, K_GEMM_O, K_GEMM_GATE_UP, K_GEMM_DOWN, K_HEAD, K_ATTENTION, K_SCORE_SELECT = 0, 1, 2, 3, 4, 6, 7


class ModelDims(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int), ("vocab", ctypes.c_int),
                ("mask_id", ctypes.c_int), ("rope_theta", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("dtype", ctypes.c_int)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class Weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("w_out", ctypes.c_void_p), ("wq", _PP), ("wk", _PP),
                ("wv", _PP), ("wo", _PP), ("wg", _PP), ("wu", _PP), ("wd", _PP)]


class RunConfig(ctypes.Structure):
    _fields_ = [("score_mode", ctypes.c_int), ("alpha", ctypes.c_float), ("lambda_", ctypes.c_float),
                ("skip_layer", ctypes.c_int), ("keep_ratio", ctypes.c_float),
                ("refresh_interval", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_len", ctypes.c_int), ("skip_layer2", ctypes.c_int),
                ("keep_ratio2", ctypes.c_float), ("score_tensor", ctypes.c_int), ("scope", ctypes.c_int)]


class StateView(ctypes.Structure):
    _fields_ = [("h_cache", ctypes.c_void_p), ("k_cache", _PP), ("v_cache", _PP),
                ("conf_cache", ctypes.c_void_p), ("tok_cache", ctypes.c_void_p),
                ("n_cached_layers", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_len", ctypes.c_int)]


_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_sigs = {
    "esd_create": [ctypes.POINTER(ModelDims), ctypes.POINTER(Weights), ctypes.POINTER(RunConfig),
                   ctypes.POINTER(_vp)],
    "esd_destroy": [_vp],
    "esd_keep_count": [_vp, _i],
    "esd_state": [_vp, ctypes.POINTER(StateView)],
    "esd_embed": [_vp, _vp, _i, _i, _vp, _vp],
    "esd_importance_select": [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp],
    "esd_topk_select": [_vp, _vp, _i, _i, _i, _vp, _vp],
    "esd_context_saliency": [_vp, _vp, _vp, _i, _i, _f, _vp, _vp, _vp, _vp],
    "esd_dyllm_layers_forward": [_vp, _i, _i, _vp, _i, _i, _vp, _i, _vp, _vp, _vp],
    "esd_dyllm_layers_forward_approx": [_vp, _i, _i, _vp, _i, _i, _vp, _i, _vp, _vp, _vp],
    "esd_approx_attention": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _vp, _vp],
    "esd_gather_rows": [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp],
    "esd_sparse_layers_forward": [_vp, _i, _i, _vp, _i, _i, _i, _vp, _vp],
    "esd_confidence_argmax": [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp],
    "esd_partial_attention": [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp],
    "esd_logits": [_vp, _vp, _i, _vp, _vp],
    "esd_remask": [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp],
    "esd_denoise_step": [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp],
    "esd_denoise_step_region": [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp],
    "esd_generate": [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp],
    "esd_sync_check": [_vp, _vp],
    "esd_selftest_wait_timeout": [_vp, ctypes.c_uint, _vp],
    "esd_profile_enable": [_vp, _i, _i, _i],
    "esd_profile_read": [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64), _i],
    "esd_confidence_argmax_noalloc": [_vp, _i, _vp, _i, _i, _i, _f, _vp, _i, _i, _vp, _vp, _vp],
    "esd_noalloc_check": [_vp],
    "esd_noalloc_selftest_wait_timeout": [ctypes.c_uint, _vp],
}
for _name, _args in _sigs.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int
_lib.esd_last_error.argtypes = [_vp]
_lib.esd_last_error.restype = ctypes.c_char_p
_lib.esd_launch_count.argtypes = [_vp]
_lib.esd_launch_count.restype = ctypes.c_uint64


class EsdError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _storage_dtype(dims: ModelDims):
    return torch.bfloat16 if dims.dtype == DTYPE_BF16 else torch.float32


class _CudaView:
    """Exposes a device pointer owned by the library to torch (no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


_TYPESTR = {torch.float32: "<f4", torch.int32: "<i4"}


class Context:
    """An ``esd_ctx``: borrows the weight tensors for its lifetime."""

    def __init__(self, dims: ModelDims, weights: dict, run: RunConfig):
        self.dims, self.run = dims, run
        self._keep = weights  # keep the tensors alive
        n = dims.n_layers
        arr = lambda key: (ctypes.c_void_p * n)(*[w[key].data_ptr() for w in weights["layers"]])
        self._arrs = {k: arr(k) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd")}
        cast = lambda a: ctypes.cast(a, _PP)
        self._w = Weights(weights["embed"].data_ptr(), weights["w_out"].data_ptr(),
                          *[cast(self._arrs[k]) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd")])
        h = ctypes.c_void_p()
        st = _lib.esd_create(ctypes.byref(dims), ctypes.byref(self._w), ctypes.byref(run),
                             ctypes.byref(h))
        if st != ESD_OK:
            raise EsdError(st, "esd_create failed")
        self.handle = h

    # -- plumbing
    def _check(self, st: int):
        if st != ESD_OK:
            raise EsdError(st, _lib.esd_last_error(self.handle).decode())

    def close(self):
        if getattr(self, "handle", None):
            _lib.esd_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def storage_dtype(self):
        return _storage_dtype(self.dims)

    def keep_count(self, L: int) -> int:
        return _lib.esd_keep_count(self.handle, L)

    def launch_count(self) -> int:
        return int(_lib.esd_launch_count(self.handle))

    def state(self, B: int, L: int) -> dict:
        """Torch views of the context-owned caches for a (B, L) batch."""
        v = StateView()
        self._check(_lib.esd_state(self.handle, ctypes.byref(v)))
        d, H, hd = self.dims.d, self.dims.n_heads, self.dims.head_dim
        dt = self.storage_dtype
        esz = 2 if dt == torch.bfloat16 else 4

        def view(ptr, shape, dtype):
            if dtype == torch.bfloat16:
                t = torch.as_tensor(_CudaView(ptr, (int(torch.tensor(shape).prod()),), "<i2"),
                                    device="cuda")
                return t.view(torch.bfloat16).view(*shape)
            return torch.as_tensor(_CudaView(ptr, shape, _TYPESTR[dtype]), device="cuda")

        out = {"h_cache": view(v.h_cache, (B, L, d), dt),
               "k_cache": [view(v.k_cache[i], (B, L, H, hd), dt) for i in range(v.n_cached_layers)],
               "v_cache": [view(v.v_cache[i], (B, L, H, hd), dt) for i in range(v.n_cached_layers)],
               "conf_cache": view(v.conf_cache, (B, L), torch.float32),
               "tok_cache": view(v.tok_cache, (B, L), torch.int32)}
        del esz
        return out

    # -- the hot-path calls
    def embed(self, tok, x, stream=None):
        B, L = tok.shape
        self._check(_lib.esd_embed(self.handle, _ptr(tok), B, L, _ptr(x), _stream(stream)))

    def importance_select(self, x, h_cache, conf_prev, B, L, k, idx_out, scores_out=None,
                          stream=None):
        self._check(_lib.esd_importance_select(self.handle, _ptr(x), _ptr(h_cache),
                                               _ptr(conf_prev), B, L, k, _ptr(scores_out),
                                               _ptr(idx_out), _stream(stream)))

    def context_saliency(self, c_cur, c_prev, B, L, tau, idx_out, count_out, sim_out=None,
                         stream=None):
        """Rows whose attention context moved (cosine to the previous step's
        context below tau), per sequence, ascending; see esd_context_saliency."""
        self._check(_lib.esd_context_saliency(self.handle, _ptr(c_cur), _ptr(c_prev), B, L, float(tau),
                                              _ptr(sim_out), _ptr(idx_out), _ptr(count_out),
                                              _stream(stream)))

    def dyllm_layers_forward(self, layer_begin, layer_end, x, B, L, taus=None, refresh=False,
                             sim_out=None, stream=None, approx=False, counts_out=None):
        """DyLLM token-selection layers on x [B*L, d] in place; see
        esd_dyllm_layers_forward (approx: esd_dyllm_layers_forward_approx,
        contexts from the saliency-aware approximate attention). Returns the
        salient row counts [layers, B]: counts_out when given (a device int32
        tensor, filled asynchronously), else a numpy int32 array (the call
        then waits for the stream)."""
        n = layer_end - layer_begin
        counts = np.zeros((n, B), dtype=np.int32) if counts_out is None else counts_out
        tau = None
        if taus is not None:
            tau = np.ascontiguousarray(np.broadcast_to(np.asarray(taus, dtype=np.float32), (n,)))
        fn = _lib.esd_dyllm_layers_forward_approx if approx else _lib.esd_dyllm_layers_forward
        self._check(fn(
            self.handle, layer_begin, layer_end, _ptr(x), B, L,
            None if tau is None else tau.ctypes.data, int(refresh),
            counts.ctypes.data if counts_out is None else _ptr(counts_out),
            _ptr(sim_out), _stream(stream)))
        return counts

    def topk_select(self, scores, B, L, k, idx_out, stream=None):
        self._check(_lib.esd_topk_select(self.handle, _ptr(scores), B, L, k, _ptr(idx_out),
                                         _stream(stream)))

    def gather_rows(self, x, idx, B, L, k, x_sel, h_cache=None, stream=None):
        self._check(_lib.esd_gather_rows(self.handle, _ptr(x), _ptr(idx), B, L, k, _ptr(x_sel),
                                         _ptr(h_cache), _stream(stream)))

    def sparse_layers_forward(self, layer_begin, layer_end, idx, B, L, k, x_sel, stream=None):
        self._check(_lib.esd_sparse_layers_forward(self.handle, layer_begin, layer_end, _ptr(idx),
                                                   B, L, k, _ptr(x_sel), _stream(stream)))

    def approx_attention(self, q, k, v, v_prev, changed_idx, changed_count, B, L, ctx_io, p,
                         stream=None):
        """Saliency-aware approximate attention of one layer, contexts ctx_io
        and probabilities p [B, H, L, L] float32 updated in place; see
        esd_approx_attention."""
        self._check(_lib.esd_approx_attention(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(v_prev),
                                              _ptr(changed_idx), _ptr(changed_count), B, L,
                                              _ptr(ctx_io), _ptr(p), _stream(stream)))

    def partial_attention(self, q, k_cache, v_cache, B, L, k, out, stream=None):
        self._check(_lib.esd_partial_attention(self.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                               B, L, k, _ptr(out), _stream(stream)))

    def confidence_argmax(self, x_rows, idx, B, L, k, conf_out, tok_out, stream=None):
        self._check(_lib.esd_confidence_argmax(self.handle, _ptr(x_rows), _ptr(idx), B, L, k,
                                               _ptr(conf_out), _ptr(tok_out), _stream(stream)))

    def logits(self, x_rows, rows, out, stream=None):
        self._check(_lib.esd_logits(self.handle, _ptr(x_rows), rows, _ptr(out), _stream(stream)))

    def remask(self, tok, masked, conf_cache, tok_cache, B, L, block_begin, block_end, n_unmask,
               stream=None):
        self._check(_lib.esd_remask(self.handle, _ptr(tok), _ptr(masked), _ptr(conf_cache),
                                    _ptr(tok_cache), B, L, block_begin, block_end, n_unmask,
                                    _stream(stream)))

    def denoise_step(self, tok, masked, block_begin, block_end, n_unmask, force_dense=False,
                     stream=None):
        B, L = tok.shape
        self._check(_lib.esd_denoise_step(self.handle, _ptr(tok), _ptr(masked), B, L, block_begin,
                                          block_end, n_unmask, int(force_dense), _stream(stream)))

    def denoise_step_region(self, tok, masked, region_begin, region_end, block_begin, block_end, n_unmask,
                            force_dense=False, stream=None):
        """esd_denoise_step_region: recompute rows [region_begin, region_end)
        (block or response scope), remask within [block_begin, block_end)."""
        B, L = tok.shape
        self._check(_lib.esd_denoise_step_region(self.handle, _ptr(tok), _ptr(masked), B, L, region_begin,
                                                 region_end, block_begin, block_end, n_unmask, int(force_dense),
                                                 _stream(stream)))

    def generate(self, prompt, gen: int, block_len: int, n_unmask: int, out=None, vanilla=False,
                 stream=None):
        """prompt: int32 [B, P] tensor on the host or the device; returns out [B, gen]."""
        B, P = prompt.shape
        if out is None:
            out = torch.empty((B, gen), dtype=torch.int32, device=prompt.device)
        self._check(_lib.esd_generate(self.handle, _ptr(prompt), B, P, gen, block_len, n_unmask,
                                      int(vanilla), _ptr(out), _stream(stream)))
        return out

    def profile_enable(self, kernel: int, rows_min: int = 0, rows_max: int = 1 << 30):
        self._check(_lib.esd_profile_enable(self.handle, kernel, rows_min, rows_max))

    def profile_read(self, reset: bool = True):
        """(total device ms, launches) of the profiled family since the last reset."""
        t = ctypes.c_double()
        n = ctypes.c_uint64()
        self._check(_lib.esd_profile_read(self.handle, ctypes.byref(t), ctypes.byref(n), int(reset)))
        return t.value, int(n.value)

    def sync_check(self, stream=None):
        self._check(_lib.esd_sync_check(self.handle, _stream(stream)))

    def selftest_wait_timeout(self, polls=1 << 16, stream=None):
        """Make one bounded device wait expire; the next sync_check raises
        EsdError(ESD_ERR_TIMEOUT). See esd_selftest_wait_timeout."""
        self._check(_lib.esd_selftest_wait_timeout(self.handle, int(polls), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 8 << 20


def confidence_argmax_noalloc(x_rows, rows: int, w_out, d: int, vocab: int, mask_id: int,
                              rms_eps: float, idx, L: int, k: int, conf_out, tok_out, stream=None):
    """esd_confidence_argmax_noalloc: the head for bf16 models without a context
    and without any device allocation (for callers that cannot allocate). The
    outputs are valid once noalloc_check() returns without raising."""
    st = _lib.esd_confidence_argmax_noalloc(_ptr(x_rows), rows, _ptr(w_out), d, vocab, mask_id,
                                            rms_eps, _ptr(idx), L, k, _ptr(conf_out),
                                            _ptr(tok_out), _stream(stream))
    if st != ESD_OK:
        raise EsdError(st, "esd_confidence_argmax_noalloc failed (sizes beyond the scratch limit, "
                           "bad arguments or a CUDA error)")


def noalloc_check(stream=None):
    """esd_noalloc_check: raises EsdError(ESD_ERR_TIMEOUT) when a device wait of
    the last allocation-free head call on this device ran out."""
    st = _lib.esd_noalloc_check(_stream(stream))
    if st != ESD_OK:
        raise EsdError(st, "the last allocation-free head call did not complete (status %d)" % st)


def noalloc_selftest_wait_timeout(polls=1 << 16, stream=None):
    """esd_noalloc_selftest_wait_timeout: make one bounded wait on the
    allocation-free head's status word run out (no fault)."""
    st = _lib.esd_noalloc_selftest_wait_timeout(int(polls), _stream(stream))
    if st != ESD_OK:
        raise EsdError(st, "esd_noalloc_selftest_wait_timeout failed")


def make_dims(n_layers, d, n_heads, head_dim, ffn, vocab, mask_id, rope_theta=10000.0,
              rms_eps=1e-6, dtype="bf16") -> ModelDims:
    return ModelDims(n_layers, d, n_heads, head_dim, ffn, vocab, mask_id, rope_theta, rms_eps,
                     DTYPE_BF16 if dtype == "bf16" else DTYPE_F32)


def make_run(score_mode="es", alpha=0.5, lam=0.5, skip_layer=1, keep_ratio=0.25,
             refresh_interval=0, max_batch=1, max_len=128, skip_layer2=0,
             keep_ratio2=1.0, score_tensor="h", scope="all") -> RunConfig:
    return RunConfig(SCORE_COS if score_mode == "cos" else SCORE_ES, alpha, lam, skip_layer,
                     keep_ratio, refresh_interval, max_batch, max_len, skip_layer2, keep_ratio2,
                     {"h": 0, "k": 1, "v": 2}[score_tensor], {"all": 0, "block": 1, "response": 2}[scope])
