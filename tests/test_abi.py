"""The C-ABI library loads without a GPU, exports every symbol include/esd.h
declares, its ctypes mirrors match the C struct layouts, and it reports errors
instead of crashing when no device is present. No compute call is made."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "esd.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(esd_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import token_skipping_sparse_step_b200 as esd
    names = _declared()
    assert len(names) >= 15
    lib = ctypes.CDLL(esd.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(esd.EXPORTS)


def test_struct_layouts_match_c(tmp_path):
    import token_skipping_sparse_step_b200 as esd
    src = tmp_path / "sz.c"
    src.write_text('#include "esd.h"\n#include <stdio.h>\n#include <stddef.h>\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(esd_model_dims),'
                   ' sizeof(esd_weights), sizeof(esd_run_config), sizeof(esd_state_view),'
                   ' offsetof(esd_run_config, max_len), offsetof(esd_state_view, n_cached_layers));'
                   'return 0;}\n')
    exe = tmp_path / "sz"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [ctypes.sizeof(esd.ModelDims), ctypes.sizeof(esd.Weights), ctypes.sizeof(esd.RunConfig),
            ctypes.sizeof(esd.StateView), esd.RunConfig.max_len.offset, esd.StateView.n_cached_layers.offset]
    assert got == want


def test_null_arguments_are_rejected_without_a_device():
    import token_skipping_sparse_step_b200 as esd
    lib = esd._lib
    h = ctypes.c_void_p()
    assert lib.esd_create(None, None, None, ctypes.byref(h)) == 1      # ESD_ERR_INVALID_ARG
    assert lib.esd_create(None, None, None, None) == 1
    assert lib.esd_destroy(None) == 1
    assert lib.esd_sync_check(None, None) == 1
    assert lib.esd_approx_attention(None, None, None, None, None, None, None, 1, 1, None, None, None) == 1
    assert lib.esd_keep_count(None, 10) == 0
    assert lib.esd_last_error(None) == b"null context"


def test_bad_shapes_are_rejected_before_any_device_call():
    import token_skipping_sparse_step_b200 as esd
    dims = esd.make_dims(2, 256, 4, 60, 688, 1024, 1023, dtype="f32")   # d != H * hd
    run = esd.make_run(score_mode="cos", skip_layer=1, max_len=128)
    one = (ctypes.c_void_p * 2)(8, 8)
    pp = ctypes.cast(one, esd._PP)
    w = esd.Weights(8, 8, pp, pp, pp, pp, pp, pp, pp)
    h = ctypes.c_void_p()
    assert esd._lib.esd_create(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h)) == 1
    dims = esd.make_dims(2, 256, 4, 64, 688, 1024, 1023, dtype="f32")
    run = esd.make_run(score_mode="cos", skip_layer=2, max_len=128)      # skip layer out of range
    assert esd._lib.esd_create(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h)) == 1
    run = esd.make_run(score_mode="cos", skip_layer=1, keep_ratio=0.0, max_len=128)
    assert esd._lib.esd_create(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h)) == 1
    bdims = esd.make_dims(2, 256, 4, 64, 688, 1024, 1023, dtype="bf16")  # bf16 needs head_dim 128
    run = esd.make_run(skip_layer=1, max_len=128)
    assert esd._lib.esd_create(ctypes.byref(bdims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h)) == 4


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device path")
def test_create_without_device_reports_an_error():
    import token_skipping_sparse_step_b200 as esd
    dims = esd.make_dims(2, 256, 4, 64, 688, 1024, 1023, dtype="f32")
    run = esd.make_run(score_mode="cos", skip_layer=1, max_len=128)
    one = (ctypes.c_void_p * 2)(8, 8)
    pp = ctypes.cast(one, esd._PP)
    w = esd.Weights(8, 8, pp, pp, pp, pp, pp, pp, pp)
    h = ctypes.c_void_p()
    st = esd._lib.esd_create(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h))
    assert st in (2, 4) and not h.value


def test_step_variant_configs_are_validated_before_any_device_call():
    """The second skip point, the score tensor and the selection scope are
    checked at esd_create before any device call."""
    import token_skipping_sparse_step_b200 as esd
    dims = esd.make_dims(4, 256, 4, 64, 688, 1024, 1023, dtype="f32")
    one = (ctypes.c_void_p * 4)(8, 8, 8, 8)
    pp = ctypes.cast(one, esd._PP)
    w = esd.Weights(8, 8, pp, pp, pp, pp, pp, pp, pp)
    h = ctypes.c_void_p()

    def create(**kw):
        run = esd.make_run(score_mode="cos", skip_layer=1, max_len=128, **kw)
        return esd._lib.esd_create(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h))

    assert create(skip_layer2=1, keep_ratio2=0.5) == 1     # not after the first point
    assert create(skip_layer2=4, keep_ratio2=0.5) == 1     # not inside the model
    assert create(skip_layer2=3, keep_ratio2=0.0) == 1     # empty second selection
    assert create(skip_layer2=3, keep_ratio2=1.5) == 1
    run = esd.make_run(score_mode="cos", skip_layer=1, max_len=128)
    run.score_tensor = 3                                   # no such tensor
    assert esd._lib.esd_create(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h)) == 1
    run = esd.make_run(score_mode="cos", skip_layer=1, max_len=128)
    run.scope = 3                                          # no such scope
    assert esd._lib.esd_create(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(run), ctypes.byref(h)) == 1
    assert create(scope="block", score_tensor="k") == 4    # the block scope scores H
    assert create(scope="block", skip_layer2=3, keep_ratio2=0.5) == 4   # with one skip point
    assert create(scope="response", score_tensor="v") == 4              # response-only steps too
    assert create(scope="response", skip_layer2=3, keep_ratio2=0.5) == 4
    assert not h.value


def test_stream_probe_library_loads_and_rejects_bad_arguments():
    """The HBM streaming probe behind bench.py --stream-probe: built beside the
    library, one entry point, invalid arguments refused before any CUDA call."""
    path = os.path.join(ROOT, "token_skipping_sparse_step_b200", "libstream_probe.so")
    lib = ctypes.CDLL(path)
    fn = lib.esd_stream_probe
    fn.argtypes = [ctypes.c_int, ctypes.c_longlong, ctypes.c_int, ctypes.POINTER(ctypes.c_float)]
    fn.restype = ctypes.c_int
    us = ctypes.c_float(0.0)
    assert fn(2, 1 << 30, 1, ctypes.byref(us)) == 2          # unknown kind
    assert fn(0, 1000, 1, ctypes.byref(us)) == 2             # less than one 1 MiB tile
    assert fn(0, 1 << 30, 0, ctypes.byref(us)) == 2          # no launch
    assert fn(1, 1 << 30, 1, None) == 2                      # no output
