"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/tlp.h declares, and rejects bad arguments and
out-of-order calls with the documented status codes before touching a
device."""
import ctypes
import os
import re
import subprocess

import pytest

import transformer_layer_pre_b200 as tlp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tlp.h")

TL_OK, TL_EINVAL, TL_ESTATE = 0, 1, 3


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    text = re.sub(r"typedef[^;]*;", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([A-Za-z_]\w*)\s*\(", text)) - {"defined"})


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(tlp.LIB_PATH):
        from transformer_layer_pre_b200 import build_ext
        build_ext.build()
    return tlp.load_library()


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", tlp.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(lib, n)
    assert set(tlp.EXPORTED_SYMBOLS) == set(names)


def _create(lib, *args):
    h = ctypes.c_void_p()
    st = lib.layer_create(*args, ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("args", [
    (0, 128, 1024, 16, 0, 0.1, 0.1, 1, 1),        # batch 0
    (2, 128, 1000, 16, 0, 0.1, 0.1, 1, 1),        # hidden % heads
    (2, 128, 1024, 4, 0, 0.1, 0.1, 1, 1),         # head dim 256
    (2, 128, 96, 4, 0, 0.1, 0.1, 1, 1),           # head dim 24
    (2, 100, 1024, 16, 0, 0.1, 0.1, 1, 1),        # seq % 8
    (2, 128, 1024, 16, 100, 0.1, 0.1, 1, 1),      # ffn % 8
    (2, 128, 1024, 16, 0, 1.0, 0.1, 1, 1),        # p = 1
    (2, 128, 1024, 16, 0, 0.1, -0.1, 1, 1),       # p < 0
    (2, 128, 1024, 16, 0, float("nan"), 0.1, 1, 1),
])
def test_create_rejects_bad_arguments(lib, args):
    st, h = _create(lib, *args)
    assert st == TL_EINVAL and not h.value


def test_create_defaults_and_state_errors(lib):
    st, h = _create(lib, 2, 16, 64, 4, 0, 0.1, 0.1, 1, 1234)
    assert st == TL_OK and h.value
    try:
        opt = tlp.Options()
        assert lib.layer_get_options(h, ctypes.byref(opt)) == TL_OK
        assert opt.dtype == 0 and opt.training == 1 and abs(opt.ln_eps - 1e-12) < 1e-18
        assert opt.stochastic_mode == 0   # bitwise-reproducible by default
        # the dropout generator's key and counter word change without a reallocation
        assert lib.layer_set_rng(None, 1, 2) == TL_EINVAL
        assert lib.layer_set_rng(h, 99, 7) == TL_OK
        assert lib.layer_get_options(h, ctypes.byref(opt)) == TL_OK and opt.philox_offset == 7
        assert lib.layer_workspace_bytes(h) == 0
        assert lib.layer_workspace_bytes(h) == 0  # nothing allocated before options / forward
        w = tlp._Weights(*([1] * 12))
        st = lib.layer_backward(h, 1, 1, ctypes.byref(w), ctypes.byref(w), 1, None)
        assert st == TL_ESTATE
        assert b"forward" in lib.layer_last_error(h)
        st = lib.layer_forward(h, None, None, ctypes.byref(w), 1, None)
        assert st == TL_EINVAL
    finally:
        lib.layer_destroy(h)


def test_dropout_hook_rejects_unaligned_ranges(lib):
    assert lib.tl_dropout_keep_mask(1, 0, 0, 0.1, 3, 8, 1, None) == TL_EINVAL
    assert lib.tl_dropout_keep_mask(1, 0, 0, 0.1, 0, 7, 1, None) == TL_EINVAL
    assert lib.tl_dropout_keep_mask(1, 0, 0, 1.5, 0, 8, 1, None) == TL_EINVAL
