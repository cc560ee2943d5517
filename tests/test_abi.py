"""The C ABI (CPU): libnvium.so loads without a GPU, exports every function
include/nvium.h declares, and rejects bad arguments on the host before any
device work."""
import ctypes
import os
import re

import pytest

import exact_early_exit_b200 as nv
import workloads as W

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvium.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nv_[a-z0-9_]+)\s*\(", text)))


def test_library_is_built_and_loads():
    assert os.path.exists(nv.LIB_PATH), "build with python -m exact_early_exit_b200.build"
    nv.lib()


def test_every_declared_function_is_exported():
    names = declared_functions()
    assert "nv_create" in names and "nv_decode_step" in names and "nv_flush_deferred" in names
    L = ctypes.CDLL(nv.LIB_PATH)
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_binding_covers_every_declared_function():
    bound = {n for n, _, _ in nv._SIGS}
    assert set(declared_functions()) <= bound


def _cfg(**kw):
    c = nv.make_config(W.TINY, max_batch=2, max_seq=64)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value", [
    ("n_layers", 0), ("head_dim", 48), ("dtype", 7), ("page_size", 48), ("max_pending", 1),
    ("max_batch", 0), ("router_mode", 5), ("n_exits", 0), ("router_hidden", -1), ("router_hidden", 4096),
])
def test_create_rejects_bad_config_on_host(field, value):
    c = _cfg(**{field: value})
    h = ctypes.c_void_p()
    w = nv.Weights()
    st = nv.lib().nv_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h))
    assert st == nv.NV_ERR_INVALID_ARG
    assert b"invalid config" in nv.lib().nv_last_error()
    assert not h.value


def test_create_rejects_bad_exit_layers_and_null_weights():
    c = _cfg()
    c.exit_layers[1] = 1  # not increasing
    h = ctypes.c_void_p()
    assert nv.lib().nv_create(ctypes.byref(c), ctypes.byref(nv.Weights()), ctypes.byref(h)) == nv.NV_ERR_INVALID_ARG
    c = _cfg()
    assert nv.lib().nv_create(ctypes.byref(c), ctypes.byref(nv.Weights()), ctypes.byref(h)) == nv.NV_ERR_INVALID_ARG
    assert b"null" in nv.lib().nv_last_error()


def test_null_handles_are_rejected():
    L = nv.lib()
    assert L.nv_destroy(None) == nv.NV_ERR_INVALID_ARG
    assert L.nv_state_destroy(None) == nv.NV_ERR_INVALID_ARG
    assert L.nv_flush_deferred(None, None) == nv.NV_ERR_INVALID_ARG
    assert L.nv_rewind(None, None) == nv.NV_ERR_INVALID_ARG
    assert L.nv_decode_step(None, 1, None, None, None, None) == nv.NV_ERR_INVALID_ARG
    assert L.nv_score_mixture(None, None, 1, 2, None, None, None) == nv.NV_ERR_INVALID_ARG
    assert L.nv_philox4x32_10(1, None, 4, None, None) == nv.NV_ERR_INVALID_ARG


def test_last_error_is_per_thread():
    """nv_last_error is thread-local: another thread's failing call does not
    replace this thread's message."""
    import threading
    L = nv.lib()
    h = ctypes.c_void_p()
    assert L.nv_create(ctypes.byref(_cfg(n_layers=0)), ctypes.byref(nv.Weights()), ctypes.byref(h)) == \
        nv.NV_ERR_INVALID_ARG
    mine = L.nv_last_error()
    other = []

    def fail_elsewhere():
        c = _cfg()
        c.exit_layers[1] = 1
        L.nv_create(ctypes.byref(c), ctypes.byref(nv.Weights()), ctypes.byref(ctypes.c_void_p()))
        other.append(L.nv_last_error())

    t = threading.Thread(target=fail_elsewhere)
    t.start()
    t.join()
    assert other and other[0] != mine
    assert L.nv_last_error() == mine


def test_binding_constants_match_the_header():
    """Limits the binding repeats from include/nvium.h have the header's values."""
    text = open(HEADER).read()
    for name in ("NV_PHILOX_NOALLOC_MAX", "NV_MAX_EXITS"):
        m = re.search(r"#define\s+" + name + r"\s+(\d+)", text)
        assert m, name
        assert int(m.group(1)) == getattr(nv, name), name


def test_router_probs_rejects_null_state():
    assert nv.lib().nv_read_router_probs(None, None, None) == nv.NV_ERR_INVALID_ARG
