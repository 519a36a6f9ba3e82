"""Host-side checks of the C-ABI library (no GPU needed): the shared library
loads, exports every entry point include/strata_moe.h declares, and rejects
bad arguments before touching the device."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import gen
import quantized_expert_ffn_04_b200 as qe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "strata_moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(strata_(?:moe|ep)_\w+)\s*\(", text)))


def test_header_symbols_exported():
    names = _declared()
    assert len(names) >= 12
    lib = C.CDLL(qe.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(qe.SYMBOLS) == names


def test_checked_build_exports_the_same_symbols():
    """The checked variant (-DSTRATA_CHECKS=1) is the same ABI."""
    path = os.path.join(os.path.dirname(qe.LIB_PATH), "libstrata_moe_checked.so")
    assert os.path.exists(path), "build the checked variant (__graft_entry__.build())"
    lib = C.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n


def test_version_and_last_error():
    assert "sm_100a" in qe.strata_moe_version()
    assert isinstance(qe.strata_moe_last_error(), str)


def _cfg(**kw):
    c = dict(hidden=256, n_experts=16, top_k=2, inter=64, quant_bits=2, block=32, max_tokens=8,
             has_router_bias=0)
    c.update(kw)
    return qe.strata_moe_config(**c)


@pytest.mark.parametrize("kw,status", [
    (dict(quant_bits=4), qe.STRATA_ERR_UNSUPPORTED),
    (dict(block=64), qe.STRATA_ERR_UNSUPPORTED),
    (dict(hidden=200), qe.STRATA_ERR_UNSUPPORTED),
    (dict(inter=48), qe.STRATA_ERR_UNSUPPORTED),
    (dict(top_k=17), qe.STRATA_ERR_UNSUPPORTED),
    (dict(n_experts=2048, top_k=2), qe.STRATA_ERR_UNSUPPORTED),
    (dict(max_tokens=0), qe.STRATA_ERR_INVALID_ARG),
    (dict(hidden=-128), qe.STRATA_ERR_INVALID_ARG),
])
def test_create_rejects_bad_config(kw, status):
    layer = gen.layer_weights(gen.TINY, seed=0)
    w, keep = qe.make_weights(layer)
    with pytest.raises(qe.StrataError) as ei:
        qe.strata_moe_create(_cfg(**kw), w, 0)
    assert ei.value.status == status
    assert qe.strata_moe_last_error()


def test_create_rejects_null_weights_and_out():
    h = C.c_void_p()
    assert qe._lib.strata_moe_create(C.byref(_cfg()), None, 0, C.byref(h)) == \
        qe.STRATA_ERR_INVALID_ARG
    layer = gen.layer_weights(gen.TINY, seed=0)
    w, keep = qe.make_weights(layer)
    assert qe._lib.strata_moe_create(C.byref(_cfg()), C.byref(w), 0, None) == \
        qe.STRATA_ERR_INVALID_ARG
    w.shared_codes = None
    assert qe._lib.strata_moe_create(C.byref(_cfg()), C.byref(w), 0, C.byref(h)) == \
        qe.STRATA_ERR_INVALID_ARG
    assert h.value is None


def test_null_handle_calls_fail_cleanly():
    qe.strata_moe_destroy(None)  # NULL-safe
    L = qe._lib
    assert L.strata_moe_forward(None, None, 1, None, None) == qe.STRATA_ERR_INVALID_ARG
    assert L.strata_moe_route(None, None, 1, None, None, None, None, None) == \
        qe.STRATA_ERR_INVALID_ARG
    assert L.strata_moe_set_option(None, 1, 0) == qe.STRATA_ERR_INVALID_ARG
    assert L.strata_moe_sync_status(None, None) == qe.STRATA_ERR_INVALID_ARG
    assert L.strata_moe_stack_forward(None, 0, None, 1, None, None) == qe.STRATA_ERR_INVALID_ARG
    assert L.strata_moe_rmsnorm(None, None, -1, 256, None) == qe.STRATA_ERR_INVALID_ARG
    assert L.strata_moe_debug_dequant(None, 0, 0, 0, 1, 0, None) == qe.STRATA_ERR_INVALID_ARG


def test_config_struct_layout_matches_header():
    assert C.sizeof(qe.strata_moe_config) == 8 * 4
    assert C.sizeof(qe.strata_moe_weights) == 6 * C.sizeof(C.c_void_p)


def test_weights_struct_points_into_arrays():
    """Every pointer of the weights struct is the data of the kept array of the
    same field, and each kept array holds the layer's values in the C types the
    header declares (the tiny layer has no router bias, so router_b is NULL)."""
    layer = gen.layer_weights(gen.TINY, seed=0)
    w, keep = qe.make_weights(layer)
    fields = ["codes", "scales", "router_w", "router_b", "shared_codes", "shared_scales"]
    dtypes = [np.uint8, np.uint16, np.float32, np.float32, np.uint8, np.uint16]
    assert layer.router_b is None and w.router_b is None and keep[3] is None
    for name, a, dt in zip(fields, keep, dtypes):
        if a is None:
            continue
        assert getattr(w, name) == a.ctypes.data, name
        assert a.dtype == dt and a.flags.c_contiguous, name
        assert np.array_equal(a.reshape(-1), np.asarray(getattr(layer, name)).reshape(-1)), name
