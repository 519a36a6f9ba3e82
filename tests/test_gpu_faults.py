"""Failure paths that need a device but fault nothing on it.

Out-of-memory: the library's host-side allocation counter is told to refuse
the n-th allocation from now, for every n that strata_moe_create reaches.
Each refused create must return STRATA_ERR_OOM, leave *out NULL and hold no
block afterwards (the live-allocation count is back where it was); the first
create that is let through must work and give the oracle's routing.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import gen
import oracle
import quantized_expert_ffn_04_b200 as qe


def _create_raw(layer, max_tokens):
    cfg = qe.make_config(layer.shape, max_tokens)
    w, keep = qe.make_weights(layer)
    h = C.c_void_p(12345)  # must come back NULL on failure
    st = qe._lib.strata_moe_create(C.byref(cfg), C.byref(w), 0, C.byref(h))
    del keep
    return st, h


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [gen.TINY, gen.FLASH2], ids=["tiny", "flash2"])
def test_create_oom_injection_no_leak(shape):
    layer = gen.layer_weights(shape, seed=0)
    T = 8
    base = qe.strata_moe_debug_live_allocs()
    refused = 0
    h = None
    try:
        for n in range(64):
            qe.strata_moe_debug_fail_alloc(n)
            st, hh = _create_raw(layer, T)
            qe.strata_moe_debug_fail_alloc(-1)
            if st == qe.STRATA_OK:
                h = hh
                break
            assert st == qe.STRATA_ERR_OOM, (n, st, qe.strata_moe_last_error())
            assert hh.value is None, f"allocation {n}: *out not NULL after a failed create"
            assert qe.strata_moe_debug_live_allocs() == base, f"allocation {n}: blocks leaked"
            refused += 1
        assert h is not None, "create never succeeded"
    finally:
        qe.strata_moe_debug_fail_alloc(-1)
    # weights, router copy, router bias (flash2), workspace, pinned error
    # word, router split, two staging buffers
    assert refused >= 7, refused
    assert qe.strata_moe_debug_live_allocs() > base
    x = gen.hidden(T, shape.hidden, seed=3)
    xt = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).cuda()
    idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
    qe.strata_moe_route(h, xt.data_ptr(), T, idx.data_ptr(), wts.data_ptr())
    qe.strata_moe_sync_status(h)
    _, _, ridx, _ = oracle.moe_forward(layer, x)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    qe.strata_moe_destroy(h)
    assert qe.strata_moe_debug_live_allocs() == base


@pytest.mark.gpu
def test_debug_dequant_oom_injection():
    layer = gen.layer_weights(gen.TINY, seed=0)
    L = qe.Layer(layer, max_tokens=4)
    base = qe.strata_moe_debug_live_allocs()
    out = np.zeros((4, gen.TINY.hidden), dtype=np.float32)
    qe.strata_moe_debug_fail_alloc(0)
    try:
        with pytest.raises(qe.StrataError) as ei:
            qe.strata_moe_debug_dequant(L.handle, 0, 0, 0, 4, 0, out.ctypes.data)
    finally:
        qe.strata_moe_debug_fail_alloc(-1)
    assert ei.value.status == qe.STRATA_ERR_OOM
    assert qe.strata_moe_debug_live_allocs() == base
    qe.strata_moe_debug_dequant(L.handle, 0, 0, 0, 4, 0, out.ctypes.data)  # works again
    L.close()


# ------------------------------------------------------------------ checked build
_CHECKED_CHILD = r"""
import sys, numpy as np, torch
import gen, quantized_expert_ffn_04_b200 as qe
assert qe.LIB_PATH.endswith("libstrata_moe_checked.so"), qe.LIB_PATH
name, T, path, out = sys.argv[1], int(sys.argv[2]), int(sys.argv[3]), sys.argv[4]
shape = getattr(gen, name)
layer = gen.layer_weights(shape, seed=0)
x = gen.hidden(T, shape.hidden, seed=7)
L = qe.Layer(layer, max_tokens=T)
L.set_option(qe.STRATA_OPT_PATH, path)
xt = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).cuda()
y = L.forward(xt)
L.sync_status()   # raises on STRATA_ERR_BOUNDS
np.save(out, y.cpu().view(torch.int16).numpy())
L.close()
print("checked ok")
"""


@pytest.mark.gpu
@pytest.mark.parametrize("name,T,path", [("TINY", 8, 0), ("FLASH2", 4, 0), ("FLASH2", 4, 1),
                                         ("FLASH2", 300, 0), ("FLASH3", 64, 0)])
def test_checked_build_same_bits(name, T, path, tmp_path):
    """The checked library (every gather/scatter index tested on the device)
    reports no bad index on these cases and gives the normal library's bits."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = str(tmp_path / "y.npy")
    env = dict(os.environ, STRATA_MOE_CHECKED="1", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", _CHECKED_CHILD, name, str(T), str(path), out],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "checked ok" in r.stdout, r.stderr[-3000:]
    shape = getattr(gen, name)
    layer = gen.layer_weights(shape, seed=0)
    x = gen.hidden(T, shape.hidden, seed=7)
    L = qe.Layer(layer, max_tokens=T)
    L.set_option(qe.STRATA_OPT_PATH, path)
    xt = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).cuda()
    y = L.forward(xt).cpu().view(torch.int16).numpy()
    L.sync_status()
    L.close()
    assert np.array_equal(np.load(out), y)
