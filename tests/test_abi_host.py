"""Host-side checks of the C ABI: the library loads, exports every entry point
include/ssa.h declares, sizes its workspace, and rejects bad arguments on the
host before anything reaches a device.  No compute call is made."""
import ctypes

import pytest

from block_sparse_attention_ssa_b200 import api


@pytest.fixture(scope="module")
def lib():
    return api.load_library()


def test_exports_every_declared_symbol(lib):
    names = api.header_symbols()
    assert len(names) >= 10
    for name in ("ssa_block_scores", "ssa_select_topk", "ssa_fwd_dual", "ssa_bwd_dual", "ssa_dropped_mass"):
        assert name in names
    for name in names:
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.ssa_version() == 110
    for code, name in enumerate(["SSA_OK", "SSA_ERR_INVALID_ARG", "SSA_ERR_UNSUPPORTED", "SSA_ERR_CUDA",
                                 "SSA_ERR_TIMEOUT", "SSA_ERR_WORKSPACE"]):
        assert api.status_string(code) == name
    assert api.status_string(99) == "SSA_ERR_UNKNOWN"


def test_workspace_bytes():
    d = api.make_dims(2, 32, 8, 16384, 128, 64, 16)
    ws = api.ssa_workspace_bytes(d)
    rows = 2 * 32 * 16384
    # backward dominates: two fp32 [B,Hq,N,d] buffers plus row vectors
    assert ws >= 2 * rows * 128 * 4 + 2 * rows * 4
    assert ws % 256 == 0
    assert api.ssa_workspace_bytes(api.make_dims(0, 32, 8, 16384, 128, 64, 16)) == 0
    assert api.ssa_workspace_bytes(api.make_dims(1, 4, 2, 1000, 128, 64, 16)) == 0  # N % block
    assert api.ssa_workspace_bytes(api.make_dims(1, 4, 3, 1024, 128, 64, 16)) == 0  # Hq % Hkv
    assert api.ssa_workspace_bytes(api.make_dims(1, 4, 2, 1040, 64, 16, 16)) == 0   # N % 64 (block 16)
    assert api.ssa_workspace_bytes(api.make_dims(1, 4, 2, 1024, 64, 16, 16)) > 0    # block 16


def _tensor(ptr=16, sb=4096 * 128, sh=4096 * 128, sn=128):
    return ctypes.pointer(api.ssa_tensor_t(ptr, sb, sh, sn))


@pytest.mark.parametrize("field,value,code", [
    ("block", 8, api.SSA_ERR_UNSUPPORTED),
    ("block", 96, api.SSA_ERR_UNSUPPORTED),
    ("d", 96, api.SSA_ERR_UNSUPPORTED),
    ("N", 1000, api.SSA_ERR_UNSUPPORTED),
    ("N", 64 * 4096, api.SSA_ERR_UNSUPPORTED),
    ("Hkv", 3, api.SSA_ERR_INVALID_ARG),
    ("Hkv", 0, api.SSA_ERR_INVALID_ARG),
    ("topk", 0, api.SSA_ERR_INVALID_ARG),
    ("B", -1, api.SSA_ERR_INVALID_ARG),
    ("dtype", 7, api.SSA_ERR_INVALID_ARG),
    ("per_token", 2, api.SSA_ERR_INVALID_ARG),
    ("scale", float("nan"), api.SSA_ERR_INVALID_ARG),
    ("scale", 0.0, api.SSA_ERR_INVALID_ARG),
    ("scale", -0.125, api.SSA_ERR_INVALID_ARG),
    ("scale", float("inf"), api.SSA_ERR_INVALID_ARG),
])
def test_bad_dims_rejected_on_host(lib, field, value, code):
    d = api.make_dims(1, 4, 2, 1024, 128, 64, 4)
    setattr(d, field, value)
    t = _tensor()
    got = lib.ssa_fwd_dual(ctypes.byref(d), t, t, t, ctypes.c_void_p(16), t, t, ctypes.c_void_p(16),
                           ctypes.c_void_p(16), ctypes.c_void_p(16), None)
    assert got == code
    got = lib.ssa_block_scores(ctypes.byref(d), t, t, ctypes.c_void_p(16), ctypes.c_void_p(256), 1 << 40, None)
    assert got == code


def test_bad_tensors_rejected_on_host(lib):
    d = api.make_dims(1, 4, 2, 1024, 128, 64, 4)
    good = _tensor()
    p = ctypes.c_void_p(16)
    cases = [
        _tensor(ptr=8),            # misaligned base
        _tensor(sn=100),           # stride * 2 bytes not a multiple of 16
        _tensor(sn=64),            # rows overlap (stride < d)
        _tensor(sb=-128),          # negative stride
        None,                      # missing tensor
    ]
    for bad in cases:
        assert lib.ssa_fwd_dual(ctypes.byref(d), bad, good, good, p, good, good, p, p, p, None) == api.SSA_ERR_INVALID_ARG
    # null idx / outputs
    assert lib.ssa_fwd_dual(ctypes.byref(d), good, good, good, None, good, good, p, p, p, None) == api.SSA_ERR_INVALID_ARG
    assert lib.ssa_select_topk(ctypes.byref(d), None, p, None) == api.SSA_ERR_INVALID_ARG
    assert lib.ssa_device_status(None, 0, None) == api.SSA_ERR_INVALID_ARG


def test_workspace_checked_before_launch(lib):
    d = api.make_dims(1, 4, 2, 1024, 128, 64, 4)
    t = _tensor()
    p = ctypes.c_void_p(256)
    need = api.ssa_workspace_bytes(d)
    assert lib.ssa_block_scores(ctypes.byref(d), t, t, p, p, need - 1, None) == api.SSA_ERR_WORKSPACE
    assert lib.ssa_block_scores(ctypes.byref(d), t, t, p, None, need, None) == api.SSA_ERR_WORKSPACE
    assert lib.ssa_bwd_dual(ctypes.byref(d), t, t, t, p, t, t, p, p, None, None, 10.0, None, t, t, t,
                            p, 0, None) == api.SSA_ERR_WORKSPACE
    assert lib.ssa_dropped_mass(ctypes.byref(d), t, t, p, None, p, p, 16, None) == api.SSA_ERR_WORKSPACE


def test_empty_shapes_are_noops(lib):
    t = _tensor()
    p = ctypes.c_void_p(16)
    for field in ("B", "N", "Hq"):
        d = api.make_dims(1, 4, 2, 1024, 128, 64, 4)
        setattr(d, field, 0)
        assert lib.ssa_fwd_dual(ctypes.byref(d), t, t, t, p, t, t, p, p, p, None) == api.SSA_OK
        assert lib.ssa_select_topk(ctypes.byref(d), p, p, None) == api.SSA_OK


def test_selection_modes_are_exclusive(lib):
    """Per-block scoring entry points refuse per-token dims and the per-token
    selection refuses per-block dims, before anything is enqueued."""
    t = _tensor()
    dt = api.make_dims(1, 4, 2, 1024, 128, 64, 4, per_token=True)
    db = api.make_dims(1, 4, 2, 1024, 128, 64, 4)
    assert lib.ssa_block_scores(ctypes.byref(dt), t, t, ctypes.c_void_p(16), ctypes.c_void_p(256), 1 << 40,
                                None) == api.SSA_ERR_INVALID_ARG
    assert lib.ssa_select_topk(ctypes.byref(dt), ctypes.c_void_p(16), ctypes.c_void_p(16), None) == \
        api.SSA_ERR_INVALID_ARG
    assert lib.ssa_select_tokens(ctypes.byref(db), t, t, ctypes.c_void_p(16), ctypes.c_void_p(256), 1 << 40,
                                 None) == api.SSA_ERR_INVALID_ARG
    # the per-token selection mask is per token: the workspace grows accordingly
    assert api.ssa_workspace_bytes(dt) >= api.ssa_workspace_bytes(db)
