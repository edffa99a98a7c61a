"""The C-ABI library without a GPU: it loads, exports every entry point that include/moe.h
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import sparse_expert_ffn_logits_b200 as moe
from sparse_expert_ffn_logits_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load()


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:moe_status|size_t|const char\s*\*)\s*(moe_\w+)\s*\(",
                                 src, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 9, names
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert set(names) == set(moe.EXPORTS)


def _cfg(**kw):
    base = dict(hidden=2048, n_routed=64, top_k=8, inter=1024, n_shared=0, inter_shared=0,
                max_tokens=16, dtype="bf16", route="softmax_topk")
    base.update(kw)
    return moe.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(hidden=0), moe.MOE_ERR_INVALID_ARG),
    (dict(top_k=65), moe.MOE_ERR_INVALID_ARG),
    (dict(max_tokens=0), moe.MOE_ERR_INVALID_ARG),
    (dict(n_shared=1, inter_shared=0), moe.MOE_ERR_INVALID_ARG),
    (dict(dtype=7), moe.MOE_ERR_INVALID_ARG),
    (dict(route=9), moe.MOE_ERR_INVALID_ARG),
    (dict(hidden=2000), moe.MOE_ERR_UNSUPPORTED),
    (dict(hidden=16384), moe.MOE_ERR_UNSUPPORTED),
    (dict(inter=1000), moe.MOE_ERR_UNSUPPORTED),
    (dict(top_k=17, n_routed=64), moe.MOE_ERR_UNSUPPORTED),
    (dict(n_routed=1024, top_k=2), moe.MOE_ERR_UNSUPPORTED),
    (dict(max_tokens=4096), moe.MOE_ERR_UNSUPPORTED),
    (dict(n_shared=9, inter_shared=1024), moe.MOE_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_config(lib, kw, status):
    h = ctypes.c_void_p()
    assert lib.moe_create(ctypes.byref(_cfg(**kw)), ctypes.byref(h)) == status
    assert not h.value


def test_create_null_args(lib):
    h = ctypes.c_void_p()
    assert lib.moe_create(None, ctypes.byref(h)) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_create(ctypes.byref(_cfg()), None) == moe.MOE_ERR_INVALID_ARG


def test_packed_bytes(lib):
    assert moe.moe_packed_bytes(_cfg()) == (1024 * 2048 * 2, 2 * 1024 * 2048 * 2)
    c = _cfg(dtype="f32", n_shared=2, inter_shared=1408)
    assert moe.moe_packed_bytes(c, shared=1) == (1408 * 2048 * 4, 2 * 1408 * 2048 * 4)
    with pytest.raises(moe.MoEError):
        moe.moe_packed_bytes(_cfg(), shared=1)


def test_forward_rejects_null_handle(lib):
    rw = moe.MoEExpertWeights(16, 16)
    sp = moe.sparsity(("topk", 0.5))
    rc = lib.moe_forward(None, ctypes.c_void_p(16), 1, ctypes.c_void_p(16), ctypes.byref(rw), None,
                         ctypes.byref(sp), None, ctypes.c_void_p(16), None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_get_error(None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_destroy(None) == moe.MOE_OK
    assert lib.moe_debug_lists(None, 1, None, None, None, None, None, None, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lib.moe_set_dense_min_tokens(None, 8) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_set_fused(None, 1) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_force_timeout(None, None) == moe.MOE_ERR_INVALID_ARG
    n = ctypes.c_int(-1)
    assert lib.moe_last_launches(None, ctypes.byref(n)) == moe.MOE_ERR_INVALID_ARG
    ro = moe.MoERoster(16, 16, 4, 0.5)
    rc = lib.moe_forward_roster(None, ctypes.c_void_p(16), 1, ctypes.c_void_p(16),
                                ctypes.byref(ro), ctypes.byref(rw), None, ctypes.byref(sp), None,
                                ctypes.c_void_p(16), None)
    assert rc == moe.MOE_ERR_INVALID_ARG


def test_other_entry_points_reject_null_handle(lib):
    # every call that takes a handle checks it on the host, before any CUDA call
    rw = moe.MoEExpertWeights(16, 16)
    sp = moe.sparsity(("topk", 0.5))
    p16 = ctypes.c_void_p(16)
    for fn in (lib.moe_forward_host, lib.moe_forward_partial):
        assert fn(None, p16, 1, p16, ctypes.byref(rw), None, ctypes.byref(sp), None, p16,
                  None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_pack_experts(None, 0, p16, p16, p16, 1, p16, p16, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lib.moe_profile_stages(None, None, 0) == moe.MOE_ERR_INVALID_ARG
    buf = (ctypes.c_ulonglong * 4)()
    assert lib.moe_read_trace(None, buf, 4) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_set_expert_range(None, 0, 1, 0) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_cast_output(None, p16, 1, p16, None) == moe.MOE_ERR_INVALID_ARG


def test_status_strings(lib):
    for s in range(7):
        assert lib.moe_status_string(s)
    assert lib.moe_status_string(99) == b"unknown status"


@pytest.mark.parametrize("kw,n,ptrs,status", [
    (dict(), -1, (16, 16, 16, 16), moe.MOE_ERR_INVALID_ARG),        # negative count
    (dict(), 257, (16, 16, 16, 16), moe.MOE_ERR_UNSUPPORTED),       # beyond the scratch area
    (dict(), 0, (0, 0, 0, 0), moe.MOE_OK),                          # a no-op reads nothing
    (dict(), 4, (0, 16, 16, 16), moe.MOE_ERR_INVALID_ARG),          # null x
    (dict(), 4, (16, 0, 16, 16), moe.MOE_ERR_INVALID_ARG),          # null router
    (dict(), 4, (16, 16, 0, 16), moe.MOE_ERR_INVALID_ARG),          # null topk_idx
    (dict(), 4, (16, 16, 16, 0), moe.MOE_ERR_INVALID_ARG),          # null topk_w
    (dict(), 4, (8, 16, 16, 16), moe.MOE_ERR_INVALID_ARG),          # x not 16-byte aligned
    (dict(), 4, (16, 8, 16, 16), moe.MOE_ERR_INVALID_ARG),          # router not 16-byte aligned
    (dict(), 4, (16, 16, 2, 16), moe.MOE_ERR_INVALID_ARG),          # topk_idx not 4-byte aligned
    (dict(hidden=96), 4, (16, 16, 16, 16), moe.MOE_ERR_UNSUPPORTED),  # hidden not a multiple of 64
    (dict(top_k=65), 4, (16, 16, 16, 16), moe.MOE_ERR_INVALID_ARG),  # top_k above n_routed
    (dict(n_routed=600, top_k=8), 4, (16, 16, 16, 16), moe.MOE_ERR_UNSUPPORTED),
])
def test_route_noalloc_rejects_bad_arguments_before_the_device(lib, kw, n, ptrs, status):
    """Every check of the routing-only call runs on the host, before the scratch area (and so
    the device) is touched: these pointers are never dereferenced."""
    x, router, idx, w = (ctypes.c_void_p(p) if p else None for p in ptrs)
    assert lib.moe_route_noalloc(ctypes.byref(_cfg(**kw)), x, n, router, idx, w, None) == status


def test_route_noalloc_rejects_null_config(lib):
    p = ctypes.c_void_p(16)
    assert lib.moe_route_noalloc(None, p, 4, p, p, p, None) == moe.MOE_ERR_INVALID_ARG
