"""Host-side checks of the C ABI: the library loads without a GPU, exports
every entry point include/mok.h declares, sizes workspaces, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re

import pytest

import combine_device_top_b200 as mok

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(mok_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = mok.lib()
    declared = _declared()
    assert len(declared) >= 12
    missing = [n for n in declared if not hasattr(L, n)]
    assert not missing, missing
    assert set(mok.EXPORTS) <= set(declared)


def test_plan_workspace_sizes():
    L = mok.lib()
    assert L.mok_plan_workspace_bytes(8192, 384, 8) > 8192 * 8 * 4 * 7
    assert L.mok_plan_workspace_bytes(0, 8, 2) > 0            # empty token set is valid
    assert L.mok_plan_workspace_bytes(16, 8, 9) == 0          # k > E
    assert L.mok_plan_workspace_bytes(16, 2048, 2) == 0       # E above the built maximum
    assert L.mok_plan_workspace_bytes(16, 64, 33) == 0        # k above the built maximum


def test_forward_workspace_sizes():
    staged = mok.fwd_opts(mode=mok.MOK_MODE_STAGED)
    s = mok.forward_workspace_bytes(8192, 7168, 2048, 384, 8, 2560, staged)
    ns = 8192 * 8
    assert s >= ns * 7168 * 2 * 2 + ns * 2048 * 2        # rows + out + h
    p = mok.forward_workspace_bytes(8192, 7168, 2048, 384, 8, 2560, mok.fwd_opts(ring_slots=8192))
    assert p < s                                          # the ring is smaller than the full buffers
    assert mok.forward_workspace_bytes(8192, 7168, 2048, 384, 0, 2560, staged) == 0


def _plan_call(T, E, k, R, logits=1, ws=None, nbytes=0):
    p = mok.PlanT()
    L = mok.lib()
    rc = L.mok_plan(ctypes.c_void_p(logits), T, E, k, R, ctypes.c_void_p(ws), nbytes, ctypes.byref(p), None)
    return rc, L.mok_last_error_string().decode()


@pytest.mark.parametrize("T,E,k,R,code", [
    (16, 8, 9, 2, mok.MOK_ERR_INVALID_ARG),      # k > E
    (16, 8, 0, 2, mok.MOK_ERR_INVALID_ARG),      # k = 0
    (16, 8, 2, 0, mok.MOK_ERR_INVALID_ARG),      # R = 0
    (15, 8, 2, 2, mok.MOK_ERR_UNSUPPORTED),      # R does not divide T
    (16, 2048, 2, 2, mok.MOK_ERR_UNSUPPORTED),   # E above the built maximum
    (16, 8, 2, 65, mok.MOK_ERR_UNSUPPORTED),     # R above MOK_MAX_SHARDS
])
def test_plan_rejects_bad_shapes(T, E, k, R, code):
    rc, msg = _plan_call(T, E, k, R)
    assert rc == code, msg
    assert msg


def test_plan_rejects_missing_or_small_workspace():
    rc, msg = _plan_call(16, 8, 2, 2, ws=0, nbytes=0)
    assert rc == mok.MOK_ERR_WORKSPACE and "NULL" in msg
    rc, msg = _plan_call(16, 8, 2, 2, ws=256 * 7 + 128, nbytes=1 << 20)
    assert rc == mok.MOK_ERR_WORKSPACE and "aligned" in msg
    rc, msg = _plan_call(16, 8, 2, 2, ws=4096, nbytes=64)
    assert rc == mok.MOK_ERR_WORKSPACE and "small" in msg


def test_forward_rejects_unsupported_shapes():
    p = mok.PlanT(16, 8, 2, 2)
    L = mok.lib()
    arr = (ctypes.c_void_p * 2)(1, 2)
    rc = L.mok_moe_forward(arr, 100, 256, 1, 1, 1, ctypes.byref(p), 256, None, 256, 1 << 30, arr, None)
    assert rc == mok.MOK_ERR_INVALID_ARG          # plan views are NULL
    for name in ("counts", "offsets", "sched_src_rank", "sched_src_index", "row_slot", "pos", "topk_idx", "gates"):
        setattr(p, name, 4096)
    rc = L.mok_moe_forward(arr, 100, 256, 1, 1, 1, ctypes.byref(p), 256, None, 256, 1 << 30, arr, None)
    assert rc == mok.MOK_ERR_UNSUPPORTED and "H" in mok.last_error()
    rc = L.mok_moe_forward(arr, 128, 100, 1, 1, 1, ctypes.byref(p), 256, None, 256, 1 << 30, arr, None)
    assert rc == mok.MOK_ERR_UNSUPPORTED and "I" in mok.last_error()
    o = mok.fwd_opts(mode=7)
    rc = L.mok_moe_forward(arr, 128, 128, 1, 1, 1, ctypes.byref(p), 256, ctypes.byref(o), 256, 1 << 30, arr, None)
    assert rc == mok.MOK_ERR_INVALID_ARG


def _filled_plan(T, E, k, R):
    p = mok.PlanT(T, E, k, R)
    for name in ("counts", "offsets", "sched_src_rank", "sched_src_index", "row_slot", "pos", "topk_idx", "gates"):
        setattr(p, name, 4096)
    return p


@pytest.mark.parametrize("T,E,k,what", [(16, 2048, 2, "E"), (64, 64, 33, "k"), (1 << 26, 64, 32, "T * k")])
def test_hand_filled_plan_gets_the_plan_limits(T, E, k, what):
    """A plan filled by hand (e.g. from mok_plan_noalloc's outputs) is held to
    mok_plan's limits before anything is launched."""
    p = _filled_plan(T, E, k, 1)
    L = mok.lib()
    arr = (ctypes.c_void_p * 1)(4096)
    rc = L.mok_moe_forward(arr, 128, 128, 1, 1, 1, ctypes.byref(p), 256, None, 256, 1 << 30, arr, None)
    assert rc == mok.MOK_ERR_UNSUPPORTED and what in mok.last_error(), mok.last_error()
    rc = L.mok_combine(4096, mok.MOK_SLOTS_F32, 128, ctypes.byref(p), arr, None)
    assert rc == mok.MOK_ERR_UNSUPPORTED


def test_combine_rejects_an_unknown_slot_type():
    p = _filled_plan(16, 8, 2, 2)
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    rc = mok.lib().mok_combine(4096, 7, 128, ctypes.byref(p), arr, None)
    assert rc == mok.MOK_ERR_INVALID_ARG and "slot" in mok.last_error()


def test_forward_mxfp8_argument_rules():
    """The MXFP8 path runs in either mode, under the persistent mode's own
    rules, and needs every member of its weight pack.  Every call here fails
    validation before any launch (the pointers are not device memory)."""
    p = mok.PlanT(16, 8, 2, 2)
    for name in ("counts", "offsets", "sched_src_rank", "sched_src_index", "row_slot", "pos", "topk_idx", "gates"):
        setattr(p, name, 4096)
    L = mok.lib()
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    full = mok.MxWeights(4096, 4096, 4096, 4096, 4096, 4096)
    pack = ctypes.cast(ctypes.byref(full), ctypes.c_void_p)
    o = mok.fwd_opts(mode=mok.MOK_MODE_PERSISTENT, mxfp8=True)
    rc = L.mok_moe_forward(arr, 128, 128, pack, None, None, ctypes.byref(p), 8, ctypes.byref(o), 256, 1 << 30,
                           arr, None)
    assert rc == mok.MOK_ERR_INVALID_ARG and "minibatch" in mok.last_error()
    rc = L.mok_moe_forward(arr, 128, 128, pack, None, None, ctypes.byref(p), 256, ctypes.byref(o), 256, 1, arr, None)
    assert rc == mok.MOK_ERR_WORKSPACE
    # the persistent MXFP8 workspace holds E4M3 rows and h plus their scale planes
    need_mx = L.mok_forward_workspace_bytes(16, 128, 128, 8, 2, 256, ctypes.byref(o))
    need_bf = L.mok_forward_workspace_bytes(16, 128, 128, 8, 2, 256,
                                            ctypes.byref(mok.fwd_opts(mode=mok.MOK_MODE_PERSISTENT)))
    assert 0 < need_mx < need_bf
    o = mok.fwd_opts(mode=mok.MOK_MODE_STAGED, mxfp8=True)
    holed = mok.MxWeights(4096, 4096, 4096, 0, 4096, 4096)
    rc = L.mok_moe_forward(arr, 128, 128, ctypes.cast(ctypes.byref(holed), ctypes.c_void_p), None, None,
                           ctypes.byref(p), 0, ctypes.byref(o), 256, 1 << 30, arr, None)
    assert rc == mok.MOK_ERR_INVALID_ARG and "NULL" in mok.last_error()
    rc = L.mok_moe_forward(arr, 128, 128, None, None, None, ctypes.byref(p), 0, ctypes.byref(o), 256, 1 << 30,
                           arr, None)
    assert rc == mok.MOK_ERR_INVALID_ARG


def test_get_status_argument_checks():
    L = mok.lib()
    rc = L.mok_get_status(None, 0, None, None)
    assert rc == mok.MOK_ERR_INVALID_ARG


def test_mxfp8_step_entry_points_reject_bad_arguments():
    """The MXFP8 gather and FFN check shapes, pointers and alignment on the
    host, before any device work."""
    p = mok.PlanT(16, 8, 2, 2)
    for name in ("counts", "offsets", "sched_src_rank", "sched_src_index", "row_slot", "pos", "topk_idx", "gates"):
        setattr(p, name, 4096)
    L = mok.lib()
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    # H must be a multiple of 128 for the quantising gather
    assert L.mok_gather_mxfp8(arr, 192, ctypes.byref(p), 4096, 8192, None) == mok.MOK_ERR_UNSUPPORTED
    assert L.mok_gather_mxfp8(arr, 256, ctypes.byref(p), None, 8192, None) == mok.MOK_ERR_INVALID_ARG
    assert L.mok_gather_mxfp8(arr, 256, ctypes.byref(p), 4100, 8192, None) == mok.MOK_ERR_UNSUPPORTED
    assert L.mok_mxfp8_scale_rows(10) == 16 and L.mok_mxfp8_scale_rows(12) == 16 and L.mok_mxfp8_scale_rows(13) == 20
    need = L.mok_expert_ffn_mxfp8_workspace_bytes(32, 256, 8)
    assert need > 0
    w = mok.MxWeights(4096, 4096, 4096, 4096, 4096, 0)
    rc = L.mok_expert_ffn_mxfp8(4096, 8192, 256, 256, ctypes.cast(ctypes.byref(w), ctypes.c_void_p), ctypes.byref(p),
                                256, need, 4096, None)
    assert rc == mok.MOK_ERR_INVALID_ARG and "NULL" in mok.last_error()
    rc = L.mok_expert_ffn_mxfp8(4096, 8192, 256, 256, None, ctypes.byref(p), 256, need - 1, 4096, None)
    assert rc == mok.MOK_ERR_WORKSPACE


def test_binding_checks_shard_count_before_calling_the_library():
    """The library reads R pointers from each shard array, so the binding
    rejects a list of another length before any call (no device needed)."""
    import torch

    p = mok.Plan(mok.PlanT(16, 8, 2, 2), torch.empty(256, dtype=torch.uint8))
    one = [torch.empty(8, 128, dtype=torch.bfloat16)]          # R = 2 expected
    w = torch.empty(8, 128, 128, dtype=torch.bfloat16)
    pack = tuple(torch.empty(8, 128, 128, dtype=torch.uint8) for _ in range(6))
    out = torch.empty(32, 128, dtype=torch.float32)
    with pytest.raises(AssertionError):
        mok.moe_forward(one, w, w, w, p)
    with pytest.raises(AssertionError):
        mok.moe_forward_mxfp8(one, pack, p)
    with pytest.raises(AssertionError):
        mok.gather(one, p)
    with pytest.raises(AssertionError):
        mok.gather_mxfp8(one, p)
    with pytest.raises(AssertionError):
        mok.combine(out, p, one)


def test_two_wave_rows_reproduces_the_pages_minibatch():
    """The library's two-wave formula gives the pages' 2368 rows at hidden
    7168 / intermediate 2048 on 148 SMs with the fixture's tiling, and the
    kernel's own chunk units (256 rows x 128 features, or 256 with M-tile
    pairs) on the 132 GEMM CTAs of the default persistent split."""
    import json

    with open(os.path.join(ROOT, "tests", "golden", "two_wave_minibatch.json")) as f:
        g = json.load(f)
    L = mok.lib()
    assert L.mok_two_wave_rows(g["I"], g["sms"], g["tile_rows"], g["tile_cols"]) == g["minibatch_min"]
    assert L.mok_two_wave_rows(2048, 148, 128, 256) == 2368
    assert L.mok_two_wave_rows(2048, 132, 256, 128) == 2112
    assert L.mok_two_wave_rows(2048, 132, 256, 256) == 4224
    assert L.mok_two_wave_rows(14336, 148, 256, 128) == 339         # rounded up
    assert L.mok_two_wave_rows(0, 148, 128, 256) == 0
    assert L.mok_two_wave_rows(2048, -1, 128, 256) == 0


def test_host_batches_reject_null_host_pointers_before_any_copy():
    L = mok.lib()
    opts = mok.fwd_opts(mode=mok.MOK_MODE_STAGED)
    need = L.mok_forward_host_batches_workspace_bytes(64, 128, 128, 8, 2, 64, ctypes.byref(opts))
    assert need > L.mok_forward_host_workspace_bytes(64, 128, 128, 8, 2, 64, ctypes.byref(opts)) > 0
    arr = (ctypes.c_void_p * 2)(4096, None)
    good = (ctypes.c_void_p * 2)(4096, 8192)
    rc = L.mok_moe_forward_host_batches(2, good, arr, good, 64, 128, 128, 8, 2, 2, 1, 1, 1, 64, ctypes.byref(opts),
                                        4096, need, None)
    assert rc == mok.MOK_ERR_INVALID_ARG and "NULL" in mok.last_error()
    assert L.mok_moe_forward_host_batches(0, None, None, None, 64, 128, 128, 8, 2, 2, 1, 1, 1, 64, None, None, 0,
                                          None) == mok.MOK_OK
    rc = L.mok_moe_forward_host_batches(2, good, good, good, 63, 128, 128, 8, 2, 2, 1, 1, 1, 64, ctypes.byref(opts),
                                        4096, need, None)
    assert rc == mok.MOK_ERR_INVALID_ARG


def test_router_entry_points_check_arguments():
    L = mok.lib()
    assert L.mok_router_weights_bytes(7168, 384) == 384 * 7168 * 2
    assert L.mok_router_weights_bytes(512, 8) == 64 * 512 * 2           # experts padded to 64 rows (two halves)
    assert L.mok_router_weights_bytes(512, 385) == 0                      # above MOK_ROUTER_MAX_EXPERTS
    assert L.mok_router_prepare(4096, 512, 385, 4096, 8192, None) == mok.MOK_ERR_UNSUPPORTED
    assert L.mok_router_prepare(4096, 500, 8, 4096, 8192, None) == mok.MOK_ERR_UNSUPPORTED   # H % 64
    assert L.mok_router_prepare(None, 512, 8, 4096, 8192, None) == mok.MOK_ERR_INVALID_ARG
    assert L.mok_router_prepare(4096, 512, 8, 4097, 8192, None) == mok.MOK_ERR_UNSUPPORTED  # alignment
    p = mok.PlanT()
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    need = L.mok_plan_workspace_bytes(64, 8, 2)

    def call(T=64, E=8, k=2, R=2, H=128, hi=4096, lo=8192, xs=arr, ws=4096, nbytes=need):
        return L.mok_plan_router(xs, H, hi, lo, None, T, E, k, R, None, ws, nbytes, ctypes.byref(p), None)

    assert call(E=400) == mok.MOK_ERR_UNSUPPORTED
    assert call(H=96) == mok.MOK_ERR_UNSUPPORTED
    assert call(k=9) == mok.MOK_ERR_INVALID_ARG
    assert call(T=63) == mok.MOK_ERR_UNSUPPORTED
    assert call(lo=8200) == mok.MOK_ERR_UNSUPPORTED
    assert call(xs=(ctypes.c_void_p * 2)(4096, 8200)) == mok.MOK_ERR_UNSUPPORTED
    assert call(ws=4096, nbytes=need - 1) == mok.MOK_ERR_WORKSPACE


def test_forward_dispatch_warps_rules():
    """The warp layout of the persistent kernel takes 1 or 2 dispatch warps
    per CTA and no dispatch CTAs; both are checked before anything else is
    touched (the pointers here are not device memory)."""
    p = _filled_plan(16, 8, 2, 2)
    L = mok.lib()
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    for o, what in ((mok.fwd_opts(dispatch_warps=3), "dispatch_warps"),
                    (mok.fwd_opts(dispatch_warps=-1), "dispatch_warps"),
                    (mok.fwd_opts(dispatch_warps=1, dispatch_ctas=4), "exclude")):
        rc = L.mok_moe_forward(arr, 128, 128, 4096, 4096, 4096, ctypes.byref(p), 256, ctypes.byref(o), 256,
                               1 << 30, arr, None)
        assert rc == mok.MOK_ERR_INVALID_ARG and what in mok.last_error(), mok.last_error()
