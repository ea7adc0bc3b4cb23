"""mok_plan_noalloc: the plan for callers that cannot allocate device memory
(code recording a stream capture, allocator-less runtimes, hooks that must
not touch the allocator).  It keeps its scratch in a library-owned device
array; its results must equal mok_plan's.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.  It must pass alone in a fresh
process and after the other tests.
"""
import ctypes

import pytest
import torch

import combine_device_top_b200 as mok
import mokgen

pytestmark = pytest.mark.gpu


def _noalloc_plan(logits: torch.Tensor, k: int, R: int):
    T, E = logits.shape
    dev = logits.device
    out = {
        "counts": torch.full((E,), -1, dtype=torch.int32, device=dev),
        "offsets": torch.full((E + 1,), -1, dtype=torch.int32, device=dev),
        "src_rank": torch.full((T * k,), -1, dtype=torch.int32, device=dev),
        "src_index": torch.full((T * k,), -1, dtype=torch.int32, device=dev),
        "row_slot": torch.full((T * k,), -1, dtype=torch.int32, device=dev),
        "pos": torch.full((T * k,), -1, dtype=torch.int32, device=dev),
        "topk_idx": torch.full((T * k,), -1, dtype=torch.int32, device=dev),
        "gates": torch.full((T * k,), float("nan"), dtype=torch.float32, device=dev),
    }
    order = ("counts", "offsets", "src_rank", "src_index", "row_slot", "pos", "topk_idx", "gates")
    rc = mok.lib().mok_plan_noalloc(ctypes.c_void_p(logits.data_ptr()), T, E, k, R,
                                    *(ctypes.c_void_p(out[n].data_ptr()) for n in order),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == mok.MOK_OK, mok.last_error()
    return out


def _compare(logits: torch.Tensor, k: int, R: int):
    got = _noalloc_plan(logits, k, R)
    ref = mok.plan(logits, k, R)           # the existing entry point, with a workspace
    torch.cuda.synchronize()
    assert torch.equal(got["counts"], ref.counts())
    assert torch.equal(got["offsets"], ref.offsets())
    assert torch.equal(got["src_rank"], ref.src_rank())
    assert torch.equal(got["src_index"], ref.src_index())
    assert torch.equal(got["row_slot"], ref.row_slot())
    assert torch.equal(got["pos"], ref.pos())
    assert torch.equal(got["topk_idx"], ref.topk_idx().reshape(-1))
    # same tolerance as the plan parity tests (the kernels are the same, so
    # the gates are in fact identical)
    assert (got["gates"] - ref.gates().reshape(-1)).abs().max().item() <= 2e-6


def test_plan_noalloc_matches_plan_on_two_calls_in_a_row():
    page = mokgen.CONFIGS["page"]
    zipf = mokgen.CONFIGS["zipf"]
    # two calls back to back on different shapes: the second must not see
    # anything the first left in the shared scratch array
    _compare(mokgen.router_logits(page).cuda(), page.k, page.R)
    _compare(mokgen.router_logits(zipf).cuda(), zipf.k, zipf.R)
    # and once more on a tie-heavy, ragged shape
    ties = mokgen.small_ints(9, 4242, (1000, 64), 3).cuda()
    _compare(ties, 4, 8)


def test_plan_noalloc_rejects_shapes_beyond_its_scratch():
    T, E, k = 1 << 17, 1024, 8                 # needs ~4.6 MiB of scratch
    logits = torch.zeros((1, 1), dtype=torch.float32, device="cuda")
    dummy = ctypes.c_void_p(logits.data_ptr())
    rc = mok.lib().mok_plan_noalloc(dummy, T, E, k, 8, *([dummy] * 8), None)
    assert rc == mok.MOK_ERR_UNSUPPORTED
    assert "MOK_PLAN_NOALLOC_SCRATCH_BYTES" in mok.last_error()


def test_plan_noalloc_leaves_device_memory_untouched():
    """The call allocates nothing: device free memory is the same before and
    after its first call on a new shape.  One call on another shape comes
    first: the first call in a process loads the code module that holds the
    static scratch array (its fixed 2 MiB, held until exit, as documented).
    mok_plan then runs on the new shape, so its kernels' code is loaded too
    (lazy module loading takes device memory for code, which is not an
    allocation of this entry point)."""
    _noalloc_plan(mokgen.small_ints(11, 76, (64, 16), 5).cuda(), 2, 2)
    logits = mokgen.small_ints(11, 77, (777, 96), 5).cuda()
    k, R = 6, 7
    mok.plan(logits, k, R)
    T, E = logits.shape
    outs = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1, T * k, T * k, T * k, T * k, T * k)]
    gates = torch.empty(T * k, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    rc = mok.lib().mok_plan_noalloc(ctypes.c_void_p(logits.data_ptr()), T, E, k, R,
                                    *(ctypes.c_void_p(t.data_ptr()) for t in outs), ctypes.c_void_p(gates.data_ptr()),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == mok.MOK_OK, mok.last_error()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
