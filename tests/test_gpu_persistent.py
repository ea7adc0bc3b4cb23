"""GPU tests of the SM-partitioned persistent forward (ring token buffer,
minibatches, device counters): bit-identical to the staged path at every
minibatch size, ring size and dispatch/GEMM split, matching the oracle, and
reporting a timeout cleanly when its waits are given a tiny bound."""
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
from helpers import Case, assert_bf16_close
from test_gpu_forward import FFN_CASES

pytestmark = pytest.mark.gpu

STAGED = mok.MOK_MODE_STAGED
PERSIST = mok.MOK_MODE_PERSISTENT


def _run(case: Case, mode, minibatch, **kw):
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    opts = mok.fwd_opts(mode=mode, **kw)
    ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, minibatch, opts)
    code = mok.get_status(ws)
    return torch.cat([s for s in ys]), code, ws


@pytest.mark.parametrize("name", list(FFN_CASES))
def test_persistent_matches_staged_and_oracle(name):
    case = Case(FFN_CASES[name])
    y_s, code_s, _ = _run(case, STAGED, 0)
    y_p, code_p, _ = _run(case, PERSIST, 64)
    assert code_s == mok.MOK_OK and code_p == mok.MOK_OK
    assert torch.equal(y_p, y_s)
    assert_bf16_close(y_p.cpu(), case.oracle_y(), name)


@pytest.mark.parametrize("minibatch,ring,dispatch", [(16, 0, 4), (256, 0, 16), (600, 1300, 8),
                                                     (2560, 0, 16), (4096, 8192, 2)])
def test_persistent_invariant_to_minibatch_ring_and_split(minibatch, ring, dispatch):
    cfg = mokgen.scaled(mokgen.CONFIGS["page"], E=48, T=1024)
    case = Case(cfg)
    y_s, _, _ = _run(case, STAGED, 0)
    y_p, code, _ = _run(case, PERSIST, minibatch, ring_slots=ring, dispatch_ctas=dispatch)
    assert code == mok.MOK_OK
    assert torch.equal(y_p, y_s)


@pytest.mark.parametrize("minibatch,ring,dwarps,gemm", [(16, 0, 1, 0), (256, 0, 2, 0), (600, 1300, 2, 0),
                                                        (2560, 0, 2, 0), (128, 0, 1, 5), (4096, 8192, 1, 0)])
def test_persistent_warp_layout_equals_staged(minibatch, ring, dwarps, gemm):
    """The warp layout (no dispatch CTAs: every CTA runs the GEMM roles and
    1 or 2 dispatch warps that claim rows 16 at a time) computes the staged
    path's bits at every minibatch size, ring size and grid."""
    cfg = mokgen.scaled(mokgen.CONFIGS["page"], E=48, T=1024)
    case = Case(cfg)
    y_s, _, _ = _run(case, STAGED, 0)
    y_p, code, _ = _run(case, PERSIST, minibatch, ring_slots=ring, dispatch_warps=dwarps, gemm_ctas=gemm)
    assert code == mok.MOK_OK, mok.last_error()
    assert torch.equal(y_p, y_s)


def test_persistent_small_gemm_grid():
    case = Case(FFN_CASES["multi_chunk"])
    y_s, _, _ = _run(case, STAGED, 0)
    y_p, code, _ = _run(case, PERSIST, 128, dispatch_ctas=3, gemm_ctas=5)
    assert code == mok.MOK_OK
    assert torch.equal(y_p, y_s)


def test_persistent_wait_timeout_reports_status_and_recovers():
    """Every device wait is bounded: with a 1 ns bound the waits give up, the
    kernel leaves cleanly with MOK_ERR_TIMEOUT in the status word, and the
    next forward on the same workspace is correct."""
    case = Case(FFN_CASES["tiny"])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    y_s, _, _ = _run(case, STAGED, 0)
    for dwarps in (0, 2):  # dispatch CTAs, then the warp layout
        bad = mok.fwd_opts(mode=PERSIST, timeout_ns=1, dispatch_warps=dwarps)
        ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, 64, bad)
        assert mok.get_status(ws) == mok.MOK_ERR_TIMEOUT
        assert "status" in mok.last_error()
        good = mok.fwd_opts(mode=PERSIST, dispatch_warps=dwarps)
        ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, 64, good, ws=ws)
        assert mok.get_status(ws) == mok.MOK_OK
        assert torch.equal(torch.cat(ys), y_s)


@pytest.mark.parametrize("minibatch,ring,dispatch", [(64, 256, 4), (100, 320, 2), (16, 256, 8), (64, 256, -1),
                                                     (16, 256, -2)])
def test_persistent_ring_wraps_on_a_small_shape(minibatch, ring, dispatch):
    """Experts far taller than the ring half (one takes most tokens): every
    expert is split across minibatches, the ring wraps many times and the
    dispatch side throttles on the GEMM side's progress.  Every token is
    checked against the oracle, and the result equals the staged path's."""
    cfg = mokgen.scaled(mokgen.CONFIGS["tiny"], T=1024, H=256, I=128, E=6, k=2, R=4, seed=111)
    case = Case(cfg)
    logits = case.logits.clone()
    logits[:, 2] += 4.0                          # expert 2 is in almost every token's top-2
    case.logits, case.dlogits = logits, logits.cuda()
    y_s, code_s, _ = _run(case, STAGED, 0)
    # dispatch < 0: the warp layout with -dispatch dispatch warps per CTA
    split = dict(dispatch_ctas=dispatch) if dispatch > 0 else dict(dispatch_warps=-dispatch)
    y_p, code_p, _ = _run(case, PERSIST, minibatch, ring_slots=ring, **split)
    assert code_s == mok.MOK_OK and code_p == mok.MOK_OK
    counts = mok.plan(case.dlogits, cfg.k, cfg.R).counts().cpu()
    assert counts.max().item() > 4 * (ring // 2)  # the tallest expert spans several ring halves
    assert torch.equal(y_p, y_s)
    assert_bf16_close(y_p.cpu(), case.oracle_y(), f"ring {ring}")


@pytest.mark.parametrize("name,minibatch", [("page", 0), ("page", 2560), ("zipf", 0), ("zipf", 2560)])
def test_minibatches_hold_two_waves_of_gemm_units(name, minibatch):
    """The device-built minibatches of the page and zipf shapes (bench.py's
    ring) hold at least two full waves of gate/up units for the GEMM CTAs
    (the last minibatch takes what is left), at least `minibatch` rows, at
    most half the ring, and start at expert boundaries unless an expert is
    taller than the ring half."""
    cfg = mokgen.CONFIGS[name]
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    opts = mok.fwd_opts(mode=PERSIST, ring_slots=cfg.ring_slots, dispatch_ctas=8)
    row0, units = mok.minibatch_bounds(p, cfg.H, cfg.I, minibatch, opts)
    gemm_ctas = torch.cuda.get_device_properties(0).multi_processor_count - 8
    ns, cap = cfg.slots, cfg.ring_slots // 2
    bounds = row0 + [ns]
    offsets = set(p.offsets().cpu().tolist())
    assert row0[0] == 0 and len(row0) >= 2
    for b in range(len(row0)):
        rows = bounds[b + 1] - bounds[b]
        assert rows <= cap
        if b < len(row0) - 1:
            assert units[b] >= 2 * gemm_ctas or rows == cap, (b, units[b], rows)
            assert rows >= minibatch or rows == cap
            assert bounds[b + 1] in offsets or rows == cap
