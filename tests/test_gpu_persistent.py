"""GPU tests of the SM-partitioned persistent forward (ring token buffer,
minibatches, device counters): bit-identical to the staged path at every
minibatch size, ring size and dispatch/GEMM split, matching the oracle, and
reporting a timeout cleanly when its waits are given a tiny bound."""
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
from helpers import Case, assert_bf16_close, sample_tokens
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
    bad = mok.fwd_opts(mode=PERSIST, timeout_ns=1)
    ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, 64, bad)
    assert mok.get_status(ws) == mok.MOK_ERR_TIMEOUT
    assert "status" in mok.last_error()
    good = mok.fwd_opts(mode=PERSIST)
    ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, 64, good, ws=ws)
    assert mok.get_status(ws) == mok.MOK_OK
    y_s, _, _ = _run(case, STAGED, 0)
    assert torch.equal(torch.cat(ys), y_s)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["page", "zipf"])
def test_persistent_full_size(name):
    """Full size in the launch configuration bench.py times: bit-identical to
    the staged path; sampled tokens against the oracle."""
    cfg = mokgen.CONFIGS[name]
    case = Case(cfg, weights_on_host=False)
    y_s, code_s, ws = _run(case, STAGED, 0)
    del ws
    torch.cuda.empty_cache()
    y_p, code_p, _ = _run(case, PERSIST, cfg.minibatch, ring_slots=cfg.ring_slots)
    assert code_s == mok.MOK_OK and code_p == mok.MOK_OK
    assert torch.equal(y_p, y_s)
    ids = sample_tokens(cfg.T, 6, seed=cfg.seed + 7)
    assert_bf16_close(y_p[ids].cpu(), case.oracle_y(ids), name)
