"""The tie-tolerant top-k check that a router computed on the device (in
fp32, any summation order) will be held to: accepted where rounding can
flip a near-tie, exact everywhere else.  CPU only; the selections come from
the oracle and from hand-made perturbations."""
import torch

import mokgen
import oracle
from helpers import topk_within_tolerance


def _exact_and_rounded(T=256, E=64, k=8, seed=3):
    cfg = mokgen.scaled(mokgen.CONFIGS["page"], T=T, E=E, k=k, H=512, seed=seed)
    x = mokgen.tokens(cfg)
    w = mokgen.router_weight(cfg)
    exact = oracle.router_logits(x, w)
    rounded = mokgen.router_logits(cfg, x)                  # fp32, the harness's own product
    n, u = cfg.H, 2.0 ** -24
    bound = (n * u / (1 - n * u) * (x.double().abs() @ w.double().abs())).max(1).values
    return exact, rounded, 2 * bound                        # two logits, each off by <= bound


def test_fp32_selection_is_accepted():
    exact, rounded, tol = _exact_and_rounded()
    idx, _ = oracle.topk_gates(rounded, 8)
    ok, strict = topk_within_tolerance(idx, exact, tol)
    assert ok.all()
    # where the choice is unambiguous it equals the exact top-k
    want = torch.tensor([sorted(range(64), key=lambda e: (-exact[t, e].item(), e))[:8] for t in range(256)])
    assert torch.equal(idx.long()[strict], want[strict])
    assert strict.float().mean() > 0.9


def test_near_tie_swap_is_accepted_and_clear_swap_is_rejected():
    exact = torch.tensor([[5.0, 4.0, 3.0, 2.9999999, 1.0]], dtype=torch.float64)
    tol = torch.tensor([1e-6], dtype=torch.float64)
    ok, strict = topk_within_tolerance(torch.tensor([[0, 1, 3]]), exact, tol)      # 3 for 2: a near-tie
    assert ok.all() and not strict.any()
    ok, _ = topk_within_tolerance(torch.tensor([[0, 1, 4]]), exact, tol)           # 4 for 2: off by 2.0
    assert not ok.any()
    ok, _ = topk_within_tolerance(torch.tensor([[1, 0, 2]]), exact, tol)           # rank order broken
    assert not ok.any()
    ok, _ = topk_within_tolerance(torch.tensor([[0, 0, 1]]), exact, tol)           # duplicate expert
    assert not ok.any()
    ok, strict = topk_within_tolerance(torch.tensor([[0, 1, 2]]), exact, tol)
    assert ok.all() and not strict.any()          # the boundary is a near-tie, so not strict either
    ok, strict = topk_within_tolerance(torch.tensor([[0, 1]]), exact, tol)
    assert ok.all() and strict.all()
