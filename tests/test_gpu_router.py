"""GPU parity of the router projection fused with the top-k (mok_plan_router)
against the oracle's router (fp64) and the plan computed from given logits.

The device computes x (w_hi + w_lo) with fp32 accumulation, so its logits
differ from the exact projection within a rounding bound, and near-ties
within that bound may be ordered either way: the selection is checked with
the tie-tolerant rule (helpers.topk_within_tolerance), and every token whose
deciding gaps all exceed the bound must select exactly the oracle's experts.
Given its own logits, the router's top-k, gates and schedule must equal
mok_plan's on those logits bit for bit."""
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
import oracle
from helpers import topk_within_tolerance

pytestmark = pytest.mark.gpu


def _router_inputs(cfg):
    x = mokgen.tokens(cfg)
    w = mokgen.router_weight(cfg)
    prior = mokgen.zipf_log_prior(cfg.E, cfg.zipf_s) if cfg.zipf_s else None
    return x, w, prior


def test_router_weight_split_is_exact():
    """w_hi = bf16(W_r), w_lo = bf16(W_r - w_hi), expert-major, zero padding rows."""
    cfg = mokgen.scaled(mokgen.CONFIGS["tiny"], H=256, E=200)
    w = mokgen.router_weight(cfg)
    w[0, :4] = torch.tensor([0.0, -0.0, 1e-30, -3.0e38])
    hi, lo = mok.router_prepare(w.cuda())
    hi, lo = hi.cpu(), lo.cpu()
    assert hi.shape == (256, 256)
    want_hi = w.t().contiguous().to(torch.bfloat16)
    want_lo = (w.t() - want_hi.float()).to(torch.bfloat16)
    assert torch.equal(hi[:200].view(torch.int16), want_hi.view(torch.int16))
    assert torch.equal(lo[:200].view(torch.int16), want_lo.view(torch.int16))
    assert (hi[200:] == 0).all() and (lo[200:] == 0).all()


CASES = {
    "tiny": mokgen.CONFIGS["tiny"],
    "ragged": mokgen.scaled(mokgen.CONFIGS["tiny"], T=300, H=192, E=40, k=5, R=3, seed=301),
    "k32": mokgen.scaled(mokgen.CONFIGS["tiny"], T=130, H=128, E=64, k=32, R=2, seed=302),
    "mixtral": mokgen.CONFIGS["mixtral"],
    "page": mokgen.CONFIGS["page"],
    "zipf": mokgen.CONFIGS["zipf"],
}


@pytest.mark.parametrize("name", list(CASES))
def test_router_plan_matches_oracle(name):
    cfg = CASES[name]
    x, w, prior = _router_inputs(cfg)
    hi, lo = mok.router_prepare(w.cuda())
    dx = x.cuda()
    logits = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device="cuda")
    p = mok.plan_router(mok.shards(dx, cfg.R), hi, lo, cfg.E, cfg.k, prior.cuda() if prior is not None else None,
                        logits_out=logits)
    assert mok.get_status(p.ws) == mok.MOK_OK
    got = logits.cpu().double()
    exact = oracle.router_logits(x, w, prior)
    # the rounding bound of x (w_hi + w_lo) with fp32 accumulation: the split
    # leaves |W_r - w_hi - w_lo| <= 2^-17 |W_r|; each MMA adds a K = 16
    # product sum (exact bf16 products) to the fp32 accumulator, H / 16
    # additions of at most 2^-23 of sum |x w| each (allowing round toward
    # zero), doubled for margin
    mag = x.double().abs() @ w.double().abs()
    bound = (2.0 ** -17 + (cfg.H / 16 + 16) * 2.0 ** -22) * mag + 1e-6
    assert ((got - exact).abs() <= bound).all(), ((got - exact).abs() / bound).max().item()
    # selection: correct up to near-ties inside the bound; exact where no gap is that close
    tol = bound.max(dim=1).values * 2
    idx = p.topk_idx().cpu()
    ok, strict = topk_within_tolerance(idx, exact, tol)
    assert ok.all(), int((~ok).sum())
    want_idx, want_g = oracle.topk_gates(exact.float(), cfg.k)
    assert torch.equal(idx[strict], want_idx[strict])
    assert strict.float().mean().item() > 0.1      # the exact-selection check covers real tokens
    # given its own logits, the router plans exactly what mok_plan plans
    q = mok.plan(logits, cfg.k, cfg.R)
    for f in ("topk_idx", "counts", "offsets", "src_rank", "src_index", "row_slot", "pos"):
        assert torch.equal(getattr(p, f)().cpu(), getattr(q, f)().cpu()), f
    assert torch.equal(p.gates().cpu(), q.gates().cpu())
    # and the schedule is the oracle's schedule of that selection
    sch = oracle.schedule(idx, cfg.E, cfg.R)
    for f in ("counts", "offsets", "src_rank", "src_index", "row_slot", "pos"):
        assert torch.equal(getattr(p, f)().cpu(), sch[f]), f


def test_router_plan_without_logits_output_and_forward():
    """No logits array: same plan; the forward on it equals the forward on
    mok_plan's plan of the same logits."""
    cfg = mokgen.scaled(mokgen.CONFIGS["tiny"], seed=303)
    x, w, prior = _router_inputs(cfg)
    hi, lo = mok.router_prepare(w.cuda())
    dx = x.cuda()
    logits = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device="cuda")
    p1 = mok.plan_router(mok.shards(dx, cfg.R), hi, lo, cfg.E, cfg.k, logits_out=logits)
    p2 = mok.plan_router(mok.shards(dx, cfg.R), hi, lo, cfg.E, cfg.k)
    assert torch.equal(p1.topk_idx().cpu(), p2.topk_idx().cpu())
    assert torch.equal(p1.gates().cpu(), p2.gates().cpu())
    wg, wu, wd = (t.cuda() for t in mokgen.all_expert_weights(cfg))
    q = mok.plan(logits, cfg.k, cfg.R)
    opts = mok.fwd_opts(mode=mok.MOK_MODE_STAGED)
    y1, _ = mok.moe_forward(mok.shards(dx, cfg.R), wg, wu, wd, p2, 0, opts)
    y2, _ = mok.moe_forward(mok.shards(dx, cfg.R), wg, wu, wd, q, 0, opts)
    assert torch.equal(torch.cat(y1), torch.cat(y2))
