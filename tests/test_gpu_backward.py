"""GPU parity of the layer's backward (mok_moe_backward) against the
backward oracle (fp64 chain rule of the forward definition).

Bound: every backward output is compared by relative Frobenius error <= 1e-2.
The longest rounding chain of the GPU backward has five bf16 roundings of
relative size at most 2^-9 each (the do rows, the saved a and b, the
[da | db] rows and the output itself), so 5 x 2^-9 ~ 9.8e-3 bounds the
relative error of any element to first order; the Frobenius error of
independent roundings is far smaller.  dlogits compare the same way, and
its zero pattern (unselected experts) exactly."""
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
import oracle
from helpers import rel_fro

pytestmark = pytest.mark.gpu

REL_FRO_BWD = 1e-2

CASES = {
    "tiny": mokgen.scaled(mokgen.CONFIGS["tiny"], T=128, H=256, I=128, seed=401),
    "ragged": mokgen.scaled(mokgen.CONFIGS["tiny"], T=300, H=256, I=256, E=6, k=3, R=3, seed=402),
    "many_experts": mokgen.scaled(mokgen.CONFIGS["tiny"], T=192, H=384, I=128, E=24, k=4, R=2, seed=403),
    "wide": mokgen.scaled(mokgen.CONFIGS["tiny"], T=64, H=1024, I=512, E=4, k=2, R=2, seed=404),
    # experts of about 640 rows: the weight-gradient kernel reloads the A
    # tile for every N tile (more K stages than its resident slots)
    "tall": mokgen.scaled(mokgen.CONFIGS["tiny"], T=640, H=256, I=256, E=2, k=2, R=2, seed=406),
}


def _run(cfg, empty_experts=()):
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    if empty_experts:
        logits = logits.clone()
        logits[:, list(empty_experts)] -= 100.0
    wg, wu, wd = mokgen.all_expert_weights(cfg)
    dy = mokgen.normal(cfg.seed, 99, (cfg.T, cfg.H), 1.0)
    dwg_, dwu_, dwd_ = (w.cuda() for w in (wg, wu, wd))
    dx_ = x.cuda()
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    opts = mok.fwd_opts(mode=mok.MOK_MODE_STAGED, save_for_backward=True)
    ys, fws = mok.moe_forward(mok.shards(dx_, cfg.R), dwg_, dwu_, dwd_, p, 0, opts)
    assert mok.get_status(fws) == mok.MOK_OK
    dys = mok.shards(dy.cuda(), cfg.R)
    dxs, (gwg, gwu, gwd), dl, bws = mok.moe_backward(dys, dwg_, dwu_, dwd_, p, fws)
    assert mok.get_status(bws) == mok.MOK_OK
    got = dict(dx=torch.cat([s.cpu() for s in dxs]), dwg=gwg.cpu(), dwu=gwu.cpu(), dwd=gwd.cpu(), dlogits=dl.cpu())
    want = oracle.moe_backward(x, logits, wg, wu, wd, dy.double(), cfg.k, cfg.R)
    y_fwd = torch.cat([s.cpu() for s in ys])
    return got, want, y_fwd, p


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    got, want, _, _ = _run(CASES[name])
    for key in ("dx", "dwg", "dwu", "dwd", "dlogits"):
        err = rel_fro(got[key], want[key])
        assert err <= REL_FRO_BWD, f"{name} {key}: relative Frobenius {err:.3e}"
    # unselected logits get exactly zero gradient
    assert torch.equal(got["dlogits"] == 0, want["dlogits"] == 0)


def test_backward_experts_without_rows_get_zero_gradients():
    cfg = mokgen.scaled(mokgen.CONFIGS["tiny"], T=128, H=256, I=128, E=8, k=2, seed=405)
    got, want, _, p = _run(cfg, empty_experts=(1, 6))
    counts = p.counts().cpu()
    assert counts[1] == 0 and counts[6] == 0
    for key in ("dwg", "dwu", "dwd"):
        assert (got[key][[1, 6]] == 0).all()
        err = rel_fro(got[key], want[key])
        assert err <= REL_FRO_BWD, f"{key}: relative Frobenius {err:.3e}"


def test_save_for_backward_keeps_the_forward_bits():
    """Saving a and b changes nothing in the forward's result."""
    cfg = CASES["ragged"]
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    w = [t.cuda() for t in mokgen.all_expert_weights(cfg)]
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    xs = mok.shards(x.cuda(), cfg.R)
    y1, _ = mok.moe_forward(xs, *w, p, 0, mok.fwd_opts(mode=mok.MOK_MODE_STAGED))
    y2, _ = mok.moe_forward(xs, *w, p, 0, mok.fwd_opts(mode=mok.MOK_MODE_STAGED, save_for_backward=True))
    assert torch.equal(torch.cat(y1), torch.cat(y2))


@pytest.mark.parametrize("name", ["wide", "tall"])
def test_backward_cta_pairs_are_exact(name, monkeypatch):
    """The dh and dx phases on CTA pairs (one M = 256 MMA over two SMs) give
    the same bits as on single CTAs; the weight gradients do not depend on
    the setting at all."""
    got = {}
    for cta_pair in ("0", "1"):
        monkeypatch.setenv("MOK_GEMM_CTA_PAIR", cta_pair)
        got[cta_pair], _, _, _ = _run(CASES[name])
    for key in ("dx", "dwg", "dwu", "dwd", "dlogits"):
        assert torch.equal(got["0"][key], got["1"][key]), key
