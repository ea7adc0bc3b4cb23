"""Full-size configurations, in the launch configuration bench.py times.

bf16 path (Mixtral-shaped, page and zipf shapes): every token of y is
checked against the oracle, and the persistent SM-partitioned kernel (the
configuration's minibatch and ring; dispatch CTAs, and dispatch warps in
every CTA) must produce the staged path's bits.
MXFP8 page shape: every row is computed on the GPU, the persistent kernel
is bit-identical to staged, and a token set that covers every expert (each
expert's rows are checked through at least one of its tokens) is compared
with the oracle's emulation of the quantisation.
"""
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
import oracle
from helpers import Case, assert_bf16_close

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

STAGED = mok.MOK_MODE_STAGED
PERSIST = mok.MOK_MODE_PERSISTENT
REL_FRO_MX = 2e-2


def _forward(case: Case, mode, minibatch, ring_slots=0, dispatch_warps=0):
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, minibatch,
                             mok.fwd_opts(mode=mode, ring_slots=ring_slots, dispatch_warps=dispatch_warps))
    code = mok.get_status(ws)
    y = torch.cat([s.cpu() for s in ys])
    del ws, ys
    torch.cuda.empty_cache()
    return y, code


def _oracle_all_tokens(case: Case, block: int = 4096) -> torch.Tensor:
    """The oracle's y for every token, in blocks of tokens (one expert's
    weights are regenerated per block, so the host never holds them all)."""
    cfg = case.cfg
    out = []
    for t0 in range(0, cfg.T, block):
        ids = list(range(t0, min(cfg.T, t0 + block)))
        y, _, _ = oracle.forward_tokens(cfg, case.x, case.logits, ids, case.weight_fn)
        out.append(y)
    return torch.cat(out)


@pytest.mark.parametrize("name", ["mixtral", "page", "zipf"])
def test_forward_full_size_every_token(name):
    cfg = mokgen.CONFIGS[name]
    case = Case(cfg, weights_on_host=False)
    y, code = _forward(case, STAGED, 0)
    assert code == mok.MOK_OK
    assert torch.isfinite(y.float()).all()
    y_p, code_p = _forward(case, PERSIST, cfg.minibatch, cfg.ring_slots)
    assert code_p == mok.MOK_OK
    assert torch.equal(y_p, y)
    y_w, code_w = _forward(case, PERSIST, cfg.minibatch, cfg.ring_slots, dispatch_warps=2)
    assert code_w == mok.MOK_OK
    assert torch.equal(y_w, y)
    want = _oracle_all_tokens(case)
    assert_bf16_close(y, want, name)


def _covering_tokens(topk_idx: torch.Tensor, E: int) -> list[int]:
    """Tokens such that every expert with rows is selected by at least one
    of them: for each expert not yet covered, its first token."""
    covered = torch.zeros(E, dtype=torch.bool)
    ids = []
    for e in range(E):
        if covered[e]:
            continue
        hit = (topk_idx == e).any(1).nonzero().view(-1)
        if hit.numel() == 0:
            continue
        t = int(hit[0])
        ids.append(t)
        covered[topk_idx[t].long()] = True
    return sorted(ids)


def _mx_oracle_tokens(cfg, x, logits, ids):
    """Oracle y (MXFP8 emulation) for the tokens `ids`, one oracle call per expert."""
    idx, g = oracle.topk_gates(logits[ids], cfg.k)
    o_slot = torch.zeros((len(ids), cfg.k, cfg.H), dtype=torch.float64)
    need = {}
    for a in range(len(ids)):
        for j in range(cfg.k):
            need.setdefault(int(idx[a, j]), []).append((a, j))
    for e, uses in sorted(need.items()):
        rows = torch.stack([x[ids[a]] for a, _ in uses])
        o = oracle.mxfp8_expert_ffn(rows, *mokgen.expert_weights(cfg, e))
        for r, (a, j) in enumerate(uses):
            o_slot[a, j] = o[r]
    return oracle.combine(o_slot, g)


def test_mxfp8_full_size_covering_every_expert():
    cfg = mokgen.CONFIGS["page_mxfp8"]
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    wg, wu, wd = mokgen.upload_expert_weights(cfg, "cuda")
    pack = (*mok.quantize_weights_mxfp8(wg), *mok.quantize_weights_mxfp8(wu), *mok.quantize_weights_mxfp8(wd))
    del wg, wu, wd
    torch.cuda.empty_cache()
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    xs = mok.shards(x.cuda(), cfg.R)
    ys, ws = mok.moe_forward_mxfp8(xs, pack, p)
    assert mok.get_status(ws) == mok.MOK_OK
    y = torch.cat([s.cpu() for s in ys])
    del ws
    opts = mok.fwd_opts(mode=PERSIST, mxfp8=True, ring_slots=cfg.ring_slots)
    ys_p, ws_p = mok.moe_forward_mxfp8(xs, pack, p, minibatch=cfg.minibatch, opts=opts)
    assert mok.get_status(ws_p) == mok.MOK_OK
    assert torch.equal(torch.cat([s.cpu() for s in ys_p]), y)
    del ws_p
    topk = p.topk_idx().cpu()
    ids = _covering_tokens(topk, cfg.E)
    assert set(topk[ids].view(-1).tolist()) == set(topk.view(-1).tolist())
    want = _mx_oracle_tokens(cfg, x, logits, ids)
    got = y[ids].double()
    rel = (torch.linalg.norm(got - want) / torch.linalg.norm(want)).item()
    assert rel <= REL_FRO_MX, rel
    # and token by token (each token's own relative error)
    per = torch.linalg.norm(got - want, dim=1) / torch.linalg.norm(want, dim=1)
    assert per.max().item() <= 2 * REL_FRO_MX, per.max().item()
