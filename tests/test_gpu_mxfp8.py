"""MXFP8 on the GPU: quantiser bytes and scales bit-exact against the
oracle's emulation of the OCP MX definition, and the MXFP8 forward layer
against the emulated oracle (relative Frobenius <= 2e-2)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
import oracle

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _oracle_quant(v: np.ndarray):
    """Blocks of 32 consecutive values -> (bytes, scales) from the oracle."""
    L = oracle.lib()
    v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    nb = v.size // 32
    q = np.zeros(v.size, np.uint8)
    s = np.zeros(nb, np.uint8)
    assert L.oracle_mxfp8_quantize(v.ctypes.data, nb, q.ctypes.data, s.ctypes.data) == 0
    return q, s


def _spread(rows, K, seed):
    """bf16 rows with block magnitudes spread over many binades, zeros and ties."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, K, generator=g)
    mag = torch.pow(2.0, torch.randint(-40, 40, (rows, K // 32), generator=g).float())
    x = x * mag.repeat_interleave(32, dim=1)
    x[0, :32] = 0.0
    x[1, :32] = -0.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,K", [(64, 256), (37, 7168), (5, 32)])
def test_row_quantiser_bit_exact_bf16(rows, K):
    x = _spread(rows, K, seed=rows + K)
    q, s = mok.mxfp8_quantize_rows(x.cuda())
    wq, ws = _oracle_quant(x.float().numpy())
    assert np.array_equal(q.cpu().numpy().reshape(-1), wq)
    assert np.array_equal(s.cpu().numpy().reshape(-1), ws)


def test_row_quantiser_bit_exact_fp32_golden_blocks():
    """fp32 input (the form the SwiGLU epilogue quantises): the hand-computed
    edge-case blocks plus random fp32 data."""
    with open(os.path.join(GOLDEN, "mxfp8_blocks.json")) as f:
        spec = json.load(f)
    blocks = []
    for case in spec["cases"]:
        v = np.zeros(32, np.float32)
        for i, val in case["values"].items():
            v[int(i)] = val
        blocks.append(v)
    g = np.random.default_rng(3)
    rnd = (g.standard_normal((10, 32)) * np.exp2(g.integers(-60, 60, (10, 1)))).astype(np.float32)
    data = np.concatenate([np.stack(blocks), rnd]).reshape(-1, 64)  # two blocks per row
    q, s = mok.mxfp8_quantize_rows(torch.from_numpy(data).cuda())
    wq, ws = _oracle_quant(data)
    assert np.array_equal(q.cpu().numpy().reshape(-1), wq)
    assert np.array_equal(s.cpu().numpy().reshape(-1), ws)
    # and the golden bytes themselves
    gq = q.cpu().numpy().reshape(-1, 32)
    gs = s.cpu().numpy().reshape(-1)
    for i, case in enumerate(spec["cases"]):
        assert gs[i] == int(case["scale"], 16), case["name"]
        for j, b in case["bytes"].items():
            assert gq[i, int(j)] == int(b, 16), (case["name"], j)


REL_FRO_MX = 2e-2

MX_CASES = {
    "tiny": mokgen.scaled(mokgen.CONFIGS["tiny"], seed=201),
    "page_like": mokgen.scaled(mokgen.CONFIGS["page"], T=256, E=12, seed=202),
    "ragged": mokgen.scaled(mokgen.CONFIGS["tiny"], T=600, H=384, I=192, E=5, k=3, R=3, seed=203),
}


def _mx_pack(dwg, dwu, dwd):
    qg, sg = mok.quantize_weights_mxfp8(dwg)
    qu, su = mok.quantize_weights_mxfp8(dwu)
    qd, sd = mok.quantize_weights_mxfp8(dwd)
    return (qg, sg, qu, su, qd, sd)


@pytest.mark.parametrize("name", list(MX_CASES))
def test_mxfp8_forward_matches_emulated_oracle(name):
    cfg = MX_CASES[name]
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    wg, wu, wd = mokgen.all_expert_weights(cfg)
    pack = _mx_pack(wg.cuda(), wu.cuda(), wd.cuda())
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    ys, ws = mok.moe_forward_mxfp8(mok.shards(x.cuda(), cfg.R), pack, p)
    assert mok.get_status(ws) == mok.MOK_OK
    y = torch.cat([s.cpu() for s in ys]).double()
    want = oracle.moe_forward_mxfp8(x, logits, wg, wu, wd, cfg.k, cfg.R)
    rel = (torch.linalg.norm(y - want) / torch.linalg.norm(want)).item()
    assert rel <= REL_FRO_MX, rel


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_mxfp8_steps_one_at_a_time_equal_forward(name):
    """mok_gather_mxfp8 + mok_expert_ffn_mxfp8 + mok_combine compute exactly
    what mok_moe_forward's MXFP8 path computes."""
    cfg = MX_CASES[name]
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    wg, wu, wd = mokgen.all_expert_weights(cfg)
    pack = _mx_pack(wg.cuda(), wu.cuda(), wd.cuda())
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    xs = mok.shards(x.cuda(), cfg.R)
    ys, _ = mok.moe_forward_mxfp8(xs, pack, p)
    rows_q, planes = mok.gather_mxfp8(xs, p)
    out, ws = mok.expert_ffn_mxfp8(rows_q, planes, pack, p)
    assert mok.get_status(ws) == mok.MOK_OK
    y2 = [torch.empty_like(s) for s in xs]
    mok.combine(out, p, y2)
    assert torch.equal(torch.cat([s.cpu() for s in ys]), torch.cat([s.cpu() for s in y2]))


@pytest.mark.parametrize("name,minibatch,ring,dispatch", [("tiny", 64, 0, 16), ("page_like", 256, 0, 4),
                                                          ("page_like", 16, 0, 2), ("ragged", 600, 1300, 8),
                                                          ("page_like", 256, 0, -2), ("ragged", 600, 1300, -1)])
def test_mxfp8_persistent_equals_staged(name, minibatch, ring, dispatch):
    """The persistent SM-partitioned kernel on the MXFP8 path (its dispatch
    CTAs quantise the rows into the ring) computes the staged path's bits at
    every minibatch size, ring size and dispatch/GEMM split: quantisation is
    per row and per 32-block, and each token's MMA column does not depend on
    how the rows are cut into chunks."""
    cfg = MX_CASES[name]
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    wg, wu, wd = mokgen.all_expert_weights(cfg)
    pack = _mx_pack(wg.cuda(), wu.cuda(), wd.cuda())
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    xs = mok.shards(x.cuda(), cfg.R)
    ys_s, ws_s = mok.moe_forward_mxfp8(xs, pack, p)
    # dispatch < 0: the warp layout (quantising dispatch warps in every CTA)
    split = dict(dispatch_ctas=dispatch) if dispatch > 0 else dict(dispatch_warps=-dispatch)
    opts = mok.fwd_opts(mode=mok.MOK_MODE_PERSISTENT, mxfp8=True, ring_slots=ring, **split)
    ys_p, ws_p = mok.moe_forward_mxfp8(xs, pack, p, minibatch=minibatch, opts=opts)
    assert mok.get_status(ws_s) == mok.MOK_OK and mok.get_status(ws_p) == mok.MOK_OK
    y_s = torch.cat([s.cpu() for s in ys_s])
    y_p = torch.cat([s.cpu() for s in ys_p])
    want = oracle.moe_forward_mxfp8(x, logits, wg, wu, wd, cfg.k, cfg.R)
    rel = (torch.linalg.norm(y_p.double() - want) / torch.linalg.norm(want)).item()
    assert rel <= REL_FRO_MX, rel
    assert torch.equal(y_p, y_s), (y_p.double() - y_s.double()).abs().max().item()


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_mxfp8_gather_bit_exact(name):
    """The fused quantising gather: row bytes and scale planes equal the
    oracle's quantisation of each row's token, bit for bit."""
    cfg = MX_CASES[name]
    if cfg.H % 128:
        cfg = mokgen.scaled(cfg, H=256)
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    p = mok.plan(logits.cuda(), cfg.k, cfg.R)
    rows_q, planes = mok.gather_mxfp8(mok.shards(x.cuda(), cfg.R), p)
    rows_q, planes = rows_q.cpu().numpy(), planes.cpu().numpy()
    pl = oracle.plan(logits, cfg.k, cfg.R)
    tok = (pl["src_rank"] * (cfg.T // cfg.R) + pl["src_index"]).numpy()
    wq, ws = _oracle_quant(x.float().numpy()[tok])
    ns = cfg.T * cfg.k
    assert np.array_equal(rows_q.reshape(-1), wq)
    # planes [H/128][sc_rows][4] -> per row, blocks in order
    got_s = planes[:, :ns, :].transpose(1, 0, 2).reshape(ns, cfg.H // 32)
    assert np.array_equal(got_s.reshape(-1), ws)


def test_weight_quantiser_bit_exact():
    E, K, N = 3, 256, 192
    w = _spread(E * K, N, seed=9).reshape(E, K, N)
    q, s = mok.quantize_weights_mxfp8(w.cuda())
    q, s = q.cpu().numpy(), s.cpu().numpy()
    for e in range(E):
        cols = w[e].float().t().contiguous().numpy()  # [N, K]: blocks along K are contiguous
        wq, ws = _oracle_quant(cols)
        assert np.array_equal(q[e].T.reshape(-1), wq)
        assert np.array_equal(s[e].T.reshape(-1), ws)
