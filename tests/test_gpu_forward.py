"""GPU parity of the dispatch (gather), the grouped SwiGLU GEMM, the combine
and the whole forward layer against the oracle, through the C ABI."""
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
import oracle
from helpers import Case, assert_bf16_close, decode_slots, encode_slots, sample_tokens

pytestmark = pytest.mark.gpu

STAGED = mok.MOK_MODE_STAGED


def small(name="tiny", **kw):
    return mokgen.scaled(mokgen.CONFIGS[name], **kw)


# shapes that span several tiles in M, N and K, ragged chunk tails and
# experts with more than one 256-row chunk
FFN_CASES = {
    "tiny": small(),
    "one_expert_dense": small(name="tiny", T=384, H=256, I=128, E=1, k=1, R=2, seed=101),
    "multi_chunk": small(T=1100, H=384, I=192, E=3, k=2, R=4, seed=102),
    "many_experts": small(T=640, H=256, I=128, E=96, k=6, R=5, seed=103),
    "wide": small(T=96, H=1024, I=512, E=4, k=2, R=3, seed=104),
    # top-k beyond the combine's 8 slots in flight (several rounds)
    "k16": small(T=128, H=256, I=128, E=32, k=16, R=2, seed=105),
    "k32": small(T=64, H=256, I=128, E=48, k=32, R=2, seed=106),
}


def _oracle_slots(case: Case, p):
    """Oracle per-slot expert outputs [T*k, H] (float64) in slot order."""
    cfg = case.cfg
    pl = oracle.plan(case.logits, cfg.k, cfg.R)
    rows = oracle.gather(case.x, cfg.R, pl["src_rank"], pl["src_index"])
    o = torch.empty((cfg.T * cfg.k, cfg.H), dtype=torch.float64)
    off = pl["offsets"]
    for e in range(cfg.E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            wg, wu, wd = case.weight_fn(e)
            o[pl["row_slot"][a:b].long()] = oracle.expert_ffn(rows[a:b], wg, wu, wd)
    return o, rows, pl


@pytest.mark.parametrize("name", ["tiny", "multi_chunk"])
def test_gather_bit_exact(name):
    case = Case(FFN_CASES[name])
    p = mok.plan(case.dlogits, case.cfg.k, case.cfg.R)
    rows = mok.gather(case.x_shards(), p)
    torch.cuda.synchronize()
    pl = oracle.plan(case.logits, case.cfg.k, case.cfg.R)
    want = oracle.gather(case.x, case.cfg.R, pl["src_rank"], pl["src_index"])
    assert torch.equal(rows.cpu(), want)


@pytest.mark.parametrize("slot_dtype", ["f16s", torch.float32, torch.bfloat16])
@pytest.mark.parametrize("name", ["many_experts", "k16", "k32"])
def test_combine_matches_oracle(name, slot_dtype):
    """The fixed-order combine over slot outputs of every form (fp16 with
    block exponents: the bf16 path, bf16: the MXFP8 path, fp32); k = 16 and
    32 take several rounds of the combine's 8 slots in flight.  The fp16
    rows span many binades (block exponents far apart)."""
    case = Case(FFN_CASES[name])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    vals = mokgen.normal(5, 77, (cfg.T * cfg.k, cfg.H), 1.0, dtype=torch.float32)
    if slot_dtype == "f16s":
        vals = vals * torch.exp2(torch.randint(-40, 40, (cfg.T * cfg.k, 1),
                                               generator=torch.Generator().manual_seed(3)).float())
        out = encode_slots(vals)
        vals = decode_slots(out, cfg.T * cfg.k, cfg.H)
    else:
        out = vals.to(slot_dtype)
        vals = out.double()
    ys = [torch.empty((cfg.S_r, cfg.H), dtype=torch.bfloat16, device="cuda") for _ in range(cfg.R)]
    mok.combine(out.cuda(), p, ys)
    torch.cuda.synchronize()
    g = oracle.plan(case.logits, cfg.k, cfg.R)["gates"]
    want = oracle.combine(vals.view(cfg.T, cfg.k, cfg.H), g)
    got = torch.cat([y.cpu() for y in ys])
    # fp32 accumulation, one bf16 rounding: within a bf16 half-ulp (2^-8
    # relative) of the exact value, plus fp32 accumulation slack
    err = (got.double() - want).abs()
    assert (err <= want.abs() * 2.0 ** -8 + 1e-5).all()


@pytest.mark.parametrize("name", list(FFN_CASES))
def test_grouped_gemm_swiglu_matches_oracle(name):
    case = Case(FFN_CASES[name])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    rows = mok.gather(case.x_shards(), p)
    out, ws = mok.expert_ffn(rows, case.dwg, case.dwu, case.dwd, p)
    torch.cuda.synchronize()
    want, _, _ = _oracle_slots(case, p)
    assert_bf16_close(decode_slots(out, p.ns, cfg.H), want, name)


@pytest.mark.parametrize("name", ["multi_chunk", "many_experts", "tiny"])
def test_grouped_gemm_m_tile_pairing_is_exact(name, monkeypatch):
    """Units of one M tile and units of two M tiles sharing each token tile
    (with 1 or 2 TMEM buffers per unit, and a single tile at an odd end of
    the M range) compute every output with the same MMA sequence: results
    are bit-identical, and both match the oracle."""
    case = Case(FFN_CASES[name])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    rows = mok.gather(case.x_shards(), p)
    got = {}
    for pair in ("0", "1"):
        monkeypatch.setenv("MOK_GEMM_PAIR", pair)
        out, ws = mok.expert_ffn(rows, case.dwg, case.dwu, case.dwd, p)
        assert mok.get_status(ws) == mok.MOK_OK
        got[pair] = out.cpu()
    assert torch.equal(got["0"], got["1"])
    want, _, _ = _oracle_slots(case, p)
    assert_bf16_close(decode_slots(got["1"], p.ns, cfg.H), want, name)


@pytest.mark.parametrize("name", ["tiny", "many_experts", "wide", "k16", "multi_chunk"])
def test_grouped_gemm_cta_pairs_are_exact(name, monkeypatch):
    """The same phases on CTA pairs (clusters of two CTAs, one M = 256 MMA
    over both CTAs' weight tiles, each CTA holding half of the token tile)
    accumulate every output in the same K order: results are bit-identical
    to one-CTA units, and match the oracle."""
    case = Case(FFN_CASES[name])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    rows = mok.gather(case.x_shards(), p)
    got = {}
    # none; the down phase; both phases; gate/up on pairs of CTAs holding two M tiles each
    for cta_pair in ("0", "1", "2", "3"):
        monkeypatch.setenv("MOK_GEMM_CTA_PAIR", cta_pair)
        out, ws = mok.expert_ffn(rows, case.dwg, case.dwu, case.dwd, p)
        assert mok.get_status(ws) == mok.MOK_OK, mok.last_error()
        got[cta_pair] = out.cpu()
    for mode in ("1", "2", "3"):
        assert torch.equal(got["0"], got[mode]), mode
    want, _, _ = _oracle_slots(case, p)
    assert_bf16_close(decode_slots(got["2"], p.ns, cfg.H), want, name)


def test_grouped_gemm_single_expert_vs_torch_fp32():
    """E = 1, k = 1: the grouped GEMM is a dense SwiGLU FFN; compare with a
    plain PyTorch fp32 reference of the same op on the GPU (h rounded to
    bf16 as the kernel stores it)."""
    case = Case(FFN_CASES["one_expert_dense"])
    cfg = case.cfg
    p = mok.plan(case.dlogits, 1, cfg.R)
    rows = mok.gather(case.x_shards(), p)
    out, _ = mok.expert_ffn(rows, case.dwg, case.dwu, case.dwd, p)
    x = case.dx.float()
    a, b = x @ case.dwg[0].float(), x @ case.dwu[0].float()
    h = (torch.nn.functional.silu(a) * b).to(torch.bfloat16).float()
    ref = h @ case.dwd[0].float()
    torch.cuda.synchronize()
    assert_bf16_close(decode_slots(out, p.ns, cfg.H), ref.cpu(), "dense")


@pytest.mark.parametrize("name", list(FFN_CASES))
def test_forward_staged_matches_oracle(name):
    case = Case(FFN_CASES[name])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, cfg.minibatch,
                             mok.fwd_opts(mode=STAGED))
    assert mok.get_status(ws) == mok.MOK_OK
    y = torch.cat([s.cpu() for s in ys])
    assert_bf16_close(y, case.oracle_y(), name)


def test_forward_host_entry_matches_device_entry():
    case = Case(FFN_CASES["tiny"])
    cfg = case.cfg
    opts = mok.fwd_opts(mode=STAGED)
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    ys, _ = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, cfg.minibatch, opts)
    ws = torch.empty(mok.forward_host_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.minibatch, opts),
                     dtype=torch.uint8, device="cuda")
    y_host = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
    mok.moe_forward_host(case.x.pin_memory(), case.logits.pin_memory(), cfg.k, cfg.R, case.dwg, case.dwu,
                         case.dwd, cfg.minibatch, opts, ws, y_host)
    assert torch.equal(y_host, torch.cat([s.cpu() for s in ys]))


@pytest.mark.parametrize("mode", [STAGED, mok.MOK_MODE_PERSISTENT])
def test_forward_host_batches_equal_single_host_calls(mode):
    """Four different batches through the overlapped host pipeline (two
    staging sets, copies on their own streams) give the bits of four
    separate mok_moe_forward_host calls."""
    case = Case(FFN_CASES["multi_chunk"])
    cfg = case.cfg
    opts = mok.fwd_opts(mode=mode)
    xs = [(case.x.float() * (1.0 + 0.25 * i)).to(torch.bfloat16).pin_memory() for i in range(4)]
    ls = [(case.logits + 0.5 * i * torch.roll(case.logits, i, 1)).contiguous().pin_memory() for i in range(4)]
    ws1 = torch.empty(mok.forward_host_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, 64, opts),
                      dtype=torch.uint8, device="cuda")
    want = []
    for i in range(4):
        y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
        mok.moe_forward_host(xs[i], ls[i], cfg.k, cfg.R, case.dwg, case.dwu, case.dwd, 64, opts, ws1, y)
        want.append(y.clone())
    wsb = torch.empty(mok.forward_host_batches_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, 64, opts),
                      dtype=torch.uint8, device="cuda")
    ys = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    mok.moe_forward_host_batches(xs, ls, cfg.k, cfg.R, case.dwg, case.dwu, case.dwd, 64, opts, wsb, ys)
    for i in range(4):
        assert torch.equal(ys[i], want[i]), i
    # again on the same workspace, every batch written to one shared buffer: the last batch wins
    shared = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
    mok.moe_forward_host_batches(xs[::-1], ls[::-1], cfg.k, cfg.R, case.dwg, case.dwu, case.dwd, 64, opts, wsb,
                                 [shared] * 4)
    assert torch.equal(shared, want[0])


def _forward_staged(case: Case, logits=None):
    cfg = case.cfg
    dlogits = case.dlogits if logits is None else logits.cuda()
    p = mok.plan(dlogits, cfg.k, cfg.R)
    ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, cfg.minibatch,
                             mok.fwd_opts(mode=STAGED))
    assert mok.get_status(ws) == mok.MOK_OK
    return torch.cat([s.cpu() for s in ys]), p


def test_forward_with_experts_that_receive_no_rows():
    """Experts 0, 5, 6 and 15 get no token (their logits are pushed far
    down): their segments are empty, the chunk list skips them, and every
    token is still correct."""
    case = Case(small(T=512, H=256, I=128, E=16, k=2, R=4, seed=107))
    logits = case.logits.clone()
    logits[:, [0, 5, 6, 15]] -= 100.0
    y, p = _forward_staged(case, logits)
    counts = p.counts().cpu()
    assert (counts[[0, 5, 6, 15]] == 0).all() and counts.sum().item() == case.cfg.T * case.cfg.k
    want, _, _ = oracle.moe_forward(case.x, logits, case.wg, case.wu, case.wd, case.cfg.k, case.cfg.R)
    assert_bf16_close(y, want, "empty experts")


@pytest.mark.parametrize("scale", [256.0, 1024.0])
def test_forward_large_magnitudes_keep_range(scale):
    """Inputs scaled so that h and the slot outputs pass 65504 (the fp16
    limit) by far: every stored intermediate has fp32's exponent range, so
    the bound holds without saturation."""
    cfg = small(seed=108)
    case = Case(cfg)
    case.x = (case.x.float() * scale).to(torch.bfloat16)
    case.dx = case.x.cuda()
    y, p = _forward_staged(case)
    want, _, _ = oracle.moe_forward(case.x, case.logits, case.wg, case.wu, case.wd, cfg.k, cfg.R)
    assert want.abs().max().item() > 65504.0
    assert torch.isfinite(y.float()).all()
    assert_bf16_close(y, want, f"x * {scale}")
    # and the slot outputs themselves, element by element
    rows = mok.gather(case.x_shards(), p)
    out, _ = mok.expert_ffn(rows, case.dwg, case.dwu, case.dwd, p)
    want_slots, _, _ = _oracle_slots(case, p)
    assert want_slots.abs().max().item() > 65504.0
    assert_bf16_close(decode_slots(out, p.ns, cfg.H), want_slots, f"slots x * {scale}")
