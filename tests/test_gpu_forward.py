"""GPU parity of the dispatch (gather), the grouped SwiGLU GEMM, the combine
and the whole forward layer against the oracle, through the C ABI."""
import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
import oracle
from helpers import Case, assert_bf16_close, sample_tokens

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


def test_combine_matches_oracle():
    case = Case(FFN_CASES["many_experts"])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    # fp16 per-slot outputs, as the grouped GEMM stores them
    out = mokgen.normal(5, 77, (cfg.T * cfg.k, cfg.H), 1.0, dtype=torch.float32).to(torch.float16)
    ys = [torch.empty((cfg.S_r, cfg.H), dtype=torch.bfloat16, device="cuda") for _ in range(cfg.R)]
    mok.combine(out.cuda(), p, ys)
    torch.cuda.synchronize()
    g = oracle.plan(case.logits, cfg.k, cfg.R)["gates"]
    want = oracle.combine(out.double().view(cfg.T, cfg.k, cfg.H), g)
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
    assert_bf16_close(out.cpu(), want, name)


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
    assert_bf16_close(got["1"], want, name)


def test_grouped_gemm_single_expert_vs_torch_fp32():
    """E = 1, k = 1: the grouped GEMM is a dense SwiGLU FFN; compare with a
    plain PyTorch fp32 reference of the same op on the GPU."""
    case = Case(FFN_CASES["one_expert_dense"])
    cfg = case.cfg
    p = mok.plan(case.dlogits, 1, cfg.R)
    rows = mok.gather(case.x_shards(), p)
    out, _ = mok.expert_ffn(rows, case.dwg, case.dwu, case.dwd, p)
    x = case.dx.float()
    a, b = x @ case.dwg[0].float(), x @ case.dwu[0].float()
    h = (torch.nn.functional.silu(a) * b).to(torch.float16).float()
    ref = h @ case.dwd[0].float()
    torch.cuda.synchronize()
    assert_bf16_close(out.float(), ref, "dense")


def test_prepare_w_down_matches_torch_conversion():
    """The fp16 copy of W_down equals torch's bf16 -> fp16 conversion in the
    representable range; out-of-range magnitudes saturate to 65504."""
    w = mokgen.normal(3, 5, (4, 96, 136), 1.0 / 96 ** 0.5)
    special = torch.tensor([0.0, -0.0, 1e-6, -3e-7, 6.0e-5, 1e5, -3e38, 65504.0, 7.0], dtype=torch.float32)
    w.view(-1)[: special.numel()] = special.to(torch.bfloat16)
    got = mok.prepare_w_down(w.cuda()).cpu()
    want = w.float().clamp(-65504, 65504).to(torch.float16)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    odd = mokgen.normal(3, 6, (1001,), 1.0)            # length not a multiple of 8
    assert torch.equal(mok.prepare_w_down(odd.cuda()).cpu(), odd.float().to(torch.float16))


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


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mixtral", "page", "zipf"])
def test_forward_staged_full_size_sampled(name):
    """Full-size configurations: every output row is produced by the GPU;
    sampled tokens are checked against the oracle."""
    cfg = mokgen.CONFIGS[name]
    case = Case(cfg, weights_on_host=False)
    p = mok.plan(case.dlogits, cfg.k, cfg.R)
    ys, ws = mok.moe_forward(case.x_shards(), case.dwg, case.dwu, case.dwd, p, cfg.minibatch,
                             mok.fwd_opts(mode=STAGED))
    assert mok.get_status(ws) == mok.MOK_OK
    y = torch.cat([s.cpu() for s in ys])
    assert torch.isfinite(y.float()).all()
    ids = sample_tokens(cfg.T, 12, seed=cfg.seed)
    want = case.oracle_y(ids)
    assert_bf16_close(y[ids], want, name)
