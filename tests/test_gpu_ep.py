"""GPU parity of the expert-parallel forward (mok_ep_dispatch_ffn +
mok_ep_combine) through the C ABI.

Every rank of a group runs here on the one GPU, driven by this process
(MOK_EP_SYNC_CALLER: all ranks' dispatch calls, then all ranks' combine
calls, ordered on one stream; no kernel waits on another).  Each rank's
token shard and slot buffer is its own allocation, so the pull reads other
ranks' buffers and the down GEMM's epilogue pushes into them exactly as it
would through peer pointers.  The results must equal the single-GPU staged
forward over the same plan bit for bit (the same per-slot arithmetic, the
same combine order), and the oracle within the forward's bound.  The device
barrier runs with one rank (it only waits for itself) and, to check that a
wait gives up, with a second counter that nothing ever increments.

Source: MoK article (tahou.com), pull-dispatch and push-combine paragraphs."""
import multiprocessing as pymp

import pytest
import torch

import combine_device_top_b200 as mok
import mokgen
from helpers import Case, assert_bf16_close

pytestmark = pytest.mark.gpu

STAGED = mok.MOK_MODE_STAGED


def small(**kw):
    return mokgen.scaled(mokgen.CONFIGS["tiny"], **kw)


CASES = {
    # uneven expert split (10 over 3 and 4 ranks), several chunks per expert
    "ragged": small(T=384, H=256, I=128, E=10, k=3, R=1, seed=701),
    # more ranks than experts on some splits: ranks with no experts
    "few_experts": small(T=384, H=384, I=192, E=3, k=2, R=1, seed=702),
    "many_experts": small(T=768, H=256, I=128, E=64, k=6, R=1, seed=703),
}


class Ranks:
    """G ranks' buffers on this GPU: tokens, slot buffers, workspaces and
    their descriptors."""

    def __init__(self, case: Case, G: int, sync=mok.MOK_EP_SYNC_CALLER):
        cfg = case.cfg
        self.case, self.G = case, G
        self.S_r = cfg.T // G
        self.xs = [case.dx[h * self.S_r:(h + 1) * self.S_r].clone() for h in range(G)]
        self.slots = [torch.zeros(mok.ep_slot_bytes(self.S_r, cfg.H, cfg.k), dtype=torch.uint8, device="cuda")
                      for _ in range(G)]
        self.parts = [mok.ep_partition(cfg.E, G, h) for h in range(G)]
        self.ws = [torch.empty(max(256, mok.ep_workspace_bytes(cfg.T, cfg.H, cfg.I, n, cfg.k)), dtype=torch.uint8,
                               device="cuda") for (_, n) in self.parts]
        self.w = [tuple(w[e0:e0 + n].contiguous() for w in (case.dwg, case.dwu, case.dwd)) for (e0, n) in self.parts]
        self.desc = [mok.ep_desc(G, h, *self.parts[h], [x.data_ptr() for x in self.xs],
                                 [s.data_ptr() for s in self.slots], sync) for h in range(G)]

    def step(self, p, step):
        ys = [torch.empty((self.S_r, self.case.cfg.H), dtype=torch.bfloat16, device="cuda") for _ in range(self.G)]
        for h in range(self.G):
            mok.ep_dispatch_ffn(p, self.desc[h], *self.w[h], step, self.ws[h])
        for h in range(self.G):
            mok.ep_combine(p, self.desc[h], ys[h], step, self.ws[h])
        for h in range(self.G):
            assert mok.get_status(self.ws[h]) == mok.MOK_OK
        return torch.cat(ys)


def _staged_y(case: Case, G: int):
    p = mok.plan(case.dlogits, case.cfg.k, G)
    ys, _ = mok.moe_forward(mok.shards(case.dx, G), case.dwg, case.dwu, case.dwd, p, 0,
                            mok.fwd_opts(mode=STAGED))
    return torch.cat(ys), p


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("G", [1, 2, 3, 4])
def test_ep_ranks_match_the_single_gpu_forward(name, G):
    case = Case(CASES[name])
    if case.cfg.T % G:
        pytest.skip("T does not split over G ranks")
    want, p = _staged_y(case, G)
    ranks = Ranks(case, G)
    got = ranks.step(p, 1)
    assert torch.equal(got, want)


def test_ep_ranks_match_the_oracle():
    case = Case(CASES["ragged"])
    ranks = Ranks(case, 3)
    p = mok.plan(case.dlogits, case.cfg.k, 3)
    got = ranks.step(p, 1)
    # the oracle's plan of the same tokens does not depend on R
    assert_bf16_close(got.cpu(), case.oracle_y(), "EP forward, 3 ranks")


def test_ep_ranks_reuse_their_buffers_over_steps():
    """Two steps with new tokens and routing through the same buffers."""
    case1 = Case(CASES["ragged"])
    ranks = Ranks(case1, 4)
    p1 = mok.plan(case1.dlogits, case1.cfg.k, 4)
    y1 = ranks.step(p1, 1)
    cfg2 = small(T=384, H=256, I=128, E=10, k=3, R=1, seed=711)
    case2 = Case(cfg2)
    for h in range(4):
        ranks.xs[h].copy_(case2.dx[h * ranks.S_r:(h + 1) * ranks.S_r])
    # the same weights: rank buffers hold case1's experts
    case2.dwg, case2.dwu, case2.dwd = case1.dwg, case1.dwu, case1.dwd
    p2 = mok.plan(case2.dlogits, cfg2.k, 4)
    y2 = ranks.step(p2, 2)
    want2, _ = _staged_y(case2, 4)
    assert torch.equal(y2, want2)
    want1, _ = _staged_y(case1, 4)
    assert torch.equal(y1, want1)


def test_ep_device_barrier_with_one_rank():
    """MOK_EP_SYNC_DEVICE with G = 1: each call's barrier waits for this
    rank's own arrival; three steps, then the counter holds 2 per step."""
    case = Case(CASES["ragged"])
    ranks = Ranks(case, 1, sync=mok.MOK_EP_SYNC_DEVICE)
    want, p = _staged_y(case, 1)
    for s in (1, 2, 3):
        assert torch.equal(ranks.step(p, s), want)
    cfg = case.cfg
    off = mok.ep_slot_bytes(ranks.S_r, cfg.H, cfg.k) - 256
    counter = ranks.slots[0][off:off + 4].cpu().view(torch.int32).item()
    assert counter == 6


def test_ep_group_driver_with_one_rank():
    """EpGroup on one rank (no process group): plan, dispatch and combine
    with the device barriers, equal to the staged forward."""
    case = Case(CASES["many_experts"])
    cfg = case.cfg
    grp = mok.EpGroup(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    grp.x.copy_(case.dx)
    want, _ = _staged_y(case, 1)
    for _ in range(2):
        y = grp.forward(case.dlogits, case.dwg, case.dwu, case.dwd)
        assert grp.status() == mok.MOK_OK
        assert torch.equal(y, want)
    grp.close()


def test_ep_barrier_wait_gives_up_and_reports():
    """A two-rank barrier whose other rank never arrives (its counter is a
    buffer nothing increments): the wait gives up after 1 ms, the status
    word reads MOK_ERR_TIMEOUT, and the context stays usable."""
    case = Case(CASES["ragged"])
    ranks = Ranks(case, 2, sync=mok.MOK_EP_SYNC_DEVICE)
    p = mok.plan(case.dlogits, case.cfg.k, 2)
    mok.ep_dispatch_ffn(p, ranks.desc[0], *ranks.w[0], 1, ranks.ws[0], timeout_ns=1_000_000)
    assert mok.get_status(ranks.ws[0]) == mok.MOK_ERR_TIMEOUT
    assert "device status 5" in mok.last_error()
    # the same buffers, now ordered by this process: correct results
    for d in ranks.desc:
        d.sync = mok.MOK_EP_SYNC_CALLER
    want, _ = _staged_y(case, 2)
    assert torch.equal(ranks.step(p, 1), want)


def _ipc_child(handle, offset, seed, q):
    """Another process on the same GPU: map the parent's token buffer and
    gather its rows through the library."""
    try:
        import combine_device_top_b200 as m
        import mokgen as mg
        cfg = mg.scaled(mg.CONFIGS["tiny"], T=128, H=256, I=128, E=8, k=2, R=1, seed=seed)
        x = mg.tokens(cfg)
        torch.cuda.init()
        base = m.ipc_import(handle)
        logits = mg.router_logits(cfg, x).cuda()
        p = m.plan(logits, cfg.k, 1)
        rows = torch.empty((cfg.T * cfg.k, cfg.H), dtype=torch.bfloat16, device="cuda")
        L = m.lib()
        import ctypes
        xs = (ctypes.c_void_p * 1)(base + offset)
        rc = L.mok_gather(xs, cfg.H, ctypes.byref(p.c), ctypes.c_void_p(rows.data_ptr()), None)
        torch.cuda.synchronize()
        pos = p.pos().cpu().view(cfg.T, cfg.k)
        ok = rc == 0 and all(torch.equal(rows[pos[:, j].long()].cpu(), x) for j in range(cfg.k))
        m.ipc_close(base)
        q.put(("ok" if ok else "mismatch", rc))
    except Exception as e:  # reported to the parent
        q.put(("error", repr(e)))


def test_ipc_export_import_between_processes():
    """CUDA IPC between two processes on one GPU: the child maps the
    parent's buffer (at an offset inside its allocation) and pulls from it."""
    cfg = mokgen.scaled(mokgen.CONFIGS["tiny"], T=128, H=256, I=128, E=8, k=2, R=1, seed=721)
    x = mokgen.tokens(cfg)
    big = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")   # x sits at an offset inside it
    view = big[4096:4096 + x.numel() * 2].view(torch.bfloat16).view(cfg.T, cfg.H)
    view.copy_(x.cuda())
    torch.cuda.synchronize()
    handle, offset = mok.ipc_export(view)
    assert offset >= 4096 and len(handle) == mok.MOK_IPC_HANDLE_BYTES
    ctx = pymp.get_context("spawn")
    q = ctx.Queue()
    proc = ctx.Process(target=_ipc_child, args=(handle, offset, 721, q))
    proc.start()
    status, detail = q.get(timeout=300)
    proc.join(timeout=120)
    assert status == "ok", detail
    assert proc.exitcode == 0


# ---------------------------------------------------------------- the MXFP8 path
def _mx_pack(wg, wu, wd):
    if wg.shape[0] == 0:  # a rank without experts: no weights to quantise
        H, I = wg.shape[1], wg.shape[2]
        shapes = [(0, H, I), (0, H // 32, I), (0, H, I), (0, H // 32, I), (0, I, H), (0, I // 32, H)]
        return tuple(torch.empty(sh, dtype=torch.uint8, device="cuda") for sh in shapes)
    return (*mok.quantize_weights_mxfp8(wg), *mok.quantize_weights_mxfp8(wu), *mok.quantize_weights_mxfp8(wd))


MX_CASES = {
    "ragged": small(T=384, H=256, I=128, E=10, k=3, R=1, seed=741),
    "few_experts": small(T=256, H=384, I=256, E=3, k=2, R=1, seed=742),
}


@pytest.mark.parametrize("name", list(MX_CASES))
@pytest.mark.parametrize("G", [1, 2, 4])
def test_ep_mxfp8_ranks_match_the_single_gpu_forward(name, G):
    """The MXFP8 path (quantising pull, block-scaled FFN, bf16 slot rows
    pushed to the token's rank) over G emulated ranks equals the staged
    MXFP8 forward bit for bit; each rank quantises only its own experts."""
    case = Case(MX_CASES[name])
    cfg = case.cfg
    p = mok.plan(case.dlogits, cfg.k, G)
    ys, _ = mok.moe_forward_mxfp8(mok.shards(case.dx, G), _mx_pack(case.dwg, case.dwu, case.dwd), p)
    want = torch.cat(ys)
    ranks = Ranks(case, G)
    for d in ranks.desc:
        d.mxfp8 = 1
    packs = [_mx_pack(*ranks.w[h]) for h in range(G)]
    y = [torch.empty((ranks.S_r, cfg.H), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    for h in range(G):
        mok.ep_dispatch_ffn_mxfp8(p, ranks.desc[h], packs[h], cfg.H, 1, ranks.ws[h])
    for h in range(G):
        mok.ep_combine(p, ranks.desc[h], y[h], 1, ranks.ws[h])
    for h in range(G):
        assert mok.get_status(ranks.ws[h]) == mok.MOK_OK
    assert torch.equal(torch.cat(y), want)


def test_ep_group_driver_mxfp8_with_one_rank():
    """EpGroup(mxfp8=True) on one rank, device barriers, two steps."""
    case = Case(MX_CASES["ragged"])
    cfg = case.cfg
    pack = _mx_pack(case.dwg, case.dwu, case.dwd)
    p = mok.plan(case.dlogits, cfg.k, 1)
    ys, _ = mok.moe_forward_mxfp8([case.dx], pack, p)
    grp = mok.EpGroup(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, mxfp8=True)
    grp.x.copy_(case.dx)
    for _ in range(2):
        y = grp.forward(case.dlogits, pack, None, None)
        assert grp.status() == mok.MOK_OK
        assert torch.equal(y, ys[0])
    grp.close()

