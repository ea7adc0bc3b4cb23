"""The expert-parallel forward across real GPUs: one process per GPU over
NCCL, peer pointers by CUDA IPC, device barriers (MOK_EP_SYNC_DEVICE).
Each rank's y must equal the single-GPU staged forward's rows of its
tokens, bit for bit.  Needs two or more GPUs; skipped otherwise.

NVLS is switched off (NCCL_NVLS_ENABLE=0) and the library's kernels use
plain peer loads and stores only.  Every wait is bounded (the process group
by a 60 s timeout, the device barrier by 2 s, the test by its join limits)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q, mxfp8=False):
    import datetime

    import torch.distributed as dist

    import combine_device_top_b200 as mok
    import mokgen
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
    torch.cuda.set_device(rank)
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", rank))
    try:
        cfg = mokgen.scaled(mokgen.CONFIGS["tiny"], T=256 * world, H=256, I=128, E=10, k=3, R=1, seed=731)
        x = mokgen.tokens(cfg)
        logits = mokgen.router_logits(cfg, x)
        wg, wu, wd = mokgen.all_expert_weights(cfg)
        grp = mok.EpGroup(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, mxfp8=mxfp8)
        S_r, e0, n = grp.S_r, grp.e0, grp.e_loc
        grp.x.copy_(x[rank * S_r:(rank + 1) * S_r].cuda())
        w = [t[e0:e0 + n].contiguous().cuda() for t in (wg, wu, wd)]
        pack = lambda ws: tuple(t for wt in ws for t in mok.quantize_weights_mxfp8(wt))
        if mxfp8:  # every rank holds at least one of the 10 experts
            w = [pack(w), None, None]
        ok = True
        for _ in range(3):
            y = grp.forward(logits[rank * S_r:(rank + 1) * S_r].contiguous().cuda(), *w)
            ok &= grp.status() == mok.MOK_OK
        # the single-GPU staged forward of the whole layer, on this GPU
        p = mok.plan(logits.cuda(), cfg.k, world)
        full = [wg.cuda(), wu.cuda(), wd.cuda()]
        if mxfp8:
            ys, _ = mok.moe_forward_mxfp8(mok.shards(x.cuda(), world), pack(full), p)
        else:
            ys, _ = mok.moe_forward(mok.shards(x.cuda(), world), *full, p, 0, mok.fwd_opts(mode=mok.MOK_MODE_STAGED))
        torch.cuda.synchronize()
        ok &= torch.equal(y, ys[rank])
        dist.barrier()
        grp.close()
        q.put((rank, bool(ok)))
    except Exception as e:  # reported to the parent
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.skipif(torch.cuda.device_count() < WORLD, reason="needs two GPUs")
@pytest.mark.parametrize("mxfp8", [False, True])
def test_ep_forward_over_two_gpus_matches_single_gpu(mxfp8):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, q, mxfp8)) for r in range(WORLD)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=120)
    assert all(v is True for v in got.values()), got
    assert all(p.exitcode == 0 for p in procs)
