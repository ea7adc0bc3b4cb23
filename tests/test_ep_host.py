"""Host-side checks of the expert-parallel calls (no GPU): slot-buffer and
workspace sizes, argument errors caught before anything is enqueued, the
expert partition, and -- with two gloo ranks on the CPU -- the group's
exchange of buffer handles and its all-gather of the logits.

Source: MoK article (tahou.com), pull-dispatch paragraph (the expert's rank
pulls by {src_rank, src_index}) and push-combine paragraph (results go back
to the token's rank)."""
import ctypes
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import combine_device_top_b200 as mok


def test_ep_slot_and_workspace_sizes():
    L = mok.lib()
    S_r, H, k = 1024, 7168, 8
    ns = S_r * k
    rows = ns * H * 2
    exp_off = (rows + 255) // 256 * 256
    slots = exp_off + ns * (H // 128)
    assert mok.ep_slot_bytes(S_r, H, k) == (slots + 255) // 256 * 256 + 256
    assert L.mok_ep_slot_bytes(S_r, 100, k) == 0       # H % 128
    assert L.mok_ep_slot_bytes(S_r, H, 0) == 0
    ws = mok.ep_workspace_bytes(8192, H, 2048, 48, k)
    assert ws >= 8192 * k * (H + 2048) * 2               # every slot's row and h row
    assert mok.ep_workspace_bytes(8192, H, 2048, 0, k) > 0
    assert L.mok_ep_workspace_bytes(8192, H, 2048, -1, k) == 0


@pytest.mark.parametrize("E,G", [(384, 8), (384, 1), (10, 4), (3, 4), (1024, 64)])
def test_ep_partition_covers_every_expert_once(E, G):
    seen = []
    for g in range(G):
        e0, n = mok.ep_partition(E, G, g)
        assert n in (E // G, E // G + 1)
        seen += list(range(e0, e0 + n))
    assert seen == list(range(E))


def _fake_plan(T=16, E=8, k=2, R=2):
    p = mok.PlanT()
    p.T, p.E, p.k, p.R = T, E, k, R
    for f in ("counts", "offsets", "sched_src_rank", "sched_src_index", "row_slot", "pos", "topk_idx", "gates"):
        setattr(p, f, 0x100000)
    return p


def _fake_ep(G=2, g=0, e0=0, e_loc=4, sync=mok.MOK_EP_SYNC_DEVICE):
    return mok.ep_desc(G, g, e0, e_loc, [0x200000 + 0x1000 * h for h in range(G)],
                       [0x400000 + 0x1000 * h for h in range(G)], sync)


def _dispatch(p, ep, H=256, I=128, step=1, ws=0x800000, nbytes=1 << 40):
    L = mok.lib()
    rc = L.mok_ep_dispatch_ffn(ctypes.byref(p), ctypes.byref(ep), H, I, ctypes.c_void_p(0x10000),
                               ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), step, 0,
                               ctypes.c_void_p(ws), nbytes, None)
    return rc, L.mok_last_error_string().decode()


@pytest.mark.parametrize("change,code,word", [
    (dict(g=2), mok.MOK_ERR_INVALID_ARG, "rank"),               # g >= G
    (dict(G=4), mok.MOK_ERR_INVALID_ARG, "group size"),        # plan R != G
    (dict(e0=6, e_loc=4), mok.MOK_ERR_INVALID_ARG, "experts"),  # beyond E
    (dict(e_loc=-1), mok.MOK_ERR_INVALID_ARG, "experts"),
    (dict(sync=7), mok.MOK_ERR_INVALID_ARG, "sync"),
])
def test_ep_dispatch_rejects_bad_groups(change, code, word):
    args = dict(G=2, g=0, e0=0, e_loc=4, sync=mok.MOK_EP_SYNC_DEVICE)
    args.update(change)
    rc, msg = _dispatch(_fake_plan(), _fake_ep(**args))
    assert rc == code and word in msg, msg


def test_ep_dispatch_rejects_bad_buffers_and_steps():
    p = _fake_plan()
    ep = _fake_ep()
    ep.slots[1] = 0x400010                                     # not 256-byte aligned
    rc, msg = _dispatch(p, ep)
    assert rc == mok.MOK_ERR_UNSUPPORTED and "256-byte" in msg
    ep = _fake_ep()
    ep.x[0] = 0x200008                                         # not 16-byte aligned
    assert _dispatch(p, ep)[0] == mok.MOK_ERR_UNSUPPORTED
    ep = _fake_ep()
    ep.x[1] = None
    assert _dispatch(p, ep)[0] == mok.MOK_ERR_INVALID_ARG
    assert _dispatch(p, _fake_ep(), step=0)[0] == mok.MOK_ERR_INVALID_ARG
    assert _dispatch(p, _fake_ep(), H=200)[0] == mok.MOK_ERR_UNSUPPORTED
    rc, msg = _dispatch(p, _fake_ep(), nbytes=1024)
    assert rc == mok.MOK_ERR_WORKSPACE and "small" in msg


def test_ep_dispatch_checks_the_path():
    L = mok.lib()
    p = _fake_plan()
    ep = _fake_ep()
    ep.mxfp8 = 1                                               # bf16 call on an MXFP8 group
    rc, msg = _dispatch(p, ep)
    assert rc == mok.MOK_ERR_INVALID_ARG and "mxfp8" in msg
    ep.mxfp8 = 2
    assert _dispatch(p, ep)[0] == mok.MOK_ERR_INVALID_ARG
    ep = _fake_ep()
    rc = L.mok_ep_dispatch_ffn_mxfp8(ctypes.byref(p), ctypes.byref(ep), 256, 128, None, 1, 0,
                                     ctypes.c_void_p(0x800000), 1 << 40, None)
    assert rc == mok.MOK_ERR_INVALID_ARG                       # no weights
    w = mok.MxWeights(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    rc = L.mok_ep_dispatch_ffn_mxfp8(ctypes.byref(p), ctypes.byref(ep), 256, 128,
                                     ctypes.cast(ctypes.byref(w), ctypes.c_void_p), 1, 0,
                                     ctypes.c_void_p(0x800000), 1 << 40, None)
    assert rc == mok.MOK_ERR_INVALID_ARG                       # MXFP8 call on a bf16 group
    assert "mxfp8" in L.mok_last_error_string().decode()


def test_ep_workspace_holds_either_path():
    T, H, I, k = 512, 7168, 2048, 8
    ns = T * k
    ws = mok.ep_workspace_bytes(T, H, I, 48, k)
    sc = lambda K: (K // 128) * (((ns + 3) & ~3) + 4) * 4
    assert ws >= ns * (H + I) * 2 and ws >= ns * (H + I) + sc(H) + sc(I)


def test_ep_combine_rejects_bad_arguments():
    L = mok.lib()
    p = _fake_plan()

    def call(ep, y=0x900000, step=1, ws=0x800000):
        return L.mok_ep_combine(ctypes.byref(p), ctypes.byref(ep), 256, step, 0, ctypes.c_void_p(y),
                                ctypes.c_void_p(ws), 1 << 20, None)
    assert call(_fake_ep(), y=0) == mok.MOK_ERR_INVALID_ARG
    assert call(_fake_ep(), y=0x900004) == mok.MOK_ERR_UNSUPPORTED
    assert call(_fake_ep(), step=0) == mok.MOK_ERR_INVALID_ARG
    assert call(_fake_ep(), ws=0) == mok.MOK_ERR_WORKSPACE
    assert call(_fake_ep(g=3)) == mok.MOK_ERR_INVALID_ARG


def test_ipc_calls_reject_null_pointers():
    L = mok.lib()
    off = ctypes.c_size_t(0)
    assert L.mok_ipc_export(None, None, ctypes.byref(off)) == mok.MOK_ERR_INVALID_ARG
    assert L.mok_ipc_import(None, None) == mok.MOK_ERR_INVALID_ARG
    assert L.mok_ipc_close(None) == mok.MOK_ERR_INVALID_ARG


# ---------------------------------------------------------------- two gloo ranks
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fake_ipc(registry):
    """Handles that carry the address itself (each rank's buffers are host
    memory here): export -> (8 address bytes padded to the handle size, 0)."""
    def export(t):
        return t.data_ptr().to_bytes(8, "little") + bytes(mok.MOK_IPC_HANDLE_BYTES - 8), 0

    def import_(h):
        registry.append(h)
        return int.from_bytes(h[:8], "little")
    return export, import_, lambda base: None


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opened = []
        T, H, I, E, k = 8 * world, 128, 64, 10, 2
        grp = mok.EpGroup(T, H, I, E, k, device="cpu", ipc=_fake_ipc(opened))
        # every rank's addresses, to compare with what each rank mapped
        ptrs = [None] * world
        dist.all_gather_object(ptrs, (grp.x.data_ptr(), grp.slots.data_ptr()))
        logits = torch.full((grp.S_r, E), float(rank), dtype=torch.float32)
        full = grp.gather_logits(logits)
        q.put(dict(rank=rank, e0=grp.e0, e_loc=grp.e_loc, S_r=grp.S_r,
                   x=[grp.desc.x[h] for h in range(world)], slots=[grp.desc.slots[h] for h in range(world)],
                   want=ptrs, opened=len(opened), rows=[int(full[i * grp.S_r, 0]) for i in range(world)],
                   shape=tuple(full.shape), G=grp.desc.G, g=grp.desc.g, sync=grp.desc.sync))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ep_group_exchanges_handles_and_logits_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=120) for _ in range(world)), key=lambda d: d["rank"])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = got[0]["want"]
    e_next = 0
    for d in got:
        assert (d["G"], d["g"], d["sync"]) == (world, d["rank"], mok.MOK_EP_SYNC_DEVICE)
        assert d["e0"] == e_next
        e_next += d["e_loc"]
        # rank h's buffers as rank g maps them: its own directly, the others
        # from the exchanged handles (two per peer)
        assert d["x"] == [w[0] for w in want] and d["slots"] == [w[1] for w in want]
        assert d["opened"] == 2 * (world - 1)
        # the logits are gathered in rank order: rank h's rows carry h
        assert d["rows"] == list(range(world)) and d["shape"] == (8 * world, 10)
    assert e_next == 10


def _rank_dies(rank, world, port, q):
    """Rank 1 leaves before the group's handle exchange; rank 0's exchange
    must end with an error (the process group's timeout or the broken
    connection), not wait for ever."""
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    def leave(msg):
        q.put((rank, msg))
        q.close()
        q.join_thread()  # the message is out before the process ends
        os._exit(0)
    if rank == 1:
        leave("left")  # between steps, with nothing in flight
    try:
        mok.EpGroup(16, 128, 64, 4, 2, device="cpu", ipc=_fake_ipc([]))
        msg = "no error"
    except Exception as e:  # the failure seen on the host
        msg = type(e).__name__
    leave(msg)


def test_ep_group_reports_a_rank_that_left():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
    assert got[1] == "left"
    assert got[0] not in ("no error",), got
