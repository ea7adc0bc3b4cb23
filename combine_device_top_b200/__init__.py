"""Forward Mixture-of-Kittens MoE layer on B200 (sm_100a).

Thin Python binding over the C ABI in ``include/mok.h`` (``libmok.so``,
built in-tree by ``combine_device_top_b200.build``).  This module only
marshals arguments: PyTorch provides device memory and the current CUDA
stream, and every step of the layer runs in the library's CUDA kernels.
There is no CPU path: if ``libmok.so`` cannot be loaded, importing the
binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from functools import lru_cache

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOK_LIB_PATH selects another build of the same ABI (e.g. a debug build)
LIB_PATH = os.environ.get("MOK_LIB_PATH") or os.path.join(_PKG, "libmok.so")

MOK_OK = 0
MOK_ERR_INVALID_ARG = 1
MOK_ERR_UNSUPPORTED = 2
MOK_ERR_WORKSPACE = 3
MOK_ERR_CUDA = 4
MOK_ERR_TIMEOUT = 5
MOK_ERR_CAPACITY = 6
MOK_MODE_PERSISTENT = 0
MOK_MODE_STAGED = 1
MOK_MAX_SHARDS = 64
MOK_SLOTS_F32 = 0
MOK_SLOTS_BF16 = 1
MOK_SLOTS_F16S = 2
MOK_EP_SYNC_CALLER = 0
MOK_EP_SYNC_DEVICE = 1
MOK_IPC_HANDLE_BYTES = 64

# every entry point of include/mok.h
EXPORTS = (
    "mok_plan_workspace_bytes", "mok_plan", "mok_forward_workspace_bytes", "mok_moe_forward",
    "mok_get_status", "mok_last_error_string", "mok_gather", "mok_expert_ffn_workspace_bytes",
    "mok_expert_ffn", "mok_combine", "mok_forward_host_workspace_bytes", "mok_moe_forward_host",
    "mok_plan_noalloc", "mok_mxfp8_quantize_rows", "mok_quantize_weights_mxfp8",
    "mok_mxfp8_scale_rows", "mok_gather_mxfp8", "mok_expert_ffn_mxfp8_workspace_bytes", "mok_expert_ffn_mxfp8",
    "mok_two_wave_rows", "mok_minibatch_bounds", "mok_forward_host_batches_workspace_bytes",
    "mok_moe_forward_host_batches", "mok_router_weights_bytes", "mok_router_prepare", "mok_plan_router",
    "mok_backward_workspace_bytes", "mok_moe_backward", "mok_slot_bytes", "mok_slot_exp_offset",
    "mok_ep_slot_bytes", "mok_ep_workspace_bytes", "mok_ep_dispatch_ffn", "mok_ep_dispatch_ffn_mxfp8",
    "mok_ep_combine",
    "mok_ipc_export", "mok_ipc_import", "mok_ipc_close",
)


class MokError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"mok error {code}: {msg}")
        self.code = code


class PlanT(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("R", ctypes.c_int32),
                ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("sched_src_rank", ctypes.c_void_p), ("sched_src_index", ctypes.c_void_p),
                ("row_slot", ctypes.c_void_p), ("pos", ctypes.c_void_p),
                ("topk_idx", ctypes.c_void_p), ("gates", ctypes.c_void_p)]


class FwdOpts(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("ring_slots", ctypes.c_int32), ("dispatch_ctas", ctypes.c_int32),
                ("gemm_ctas", ctypes.c_int32), ("mxfp8", ctypes.c_int32), ("min_waves", ctypes.c_int32),
                ("save_for_backward", ctypes.c_int32), ("dispatch_warps", ctypes.c_int32), ("timeout_ns", ctypes.c_uint64)]


class EpT(ctypes.Structure):
    """``mok_ep_t``: one rank's view of an expert-parallel group."""
    _fields_ = [("G", ctypes.c_int32), ("g", ctypes.c_int32), ("e0", ctypes.c_int32), ("e_loc", ctypes.c_int32),
                ("sync", ctypes.c_int32), ("mxfp8", ctypes.c_int32),
                ("x", ctypes.c_void_p * MOK_MAX_SHARDS), ("slots", ctypes.c_void_p * MOK_MAX_SHARDS)]


@lru_cache(maxsize=1)
def lib() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m combine_device_top_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i32, sz, vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    L.mok_plan_workspace_bytes.argtypes = [i32, i32, i32]
    L.mok_plan_workspace_bytes.restype = sz
    L.mok_plan.argtypes = [vp, i32, i32, i32, i32, vp, sz, ctypes.POINTER(PlanT), vp]
    L.mok_forward_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(FwdOpts)]
    L.mok_forward_workspace_bytes.restype = sz
    L.mok_moe_forward.argtypes = [vp, i32, i32, vp, vp, vp, ctypes.POINTER(PlanT), i32, ctypes.POINTER(FwdOpts),
                                  vp, sz, vp, vp]
    L.mok_get_status.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_int)]
    L.mok_last_error_string.argtypes = []
    L.mok_last_error_string.restype = ctypes.c_char_p
    L.mok_gather.argtypes = [vp, i32, ctypes.POINTER(PlanT), vp, vp]
    L.mok_expert_ffn_workspace_bytes.argtypes = [i32, i32, i32]
    L.mok_expert_ffn_workspace_bytes.restype = sz
    L.mok_expert_ffn.argtypes = [vp, i32, i32, vp, vp, vp, ctypes.POINTER(PlanT), vp, sz, vp, vp]
    L.mok_combine.argtypes = [vp, i32, i32, ctypes.POINTER(PlanT), vp, vp]
    L.mok_forward_host_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(FwdOpts)]
    L.mok_forward_host_workspace_bytes.restype = sz
    L.mok_moe_forward_host.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, i32,
                                       ctypes.POINTER(FwdOpts), vp, sz, vp, vp]
    L.mok_plan_noalloc.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.mok_mxfp8_quantize_rows.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    L.mok_quantize_weights_mxfp8.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    L.mok_mxfp8_scale_rows.argtypes = [i32]
    L.mok_gather_mxfp8.argtypes = [vp, i32, ctypes.POINTER(PlanT), vp, vp, vp]
    L.mok_expert_ffn_mxfp8_workspace_bytes.argtypes = [i32, i32, i32]
    L.mok_expert_ffn_mxfp8_workspace_bytes.restype = sz
    L.mok_expert_ffn_mxfp8.argtypes = [vp, vp, i32, i32, vp, ctypes.POINTER(PlanT), vp, sz, vp, vp]
    L.mok_two_wave_rows.argtypes = [i32, i32, i32, i32]
    L.mok_slot_bytes.argtypes = [i32, i32, i32]
    L.mok_slot_bytes.restype = sz
    L.mok_slot_exp_offset.argtypes = [i32, i32]
    L.mok_slot_exp_offset.restype = sz
    L.mok_backward_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    L.mok_backward_workspace_bytes.restype = sz
    L.mok_moe_backward.argtypes = [vp, i32, i32, vp, vp, vp, ctypes.POINTER(PlanT), vp, sz, vp, vp, vp, vp, vp, vp, sz,
                                   vp]
    L.mok_router_weights_bytes.argtypes = [i32, i32]
    L.mok_router_weights_bytes.restype = sz
    L.mok_router_prepare.argtypes = [vp, i32, i32, vp, vp, vp]
    L.mok_plan_router.argtypes = [vp, i32, vp, vp, vp, i32, i32, i32, i32, vp, vp, sz, ctypes.POINTER(PlanT), vp]
    L.mok_forward_host_batches_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(FwdOpts)]
    L.mok_forward_host_batches_workspace_bytes.restype = sz
    L.mok_moe_forward_host_batches.argtypes = [i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, i32,
                                               ctypes.POINTER(FwdOpts), vp, sz, vp]
    L.mok_minibatch_bounds.argtypes = [ctypes.POINTER(PlanT), i32, i32, vp, i32, ctypes.POINTER(FwdOpts), vp, sz,
                                       vp, vp, i32, ctypes.POINTER(ctypes.c_int), vp]
    u32, u64 = ctypes.c_uint32, ctypes.c_uint64
    L.mok_ep_slot_bytes.argtypes = [i32, i32, i32]
    L.mok_ep_slot_bytes.restype = sz
    L.mok_ep_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    L.mok_ep_workspace_bytes.restype = sz
    L.mok_ep_dispatch_ffn.argtypes = [ctypes.POINTER(PlanT), ctypes.POINTER(EpT), i32, i32, vp, vp, vp, u32, u64, vp,
                                      sz, vp]
    L.mok_ep_dispatch_ffn_mxfp8.argtypes = [ctypes.POINTER(PlanT), ctypes.POINTER(EpT), i32, i32, vp, u32, u64, vp,
                                            sz, vp]
    L.mok_ep_combine.argtypes = [ctypes.POINTER(PlanT), ctypes.POINTER(EpT), i32, u32, u64, vp, vp, sz, vp]
    L.mok_ipc_export.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_size_t)]
    L.mok_ipc_import.argtypes = [vp, ctypes.POINTER(ctypes.c_void_p)]
    L.mok_ipc_close.argtypes = [vp]
    for n in ("mok_ep_dispatch_ffn", "mok_ep_dispatch_ffn_mxfp8", "mok_ep_combine", "mok_ipc_export",
              "mok_ipc_import", "mok_ipc_close"):
        getattr(L, n).restype = ctypes.c_int
    for n in ("mok_plan", "mok_moe_forward", "mok_get_status", "mok_gather", "mok_expert_ffn", "mok_combine",
              "mok_moe_forward_host", "mok_plan_noalloc", "mok_mxfp8_quantize_rows",
              "mok_quantize_weights_mxfp8", "mok_mxfp8_scale_rows", "mok_gather_mxfp8", "mok_expert_ffn_mxfp8",
              "mok_two_wave_rows", "mok_minibatch_bounds", "mok_moe_forward_host_batches", "mok_router_prepare",
              "mok_plan_router", "mok_moe_backward"):
        getattr(L, n).restype = ctypes.c_int
    return L


def _check(rc: int) -> None:
    if rc != MOK_OK:
        raise MokError(rc, lib().mok_last_error_string().decode())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr_array(tensors):
    arr = (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])
    return arr


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


@dataclass
class Plan:
    """Result of :func:`plan`: a C ``mok_plan_t`` plus the workspace it views."""
    c: PlanT
    ws: torch.Tensor

    def _view(self, ptr, n, dtype):
        # zero-copy view of a plan array (the storage is ``ws``)
        off = ptr - self.ws.data_ptr()
        itemsize = torch.empty((), dtype=dtype).element_size()
        return self.ws[off:off + n * itemsize].view(dtype)

    @property
    def ns(self):
        return self.c.T * self.c.k

    def counts(self):
        return self._view(self.c.counts, self.c.E, torch.int32)

    def offsets(self):
        return self._view(self.c.offsets, self.c.E + 1, torch.int32)

    def src_rank(self):
        return self._view(self.c.sched_src_rank, self.ns, torch.int32)

    def src_index(self):
        return self._view(self.c.sched_src_index, self.ns, torch.int32)

    def row_slot(self):
        return self._view(self.c.row_slot, self.ns, torch.int32)

    def pos(self):
        return self._view(self.c.pos, self.ns, torch.int32)

    def topk_idx(self):
        return self._view(self.c.topk_idx, self.ns, torch.int32).view(self.c.T, self.c.k)

    def gates(self):
        return self._view(self.c.gates, self.ns, torch.float32).view(self.c.T, self.c.k)


def plan(logits: torch.Tensor, top_k: int, R: int, ws: torch.Tensor | None = None, stream=None) -> Plan:
    """Steps 1-2: ``mok_plan`` on fp32 device logits [T, E]."""
    assert logits.is_cuda and logits.dtype == torch.float32 and logits.is_contiguous()
    T, E = logits.shape
    need = lib().mok_plan_workspace_bytes(T, E, top_k)
    if need == 0:
        raise MokError(MOK_ERR_INVALID_ARG, "invalid plan shape")
    if ws is None:
        ws = _workspace(need, logits.device)
    p = PlanT()
    _check(lib().mok_plan(ctypes.c_void_p(logits.data_ptr()), T, E, top_k, R, ctypes.c_void_p(ws.data_ptr()),
                          ws.numel(), ctypes.byref(p), _stream(stream)))
    return Plan(p, ws)


def router_prepare(w_r: torch.Tensor, stream=None):
    """``mok_router_prepare``: W_r [H, E] fp32 (device) -> (w_hi, w_lo), each
    [E rounded up to 64, H] bf16."""
    assert w_r.is_cuda and w_r.dtype == torch.float32 and w_r.is_contiguous()
    H, E = w_r.shape
    nbytes = lib().mok_router_weights_bytes(H, E)
    if nbytes == 0:
        raise MokError(MOK_ERR_UNSUPPORTED, "router shape")
    rows = nbytes // (2 * H)
    hi = torch.empty((rows, H), dtype=torch.bfloat16, device=w_r.device)
    lo = torch.empty_like(hi)
    _check(lib().mok_router_prepare(ctypes.c_void_p(w_r.data_ptr()), H, E, ctypes.c_void_p(hi.data_ptr()),
                                    ctypes.c_void_p(lo.data_ptr()), _stream(stream)))
    return hi, lo


def plan_router(x_shards, w_hi: torch.Tensor, w_lo: torch.Tensor, E: int, top_k: int, prior=None,
                logits_out: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None) -> Plan:
    """``mok_plan_router``: the plan with the router projection on the device."""
    R = len(x_shards)
    S_r, H = x_shards[0].shape
    T = S_r * R
    need = lib().mok_plan_workspace_bytes(T, E, top_k)
    if need == 0:
        raise MokError(MOK_ERR_INVALID_ARG, "invalid plan shape")
    if ws is None:
        ws = _workspace(need, x_shards[0].device)
    p = PlanT()
    _check(lib().mok_plan_router(_ptr_array(x_shards), H, ctypes.c_void_p(w_hi.data_ptr()),
                                 ctypes.c_void_p(w_lo.data_ptr()),
                                 ctypes.c_void_p(prior.data_ptr()) if prior is not None else None, T, E, top_k, R,
                                 ctypes.c_void_p(logits_out.data_ptr()) if logits_out is not None else None,
                                 ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.byref(p), _stream(stream)))
    return Plan(p, ws)


def mxfp8_quantize_rows(src: torch.Tensor, stream=None):
    """Blocks of 32 along each row of a [rows, K] bf16/fp32 tensor -> (q uint8, scales uint8)."""
    assert src.is_cuda and src.is_contiguous() and src.dtype in (torch.bfloat16, torch.float32)
    rows, K = src.shape
    q = torch.empty((rows, K), dtype=torch.uint8, device=src.device)
    s = torch.empty((rows, K // 32), dtype=torch.uint8, device=src.device)
    _check(lib().mok_mxfp8_quantize_rows(ctypes.c_void_p(src.data_ptr()), int(src.dtype == torch.float32), rows, K,
                                         ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(s.data_ptr()),
                                         _stream(stream)))
    return q, s


def quantize_weights_mxfp8(w: torch.Tensor, stream=None):
    """Weights [E, K, N] bf16 -> (q [E, K, N] uint8, scales [E, K/32, N] uint8), blocks along K."""
    assert w.is_cuda and w.is_contiguous() and w.dtype == torch.bfloat16
    E, K, N = w.shape
    q = torch.empty((E, K, N), dtype=torch.uint8, device=w.device)
    s = torch.empty((E, K // 32, N), dtype=torch.uint8, device=w.device)
    _check(lib().mok_quantize_weights_mxfp8(ctypes.c_void_p(w.data_ptr()), E, K, N, ctypes.c_void_p(q.data_ptr()),
                                            ctypes.c_void_p(s.data_ptr()), _stream(stream)))
    return q, s


def fwd_opts(mode: int = MOK_MODE_PERSISTENT, ring_slots: int = 0, dispatch_ctas: int = 0, gemm_ctas: int = 0,
             mxfp8: bool = False, timeout_ns: int = 0, min_waves: int = 0, save_for_backward: bool = False,
             dispatch_warps: int = 0) -> FwdOpts:
    return FwdOpts(mode, ring_slots, dispatch_ctas, gemm_ctas, int(mxfp8), min_waves, int(save_for_backward),
                   dispatch_warps, timeout_ns)


def forward_workspace_bytes(T, H, I, E, k, minibatch, opts: FwdOpts | None = None) -> int:
    return lib().mok_forward_workspace_bytes(T, H, I, E, k, minibatch, ctypes.byref(opts) if opts else None)


def shards(x: torch.Tensor, R: int):
    """R contiguous row blocks of a [T, H] tensor (views, no copy)."""
    return list(x.view(R, x.shape[0] // R, x.shape[1]).unbind(0))


def moe_forward(x_shards, w_gate, w_up, w_down, p: Plan, minibatch: int = 2560, opts: FwdOpts | None = None,
                y_shards=None, ws: torch.Tensor | None = None, stream=None):
    """Steps 3-5: ``mok_moe_forward``.  Returns (y_shards, ws)."""
    R = p.c.R
    # the library reads R pointers from each shard array
    assert len(x_shards) == R and (y_shards is None or len(y_shards) == R)
    for w in (w_gate, w_up, w_down):
        assert w.dtype == torch.bfloat16, "the weights are bf16"
    H = x_shards[0].shape[1]
    I = w_gate.shape[-1]
    dev = x_shards[0].device
    if y_shards is None:
        y_shards = [torch.empty_like(s) for s in x_shards]
    if ws is None:
        need = forward_workspace_bytes(p.c.T, H, I, p.c.E, p.c.k, minibatch, opts)
        if need == 0:
            raise MokError(MOK_ERR_INVALID_ARG, "invalid forward shape")
        ws = _workspace(need, dev)
    xa, ya = _ptr_array(x_shards), _ptr_array(y_shards)
    _check(lib().mok_moe_forward(xa, H, I, ctypes.c_void_p(w_gate.data_ptr()), ctypes.c_void_p(w_up.data_ptr()),
                                 ctypes.c_void_p(w_down.data_ptr()), ctypes.byref(p.c), minibatch,
                                 ctypes.byref(opts) if opts else None, ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                 ya, _stream(stream)))
    return y_shards, ws


class MxWeights(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("gate_scales", ctypes.c_void_p), ("up", ctypes.c_void_p),
                ("up_scales", ctypes.c_void_p), ("down", ctypes.c_void_p), ("down_scales", ctypes.c_void_p)]


def moe_forward_mxfp8(x_shards, pack, p: Plan, y_shards=None, ws: torch.Tensor | None = None, stream=None,
                      minibatch: int = 0, opts: FwdOpts | None = None):
    """The forward layer on the MXFP8 path.  ``pack`` = (qg, sg, qu, su, qd,
    sd) from :func:`quantize_weights_mxfp8`.  Staged mode by default; pass
    ``opts=fwd_opts(mode=MOK_MODE_PERSISTENT, mxfp8=True)`` and a minibatch
    for the persistent kernel.  Returns (y_shards, ws)."""
    qg, sg, qu, su, qd, sd = pack
    R = p.c.R
    # the library reads R pointers from each shard array
    assert len(x_shards) == R and (y_shards is None or len(y_shards) == R)
    H = x_shards[0].shape[1]
    I = qg.shape[-1]
    dev = x_shards[0].device
    if opts is None:
        opts = fwd_opts(mode=MOK_MODE_STAGED, mxfp8=True)
    assert opts.mxfp8 == 1, "moe_forward_mxfp8 needs opts with mxfp8=True"
    if y_shards is None:
        y_shards = [torch.empty_like(s) for s in x_shards]
    if ws is None:
        need = forward_workspace_bytes(p.c.T, H, I, p.c.E, p.c.k, minibatch, opts)
        if need == 0:
            raise MokError(MOK_ERR_INVALID_ARG, "invalid forward shape")
        ws = _workspace(need, dev)
    w = MxWeights(qg.data_ptr(), sg.data_ptr(), qu.data_ptr(), su.data_ptr(), qd.data_ptr(), sd.data_ptr())
    _check(lib().mok_moe_forward(_ptr_array(x_shards), H, I, ctypes.cast(ctypes.byref(w), ctypes.c_void_p), None,
                                 None, ctypes.byref(p.c), minibatch, ctypes.byref(opts),
                                 ctypes.c_void_p(ws.data_ptr()), ws.numel(), _ptr_array(y_shards), _stream(stream)))
    return y_shards, ws


def two_wave_rows(I: int, gemm_ctas: int, tile_rows: int, tile_features: int) -> int:
    """``mok_two_wave_rows``: rows of two full waves of gate/up output tiles."""
    return lib().mok_two_wave_rows(I, gemm_ctas, tile_rows, tile_features)


def minibatch_bounds(p: Plan, H: int, I: int, minibatch: int, opts: FwdOpts, w_gate=None, ws=None, stream=None):
    """``mok_minibatch_bounds``: (first row of each minibatch, gate/up units of
    each) that mok_moe_forward uses for these arguments."""
    dev = p.ws.device
    if ws is None:
        ws = _workspace(forward_workspace_bytes(p.c.T, H, I, p.c.E, p.c.k, minibatch, opts), dev)
    cap = p.ns + 2
    row0 = (ctypes.c_int32 * cap)()
    units = (ctypes.c_int32 * cap)()
    n = ctypes.c_int(0)
    _check(lib().mok_minibatch_bounds(ctypes.byref(p.c), H, I, w_gate, minibatch, ctypes.byref(opts),
                                      ctypes.c_void_p(ws.data_ptr()), ws.numel(), row0, units, cap, ctypes.byref(n),
                                      _stream(stream)))
    return list(row0[:n.value]), list(units[:n.value])


def moe_backward(dy_shards, w_gate, w_up, w_down, p: Plan, fwd_ws: torch.Tensor, dx_shards=None, dw=None,
                 dlogits=None, ws: torch.Tensor | None = None, stream=None):
    """``mok_moe_backward``: the layer's gradients given dy (shards of [S_r, H]
    bf16).  ``fwd_ws`` is the workspace of a staged :func:`moe_forward` with
    ``save_for_backward``.  Returns (dx_shards, (dWg, dWu, dWd), dlogits, ws)."""
    R = p.c.R
    assert len(dy_shards) == R and (dx_shards is None or len(dx_shards) == R)
    H = dy_shards[0].shape[1]
    I = w_gate.shape[-1]
    E, T, k = p.c.E, p.c.T, p.c.k
    dev = dy_shards[0].device
    for w in (w_gate, w_up, w_down):
        assert w.dtype == torch.bfloat16, "the weights are bf16"
    if dx_shards is None:
        dx_shards = [torch.empty_like(s) for s in dy_shards]
    if dw is None:
        dw = (torch.empty((E, H, I), dtype=torch.bfloat16, device=dev),
              torch.empty((E, H, I), dtype=torch.bfloat16, device=dev),
              torch.empty((E, I, H), dtype=torch.bfloat16, device=dev))
    if dlogits is None:
        dlogits = torch.empty((T, E), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(lib().mok_backward_workspace_bytes(T, H, I, E, k), dev)
    _check(lib().mok_moe_backward(_ptr_array(dy_shards), H, I, ctypes.c_void_p(w_gate.data_ptr()),
                                  ctypes.c_void_p(w_up.data_ptr()), ctypes.c_void_p(w_down.data_ptr()),
                                  ctypes.byref(p.c), ctypes.c_void_p(fwd_ws.data_ptr()), fwd_ws.numel(),
                                  _ptr_array(dx_shards), *(ctypes.c_void_p(t.data_ptr()) for t in dw),
                                  ctypes.c_void_p(dlogits.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                  _stream(stream)))
    return dx_shards, dw, dlogits, ws


def get_status(ws: torch.Tensor, stream=None) -> int:
    code = ctypes.c_int(-1)
    _check(lib().mok_get_status(ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream), ctypes.byref(code)))
    return code.value


def last_error() -> str:
    return lib().mok_last_error_string().decode()


def gather(x_shards, p: Plan, rows: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    assert len(x_shards) == p.c.R
    H = x_shards[0].shape[1]
    if rows is None:
        rows = torch.empty((p.ns, H), dtype=torch.bfloat16, device=x_shards[0].device)
    _check(lib().mok_gather(_ptr_array(x_shards), H, ctypes.byref(p.c), ctypes.c_void_p(rows.data_ptr()),
                            _stream(stream)))
    return rows


def gather_mxfp8(x_shards, p: Plan, rows_q=None, scales=None, stream=None):
    """The MXFP8 gather: (rows_q [N_s, H] uint8 E4M3, scales [H/128, sc_rows, 4] uint8 E8M0)."""
    assert len(x_shards) == p.c.R
    H = x_shards[0].shape[1]
    dev = x_shards[0].device
    if rows_q is None:
        rows_q = torch.empty((p.ns, H), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.zeros((H // 128, lib().mok_mxfp8_scale_rows(p.ns), 4), dtype=torch.uint8, device=dev)
    _check(lib().mok_gather_mxfp8(_ptr_array(x_shards), H, ctypes.byref(p.c), ctypes.c_void_p(rows_q.data_ptr()),
                                  ctypes.c_void_p(scales.data_ptr()), _stream(stream)))
    return rows_q, scales


def expert_ffn_mxfp8(rows_q, scales, pack, p: Plan, out: torch.Tensor | None = None, ws=None, stream=None):
    """The MXFP8 grouped SwiGLU FFN over mok_gather_mxfp8's output; pack =
    (qg, sg, qu, su, qd, sd).  Returns (out [T*k, H] bf16 slot-indexed, ws)."""
    qg, sg, qu, su, qd, sd = pack
    H = rows_q.shape[1]
    I = qg.shape[-1]
    if out is None:
        out = torch.empty((p.ns, H), dtype=torch.bfloat16, device=rows_q.device)
    assert out.dtype == torch.bfloat16
    if ws is None:
        ws = _workspace(lib().mok_expert_ffn_mxfp8_workspace_bytes(p.ns, I, p.c.E), rows_q.device)
    w = MxWeights(qg.data_ptr(), sg.data_ptr(), qu.data_ptr(), su.data_ptr(), qd.data_ptr(), sd.data_ptr())
    _check(lib().mok_expert_ffn_mxfp8(ctypes.c_void_p(rows_q.data_ptr()), ctypes.c_void_p(scales.data_ptr()), H, I,
                                      ctypes.cast(ctypes.byref(w), ctypes.c_void_p), ctypes.byref(p.c),
                                      ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.c_void_p(out.data_ptr()),
                                      _stream(stream)))
    return out, ws


def expert_ffn(rows, w_gate, w_up, w_down, p: Plan, out: torch.Tensor | None = None, ws=None, stream=None):
    """Grouped SwiGLU FFN over expert-major rows; returns (out, ws): ``out`` is
    the slot-indexed MOK_SLOTS_F16S buffer (uint8, ``mok_slot_bytes`` bytes:
    [T*k, H] fp16, then [T*k, H/128] int8 block exponents)."""
    H = rows.shape[1]
    I = w_gate.shape[-1]
    for w in (w_gate, w_up, w_down):
        assert w.dtype == torch.bfloat16, "the weights are bf16"
    if out is None:
        out = torch.empty(lib().mok_slot_bytes(p.ns, H, MOK_SLOTS_F16S), dtype=torch.uint8, device=rows.device)
    assert out.dtype == torch.uint8 and out.numel() >= lib().mok_slot_bytes(p.ns, H, MOK_SLOTS_F16S)
    if ws is None:
        ws = _workspace(lib().mok_expert_ffn_workspace_bytes(p.ns, I, p.c.E), rows.device)
    _check(lib().mok_expert_ffn(ctypes.c_void_p(rows.data_ptr()), H, I, ctypes.c_void_p(w_gate.data_ptr()),
                                ctypes.c_void_p(w_up.data_ptr()), ctypes.c_void_p(w_down.data_ptr()),
                                ctypes.byref(p.c), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                ctypes.c_void_p(out.data_ptr()), _stream(stream)))
    return out, ws


def combine(out: torch.Tensor, p: Plan, y_shards, stream=None):
    """y = fixed-order gate-weighted sum of the per-slot outputs, fp32 accumulation.  ``out``: fp32
    or bf16 [T*k, H], or a uint8 MOK_SLOTS_F16S buffer (then ``H`` comes from the y shards)."""
    assert out.dtype in (torch.float32, torch.bfloat16, torch.uint8) and len(y_shards) == p.c.R
    H = y_shards[0].shape[-1]
    dt = {torch.float32: MOK_SLOTS_F32, torch.bfloat16: MOK_SLOTS_BF16, torch.uint8: MOK_SLOTS_F16S}[out.dtype]
    _check(lib().mok_combine(ctypes.c_void_p(out.data_ptr()), dt, H, ctypes.byref(p.c), _ptr_array(y_shards),
                             _stream(stream)))
    return y_shards


def forward_host_workspace_bytes(T, H, I, E, k, minibatch, opts: FwdOpts | None = None) -> int:
    return lib().mok_forward_host_workspace_bytes(T, H, I, E, k, minibatch, ctypes.byref(opts) if opts else None)


def _host_weights(w_gate, w_up, w_down):
    if isinstance(w_gate, tuple):
        qg, sg, qu, su, qd, sd = w_gate
        mx = MxWeights(qg.data_ptr(), sg.data_ptr(), qu.data_ptr(), su.data_ptr(), qd.data_ptr(), sd.data_ptr())
        return qg.shape[-1], (ctypes.cast(ctypes.byref(mx), ctypes.c_void_p), None, None), mx
    return w_gate.shape[-1], tuple(ctypes.c_void_p(w.data_ptr()) for w in (w_gate, w_up, w_down)), None


def moe_forward_host(x_host: torch.Tensor, logits_host: torch.Tensor, top_k: int, R: int, w_gate, w_up, w_down,
                     minibatch: int, opts: FwdOpts | None, ws: torch.Tensor, y_host: torch.Tensor, stream=None):
    """End to end from host memory: ``mok_moe_forward_host``.  On the MXFP8
    path (``opts.mxfp8``) ``w_gate`` is the pack from :func:`quantize_weights_mxfp8`
    (qg, sg, qu, su, qd, sd) and ``w_up``/``w_down`` are None."""
    T, H = x_host.shape
    E = logits_host.shape[1]
    I, wptrs, keep = _host_weights(w_gate, w_up, w_down)
    _check(lib().mok_moe_forward_host(ctypes.c_void_p(x_host.data_ptr()), ctypes.c_void_p(logits_host.data_ptr()),
                                      T, H, I, E, top_k, R, *wptrs,
                                      minibatch, ctypes.byref(opts) if opts else None,
                                      ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                      ctypes.c_void_p(y_host.data_ptr()), _stream(stream)))
    del keep
    return y_host


def forward_host_batches_workspace_bytes(T, H, I, E, k, minibatch, opts: FwdOpts | None = None) -> int:
    return lib().mok_forward_host_batches_workspace_bytes(T, H, I, E, k, minibatch,
                                                          ctypes.byref(opts) if opts else None)


def moe_forward_host_batches(xs_host, logits_host, top_k: int, R: int, w_gate, w_up, w_down, minibatch: int,
                             opts: FwdOpts | None, ws: torch.Tensor, ys_host, stream=None):
    """``mok_moe_forward_host_batches``: lists of n host tensors (x [T, H] bf16,
    logits [T, E] fp32, y [T, H] bf16), copies overlapped with the compute."""
    n = len(xs_host)
    assert len(logits_host) == n and len(ys_host) == n
    if n == 0:
        return ys_host
    T, H = xs_host[0].shape
    E = logits_host[0].shape[1]
    I, wptrs, keep = _host_weights(w_gate, w_up, w_down)
    xa, la, ya = _ptr_array(xs_host), _ptr_array(logits_host), _ptr_array(ys_host)
    _check(lib().mok_moe_forward_host_batches(n, xa, la, ya, T, H, I, E, top_k, R, *wptrs, minibatch,
                                              ctypes.byref(opts) if opts else None, ctypes.c_void_p(ws.data_ptr()),
                                              ws.numel(), _stream(stream)))
    del keep
    return ys_host


# ---------------------------------------------------------------- expert parallelism
def ep_partition(E: int, G: int, g: int) -> tuple[int, int]:
    """Experts of rank g when E experts are split over G ranks in contiguous
    blocks, the first E % G ranks holding one more: (e0, e_loc)."""
    assert 0 <= g < G and E >= 0
    base, extra = divmod(E, G)
    e0 = g * base + min(g, extra)
    return e0, base + (1 if g < extra else 0)


def ep_slot_bytes(S_r: int, H: int, k: int) -> int:
    return lib().mok_ep_slot_bytes(S_r, H, k)


def ep_workspace_bytes(T: int, H: int, I: int, e_loc: int, k: int) -> int:
    return lib().mok_ep_workspace_bytes(T, H, I, e_loc, k)


def ep_desc(G: int, g: int, e0: int, e_loc: int, x_ptrs, slot_ptrs, sync: int = MOK_EP_SYNC_DEVICE,
            mxfp8: bool = False) -> EpT:
    """A ``mok_ep_t`` from the ranks' x and slot-buffer addresses (ints, as
    this GPU addresses them)."""
    assert len(x_ptrs) == G and len(slot_ptrs) == G and 1 <= G <= MOK_MAX_SHARDS
    d = EpT()
    d.G, d.g, d.e0, d.e_loc, d.sync, d.mxfp8 = G, g, e0, e_loc, sync, int(bool(mxfp8))
    for h in range(G):
        d.x[h] = x_ptrs[h]
        d.slots[h] = slot_ptrs[h]
    return d


def ep_dispatch_ffn(p: Plan, ep: EpT, w_gate, w_up, w_down, step: int, ws: torch.Tensor, timeout_ns: int = 0,
                    stream=None) -> None:
    """Rank ep.g's barrier, pull dispatch, grouped SwiGLU FFN and push of step
    ``step``; w_* are this rank's experts' weights ([e_loc, H, I] and [e_loc, I, H] bf16)."""
    H, I = w_gate.shape[-2], w_gate.shape[-1]
    for w in (w_gate, w_up, w_down):
        assert w.dtype == torch.bfloat16 and w.shape[0] == ep.e_loc, "the rank's bf16 weights"
    _check(lib().mok_ep_dispatch_ffn(ctypes.byref(p.c), ctypes.byref(ep), H, I, ctypes.c_void_p(w_gate.data_ptr()),
                                     ctypes.c_void_p(w_up.data_ptr()), ctypes.c_void_p(w_down.data_ptr()), step,
                                     timeout_ns, ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)))


def ep_dispatch_ffn_mxfp8(p: Plan, ep: EpT, pack, H: int, step: int, ws: torch.Tensor, timeout_ns: int = 0,
                          stream=None) -> None:
    """The MXFP8 path of :func:`ep_dispatch_ffn`; pack = (qg, sg, qu, su, qd,
    sd) of this rank's experts (:func:`quantize_weights_mxfp8`)."""
    qg, sg, qu, su, qd, sd = pack
    I = qg.shape[-1]
    assert qg.shape[0] == ep.e_loc and ep.mxfp8 == 1
    w = MxWeights(qg.data_ptr(), sg.data_ptr(), qu.data_ptr(), su.data_ptr(), qd.data_ptr(), sd.data_ptr())
    _check(lib().mok_ep_dispatch_ffn_mxfp8(ctypes.byref(p.c), ctypes.byref(ep), H, I,
                                           ctypes.cast(ctypes.byref(w), ctypes.c_void_p), step, timeout_ns,
                                           ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(stream)))


def ep_combine(p: Plan, ep: EpT, y: torch.Tensor, step: int, ws: torch.Tensor, timeout_ns: int = 0,
               stream=None) -> torch.Tensor:
    """Rank ep.g's barrier and combine of step ``step`` into y [S_r, H] bf16."""
    assert y.dtype == torch.bfloat16 and y.is_contiguous()
    _check(lib().mok_ep_combine(ctypes.byref(p.c), ctypes.byref(ep), y.shape[-1], step, timeout_ns,
                                ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                _stream(stream)))
    return y


def ipc_export(t: torch.Tensor) -> tuple[bytes, int]:
    """(handle bytes, byte offset) of the cudaMalloc allocation holding ``t``."""
    h = (ctypes.c_ubyte * MOK_IPC_HANDLE_BYTES)()
    off = ctypes.c_size_t(0)
    _check(lib().mok_ipc_export(ctypes.c_void_p(t.data_ptr()), h, ctypes.byref(off)))
    return bytes(h), off.value


def ipc_import(handle: bytes) -> int:
    """Base address (an int) of another process's allocation, mapped here."""
    assert len(handle) == MOK_IPC_HANDLE_BYTES
    buf = (ctypes.c_ubyte * MOK_IPC_HANDLE_BYTES).from_buffer_copy(handle)
    base = ctypes.c_void_p(0)
    _check(lib().mok_ipc_import(buf, ctypes.byref(base)))
    return base.value


def ipc_close(base: int) -> None:
    _check(lib().mok_ipc_close(ctypes.c_void_p(base)))


class EpGroup:
    """The expert-parallel forward on this process's GPU, one process per GPU
    under ``torch.distributed`` (rank g of G): rank g holds tokens [g*S_r,
    (g+1)*S_r) of a layer of T tokens and the experts ``ep_partition(E, G, g)``.

    At construction every rank allocates its token buffer ``x`` [S_r, H] and
    its slot buffer, exports both (CUDA IPC) and maps the other ranks' (an
    all-gather of the handles: plumbing, once).  :meth:`forward` then runs a
    step: an all-gather of the logits (so every rank builds the same plan),
    the plan, and the library's two calls (pull dispatch + FFN + push, then
    combine), with the group barriers on the device.  ``ipc`` replaces the
    (export, import, close) functions, e.g. by fakes in host-only tests.
    """

    def __init__(self, T: int, H: int, I: int, E: int, k: int, device=None, group=None, ipc=None,
                 mxfp8: bool = False):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.G = dist.get_world_size(group) if dist.is_initialized() else 1
        self.g = dist.get_rank(group) if dist.is_initialized() else 0
        assert T % self.G == 0, "T must split evenly over the ranks"
        self.T, self.H, self.I, self.E, self.k = T, H, I, E, k
        self.mxfp8 = bool(mxfp8)
        self.S_r = T // self.G
        self.e0, self.e_loc = ep_partition(E, self.G, self.g)
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.export, self.import_, self.close_ = ipc or (ipc_export, ipc_import, ipc_close)
        self.step = 0
        self._opened: list[int] = []
        self.x = torch.empty((self.S_r, H), dtype=torch.bfloat16, device=self.device)
        self.slots = torch.zeros(ep_slot_bytes(self.S_r, H, k), dtype=torch.uint8, device=self.device)
        self.ws = _workspace(ep_workspace_bytes(T, H, I, self.e_loc, k), self.device)
        xp, sp = self._exchange()
        self.desc = ep_desc(self.G, self.g, self.e0, self.e_loc, xp, sp, MOK_EP_SYNC_DEVICE, self.mxfp8)

    def _exchange(self):
        """Every rank's x and slot addresses as this GPU addresses them."""
        if self.G == 1:
            return [self.x.data_ptr()], [self.slots.data_ptr()]
        mine = (self.export(self.x), self.export(self.slots))
        allv = [None] * self.G
        self.dist.all_gather_object(allv, mine, group=self.group)
        xp, sp = [], []
        for h, ((xh, xo), (sh, so)) in enumerate(allv):
            if h == self.g:
                xp.append(self.x.data_ptr())
                sp.append(self.slots.data_ptr())
                continue
            bx, bs = self.import_(xh), self.import_(sh)
            self._opened += [bx, bs]
            xp.append(bx + xo)
            sp.append(bs + so)
        return xp, sp

    def gather_logits(self, logits_local: torch.Tensor) -> torch.Tensor:
        """[T, E] fp32: the ranks' [S_r, E] logits in rank order."""
        if self.G == 1:
            return logits_local
        out = torch.empty((self.T, self.E), dtype=logits_local.dtype, device=logits_local.device)
        self.dist.all_gather_into_tensor(out, logits_local.contiguous(), group=self.group)
        return out

    def forward(self, logits_local: torch.Tensor, w_gate, w_up, w_down, y: torch.Tensor | None = None,
                timeout_ns: int = 0, stream=None) -> torch.Tensor:
        """One step over the tokens in ``self.x``: returns y [S_r, H] bf16.
        w_*: this rank's experts' weights (MXFP8 group: w_gate is the pack of
        :func:`quantize_weights_mxfp8`, w_up and w_down None).  Everything,
        the all-gather of the logits included, is ordered on ``stream``
        (default: the current stream), after whatever wrote ``self.x`` there."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            self.step += 1
            p = plan(self.gather_logits(logits_local), self.k, self.G, stream=s)
            if self.mxfp8:
                ep_dispatch_ffn_mxfp8(p, self.desc, w_gate, self.H, self.step, self.ws, timeout_ns, s)
            else:
                ep_dispatch_ffn(p, self.desc, w_gate, w_up, w_down, self.step, self.ws, timeout_ns, s)
            if y is None:
                y = torch.empty((self.S_r, self.H), dtype=torch.bfloat16, device=self.device)
            return ep_combine(p, self.desc, y, self.step, self.ws, timeout_ns, s)

    def status(self, stream=None) -> int:
        return get_status(self.ws, stream)

    def close(self) -> None:
        """Unmap the other ranks' buffers.  Call it once every rank's last
        step has finished (synchronise, then a barrier of the group)."""
        for b in self._opened:
            self.close_(b)
        self._opened = []

