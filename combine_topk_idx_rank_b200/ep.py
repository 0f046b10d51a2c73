"""Python binding of libep.so: argument marshalling only.

Every step of dispatch and combine runs in the library's sm_100a kernels;
torch provides device memory and the current CUDA stream.  There is no CPU
fallback: if libep.so is missing or cannot be loaded, importing this module
raises.

API (after the DeepEP calls described in "DeepEP V1 vs V2 comparative
analysis", sections 2-3, and the quantisation flags of "DeepEP communication
library guide v2.1"):

    ep_get_dispatch_layout(topk_idx, num_experts, num_ranks)
        -> (num_tokens_per_rank, num_tokens_per_expert, is_token_in_rank)
    ep_dispatch(x, topk_idx, topk_weights, expert_alignment=1, quant=None, *,
                num_experts, num_ranks, ...)
        -> (recv_x, recv_scales, recv_topk_idx, recv_topk_weights, handle)
    ep_combine(y, handle, topk_weights) -> combined tokens [T, H] bf16
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import functools
import os
from typing import List, Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libep.so")

(EP_OK, EP_ERR_INVALID_ARG, EP_ERR_BAD_EXPERT_ID, EP_ERR_CAPACITY, EP_ERR_CUDA, EP_ERR_TIMEOUT,
 EP_ERR_NONFINITE) = range(7)
_QUANT = {None: 0, "none": 0, "fp8": 1, "int8": 2, "mxfp4": 3}

EXPORTED = ("ep_recv_capacity_bound", "ep_workspace_bytes", "ep_get_dispatch_layout", "ep_dispatch",
            "ep_combine", "ep_read_error", "ep_copy_recv_counts", "ep_status_string", "ep_dispatch_noalloc",
            "ep_dispatch_cached", "ep_dispatch_low_latency", "ep_combine_ex", "ep_group_limited_gating",
            "ep_write_padding_rows", "ep_route", "ep_pack_peer", "ep_receiver_layout", "ep_combine_peer",
            "ep_ipc_export", "ep_ipc_import", "ep_ipc_close")


class EPError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib.ep_status_string(status).decode()} (status {status})")


class _Opts(C.Structure):
    _fields_ = [("expert_alignment", C.c_int32), ("quant", C.c_int32), ("quant_size", C.c_int32),
                ("round_scale", C.c_int32), ("num_rounds", C.c_int32), ("scale_ue8m0", C.c_int32),
                ("cumulative_local_expert_recv_stats", C.c_void_p),
                ("event_pack_begin", C.c_void_p), ("event_pack_end", C.c_void_p), ("token_offset", C.c_int32)]


class _Handle(C.Structure):
    _fields_ = [("num_tokens", C.c_int32), ("num_topk", C.c_int32), ("num_experts", C.c_int32),
                ("num_ranks", C.c_int32), ("hidden", C.c_int32), ("expert_alignment", C.c_int32),
                ("num_rounds", C.c_int32), ("low_latency", C.c_int32), ("recv_capacity", C.c_int64),
                ("topk_idx", C.c_void_p), ("psum_num_recv_tokens_per_expert", C.c_void_p),
                ("num_recv_tokens_per_expert", C.c_void_p), ("recv_src_metadata", C.c_void_p),
                ("dst_buffer_slot_idx", C.c_void_p), ("err", C.c_void_p)]


def _load(path: str = _LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(f"libep.so not found at {path}; build it with "
                          "`python -m combine_topk_idx_rank_b200.build`")
    L = C.CDLL(path)
    p, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    L.ep_recv_capacity_bound.argtypes = [i32, i32, i32, i32]
    L.ep_recv_capacity_bound.restype = i64
    L.ep_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.ep_workspace_bytes.restype = sz
    L.ep_get_dispatch_layout.argtypes = [p, i32, i32, i32, i32, p, p, p, p, p, sz, p]
    L.ep_get_dispatch_layout.restype = C.c_int
    L.ep_dispatch.argtypes = [p, i32, i32, p, p, i32, i32, i32, C.POINTER(_Opts), p, p, p, p, i64,
                              C.POINTER(_Handle), p, p, p, p, sz, p]
    L.ep_dispatch.restype = C.c_int
    L.ep_dispatch_cached.argtypes = [p, C.POINTER(_Handle), C.POINTER(_Opts), p, p, p]
    L.ep_dispatch_cached.restype = C.c_int
    L.ep_dispatch_low_latency.argtypes = [p, i32, i32, p, p, i32, i32, i32, i32, C.POINTER(_Opts), p, p, p, p,
                                          p, p, C.POINTER(_Handle), p, sz, p]
    L.ep_dispatch_low_latency.restype = C.c_int
    L.ep_combine_ex.argtypes = [p, p, i32, i32, C.POINTER(_Handle), p, p, p, p]
    L.ep_combine_ex.restype = C.c_int
    L.ep_combine.argtypes = [p, C.POINTER(_Handle), p, p, p]
    L.ep_combine.restype = C.c_int
    L.ep_read_error.argtypes = [p, p, C.POINTER(C.c_int32)]
    L.ep_read_error.restype = C.c_int
    L.ep_copy_recv_counts.argtypes = [C.POINTER(_Handle), p, p, C.POINTER(C.c_int64)]
    L.ep_copy_recv_counts.restype = C.c_int
    L.ep_group_limited_gating.argtypes = [p, i32, i32, i32, i32, i32, p, p, p, p]
    L.ep_group_limited_gating.restype = C.c_int
    L.ep_write_padding_rows.argtypes = [p, p, i32, p, i64, p, i64, p, p, i32, p, i64, p]
    L.ep_write_padding_rows.restype = C.c_int
    L.ep_route.argtypes = [p, p, i32, i32, i32, i32, i32, i32, p, p, i64, C.POINTER(_Handle), p, sz, p]
    L.ep_route.restype = C.c_int
    L.ep_pack_peer.argtypes = [p, C.POINTER(_Handle), p, p, p, i32, i32, i32, C.POINTER(_Opts), p, p, p, p, p, i64, p]
    L.ep_pack_peer.restype = C.c_int
    L.ep_receiver_layout.argtypes = [p, i32, i32, i32, i32, p, p, p]
    L.ep_receiver_layout.restype = C.c_int
    L.ep_combine_peer.argtypes = [p, C.POINTER(_Handle), p, i32, i32, i32, p, p, i64, p]
    L.ep_combine_peer.restype = C.c_int
    L.ep_ipc_export.argtypes = [p, p, C.POINTER(i64)]
    L.ep_ipc_export.restype = C.c_int
    L.ep_ipc_import.argtypes = [p, C.POINTER(p)]
    L.ep_ipc_import.restype = C.c_int
    L.ep_ipc_close.argtypes = [p]
    L.ep_ipc_close.restype = C.c_int
    L.ep_status_string.argtypes = [C.c_int]
    L.ep_status_string.restype = C.c_char_p
    return L


_lib = _load()


def library_path() -> str:
    return _LIB_PATH


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return C.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(status: int, what: str):
    if status != EP_OK:
        raise EPError(status, what)


def recv_capacity_bound(T: int, K: int, E: int, A: int) -> int:
    return int(_lib.ep_recv_capacity_bound(T, K, E, A))


def workspace_bytes(T: int, K: int, E: int, R: int) -> int:
    return int(_lib.ep_workspace_bytes(T, K, E, R))


def _on_tensor_device(fn):
    """Runs a call with its first argument's GPU as the current device, so that
    the library launches on the device whose stream it is given."""
    @functools.wraps(fn)
    def call(*args, **kw):
        t = args[0] if args else None
        if isinstance(t, torch.Tensor) and t.is_cuda:
            with torch.cuda.device(t.device):
                return fn(*args, **kw)
        return fn(*args, **kw)
    return call


def _need_cuda(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@dataclasses.dataclass
class EPHandle:
    """Routing metadata of one dispatch, reused by combine (EPHandle)."""
    num_tokens: int
    num_topk: int
    num_experts: int
    num_ranks: int
    hidden: int
    expert_alignment: int
    num_rounds: int
    recv_capacity: int
    topk_idx: torch.Tensor                          # [T, K] int32 copy
    psum_num_recv_tokens_per_expert: torch.Tensor   # [E] int32
    num_recv_tokens_per_expert: torch.Tensor        # [E] int32 (unaligned)
    recv_src_metadata: torch.Tensor                 # [cap, 2] int32 (t, k)
    dst_buffer_slot_idx: torch.Tensor               # [T, K] int32
    err: torch.Tensor                               # [1] int32
    num_recv_tokens_per_expert_list: Optional[List[int]] = None
    num_recv_rows: Optional[int] = None
    low_latency: int = 0

    def _c(self) -> _Handle:
        h = _Handle()
        h.num_tokens, h.num_topk, h.num_experts = self.num_tokens, self.num_topk, self.num_experts
        h.num_ranks, h.hidden, h.expert_alignment = self.num_ranks, self.hidden, self.expert_alignment
        h.num_rounds, h.recv_capacity = self.num_rounds, self.recv_capacity
        h.low_latency = self.low_latency
        h.topk_idx = self.topk_idx.data_ptr()
        h.psum_num_recv_tokens_per_expert = self.psum_num_recv_tokens_per_expert.data_ptr()
        h.num_recv_tokens_per_expert = self.num_recv_tokens_per_expert.data_ptr()
        h.recv_src_metadata = self.recv_src_metadata.data_ptr()
        h.dst_buffer_slot_idx = self.dst_buffer_slot_idx.data_ptr()
        h.err = self.err.data_ptr()
        return h

    def read_error(self) -> int:
        st = C.c_int32(0)
        with torch.cuda.device(self.err.device):
            _check(_lib.ep_read_error(_ptr(self.err), _stream(self.err.device), C.byref(st)), "ep_read_error")
        return st.value

    def check(self):
        st = self.read_error()
        if st != EP_OK:
            raise EPError(st, "device")


@dataclasses.dataclass
class DispatchBuffers:
    """Preallocated outputs of ep_dispatch for a fixed shape (reusable)."""
    recv_x: torch.Tensor
    recv_scales: Optional[torch.Tensor]
    recv_topk_idx: torch.Tensor
    recv_topk_weights: torch.Tensor
    handle: EPHandle
    workspace: torch.Tensor
    quant: Optional[str]
    quant_size: int


def _recv_tensors(rows: int, H: int, q: Optional[str], quant_size: int, scale_ue8m0: bool, dev):
    """recv_x and recv_scales for `rows` received rows: bf16 rows; FP8 e4m3 /
    int8 codes; or MXFP4 (two E2M1 codes per byte, uint8 [rows, H/2]).  Scales
    are fp32, or UE8M0 bytes (uint8) with scale_ue8m0 and always for MXFP4."""
    if q is None:
        return torch.empty((rows, H), dtype=torch.bfloat16, device=dev), None
    if q == "mxfp4":
        return (torch.empty((rows, H // 2), dtype=torch.uint8, device=dev),
                torch.empty((rows, H // 32), dtype=torch.uint8, device=dev))
    codes = torch.empty((rows, H), dtype=torch.float8_e4m3fn if q == "fp8" else torch.int8, device=dev)
    sdt = torch.uint8 if scale_ue8m0 else torch.float32
    return codes, torch.empty((rows, H // quant_size), dtype=sdt, device=dev)


def alloc_dispatch_buffers(num_tokens: int, hidden: int, num_topk: int, num_experts: int,
                           num_ranks: int, expert_alignment: int = 1, quant: Optional[str] = None,
                           quant_size: int = 128, num_rounds: int = 1,
                           recv_capacity: Optional[int] = None,
                           device: Optional[torch.device] = None,
                           scale_ue8m0: bool = False) -> DispatchBuffers:
    T, H, K, E, R, A = num_tokens, hidden, num_topk, num_experts, num_ranks, expert_alignment
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    cap = recv_capacity_bound(T, K, E, A) if recv_capacity is None else int(recv_capacity)
    q = None if quant in (None, "none") else quant
    recv_x, recv_scales = _recv_tensors(cap, H, q, quant_size, scale_ue8m0, dev)
    i32 = dict(dtype=torch.int32, device=dev)
    handle = EPHandle(T, K, E, R, H, A, num_rounds, cap,
                      topk_idx=torch.empty((T, K), **i32),
                      psum_num_recv_tokens_per_expert=torch.empty((E,), **i32),
                      num_recv_tokens_per_expert=torch.empty((E,), **i32),
                      recv_src_metadata=torch.empty((max(cap, 1), 2), **i32),
                      dst_buffer_slot_idx=torch.empty((T, K), **i32),
                      err=torch.zeros((1,), **i32))
    ws = torch.empty((max(workspace_bytes(T, K, E, R), 256),), dtype=torch.uint8, device=dev)
    return DispatchBuffers(recv_x, recv_scales, torch.empty((max(cap, 1), K), **i32),
                           torch.empty((max(cap, 1), K), dtype=torch.float32, device=dev), handle, ws,
                           q, quant_size)


@_on_tensor_device
def ep_get_dispatch_layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int,
                           workspace: Optional[torch.Tensor] = None, check: bool = True):
    """Routing histogram: (num_tokens_per_rank [R] i32, num_tokens_per_expert [E] i32,
    is_token_in_rank [T, R] bool)."""
    _need_cuda(topk_idx, "topk_idx", torch.int64)
    T, K = topk_idx.shape
    dev = topk_idx.device
    ntpr = torch.empty((num_ranks,), dtype=torch.int32, device=dev)
    ntpe = torch.empty((num_experts,), dtype=torch.int32, device=dev)
    itr = torch.empty((T, num_ranks), dtype=torch.bool, device=dev)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    nbytes = workspace_bytes(T, K, num_experts, num_ranks)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=dev)
    st = _lib.ep_get_dispatch_layout(_ptr(topk_idx), T, K, num_experts, num_ranks, _ptr(ntpr), _ptr(ntpe),
                                     _ptr(itr), _ptr(err), _ptr(workspace), workspace.numel(), _stream(dev))
    _check(st, "ep_get_dispatch_layout")
    if check:
        s = C.c_int32(0)
        _check(_lib.ep_read_error(_ptr(err), _stream(dev), C.byref(s)), "ep_read_error")
        if s.value:
            raise EPError(s.value, "ep_get_dispatch_layout")
    return ntpr, ntpe, itr


def _dispatch_cached(x, handle: EPHandle, quant, quant_size, round_scale, num_rounds, buffers, events,
                     scale_ue8m0=False):
    h = handle
    if tuple(x.shape) != (h.num_tokens, h.hidden):
        raise ValueError("x must be [num_tokens, hidden] of the handle")
    q = None if quant in (None, "none") else quant
    if buffers is None:
        buffers = alloc_dispatch_buffers(h.num_tokens, h.hidden, h.num_topk, h.num_experts, h.num_ranks,
                                         h.expert_alignment, q, quant_size, num_rounds, h.recv_capacity, x.device,
                                         scale_ue8m0)
    if buffers.recv_x.shape[0] != h.recv_capacity:
        raise ValueError("recv_x must have the handle's recv_capacity rows")
    opts = _Opts(h.expert_alignment, _QUANT[q], quant_size if q else 0, int(bool(round_scale)), num_rounds,
                 int(bool(scale_ue8m0)),
                 None, None if events is None else events[0].cuda_event,
                 None if events is None else events[1].cuda_event)
    st = _lib.ep_dispatch_cached(_ptr(x), C.byref(h._c()), C.byref(opts), _ptr(buffers.recv_x),
                                 _ptr(buffers.recv_scales), _stream(x.device))
    _check(st, "ep_dispatch_cached")
    recv_x, recv_scales = buffers.recv_x, buffers.recv_scales
    if h.num_recv_rows is not None:
        recv_x = recv_x[:h.num_recv_rows]
        if recv_scales is not None:
            recv_scales = recv_scales[:h.num_recv_rows]
    return recv_x, recv_scales, None, None, h


@_on_tensor_device
def ep_dispatch(x: torch.Tensor, topk_idx: Optional[torch.Tensor] = None,
                topk_weights: Optional[torch.Tensor] = None, expert_alignment: int = 1,
                quant: Optional[str] = None, *, num_experts: Optional[int] = None,
                num_ranks: Optional[int] = None, quant_size: int = 128, round_scale: bool = False,
                num_rounds: int = 1, do_cpu_sync: bool = True,
                recv_capacity: Optional[int] = None, buffers: Optional[DispatchBuffers] = None,
                cumulative_local_expert_recv_stats: Optional[torch.Tensor] = None,
                layout_out: Optional[tuple] = None, events: Optional[tuple] = None,
                handle: Optional[EPHandle] = None, scale_ue8m0: bool = False, token_offset: int = 0):
    """Dispatch: returns (recv_x, recv_scales, recv_topk_idx, recv_topk_weights, handle).

    ``token_offset`` is added to the token index of recv_src_metadata (tokens
    [o, o + T) of a batch that spans several GPUs).

    With ``do_cpu_sync`` the call waits for the GPU, checks the status word and
    trims the outputs to the rows received (``handle.num_recv_rows``); without
    it the outputs have ``recv_capacity`` rows and nothing waits.

    Cached mode: pass ``handle=`` (from an earlier call) and no topk_idx /
    topk_weights; x is re-packed with the cached routing, nothing waits, and
    recv_topk_idx / recv_topk_weights come back as None.
    """
    _need_cuda(x, "x", torch.bfloat16)
    if handle is not None:
        if topk_idx is not None or topk_weights is not None:
            raise ValueError("cached dispatch takes the routing from the handle")
        return _dispatch_cached(x, handle, quant, quant_size, round_scale, num_rounds, buffers, events,
                                scale_ue8m0)
    if topk_idx is None or topk_weights is None or num_experts is None or num_ranks is None:
        raise ValueError("topk_idx, topk_weights, num_experts and num_ranks are required")
    _need_cuda(topk_idx, "topk_idx", torch.int64)
    _need_cuda(topk_weights, "topk_weights", torch.float32)
    T, H = x.shape
    K = topk_idx.shape[1]
    if topk_idx.shape[0] != T or tuple(topk_weights.shape) != (T, K):
        raise ValueError("x, topk_idx and topk_weights disagree on the token count / top-k")
    q = None if quant in (None, "none") else quant
    if q is not None and quant_size not in (16, 32, 64, 128, 256, 512, H):
        raise ValueError(f"quant_size must be a group of 16..512 channels or hidden, got {quant_size}")
    if q == "mxfp4" and quant_size != 32:
        raise ValueError("MXFP4 uses groups of 32 channels")
    if buffers is None:
        buffers = alloc_dispatch_buffers(T, H, K, num_experts, num_ranks, expert_alignment, q,
                                         quant_size, num_rounds, recv_capacity, x.device, scale_ue8m0)
    b = buffers
    h = b.handle
    h.num_rounds = num_rounds
    opts = _Opts(expert_alignment, _QUANT[q], quant_size if q else 0, int(bool(round_scale)), num_rounds,
                 int(bool(scale_ue8m0)),
                 None if cumulative_local_expert_recv_stats is None
                 else cumulative_local_expert_recv_stats.data_ptr(),
                 None if events is None else events[0].cuda_event,
                 None if events is None else events[1].cuda_event, int(token_offset))
    ch = h._c()
    lay = layout_out or (None, None, None)
    stream = _stream(x.device)
    st = _lib.ep_dispatch(_ptr(x), T, H, _ptr(topk_idx), _ptr(topk_weights), K, num_experts, num_ranks,
                          C.byref(opts), _ptr(b.recv_x), _ptr(b.recv_scales), _ptr(b.recv_topk_idx),
                          _ptr(b.recv_topk_weights), b.recv_x.shape[0], C.byref(ch), _ptr(lay[0]),
                          _ptr(lay[1]), _ptr(lay[2]), _ptr(b.workspace), b.workspace.numel(), stream)
    _check(st, "ep_dispatch")
    h.num_tokens, h.num_topk, h.num_experts, h.num_ranks = ch.num_tokens, ch.num_topk, ch.num_experts, ch.num_ranks
    h.hidden, h.expert_alignment, h.recv_capacity = ch.hidden, ch.expert_alignment, ch.recv_capacity
    recv_x, recv_scales, rti, rtw = b.recv_x, b.recv_scales, b.recv_topk_idx, b.recv_topk_weights
    if do_cpu_sync:
        h.check()
        counts = (C.c_int32 * num_experts)()
        n = C.c_int64(0)
        _check(_lib.ep_copy_recv_counts(C.byref(ch), stream, counts, C.byref(n)), "ep_copy_recv_counts")
        h.num_recv_tokens_per_expert_list = list(counts)
        h.num_recv_rows = n.value
        recv_x, rti, rtw = recv_x[:n.value], rti[:n.value], rtw[:n.value]
        if recv_scales is not None:
            recv_scales = recv_scales[:n.value]
    return recv_x, recv_scales, rti, rtw, h


@_on_tensor_device
def ep_combine(y: torch.Tensor, handle: EPHandle, topk_weights: torch.Tensor,
               out: Optional[torch.Tensor] = None, *, y_scales: Optional[torch.Tensor] = None,
               quant_size: int = 128, shared: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Combine: out[t] = bf16(sum_k w[t,k] * y[dst_buffer_slot_idx[t,k]]), fp32 in k order.

    y may be bf16, or FP8 e4m3 / int8 codes with ``y_scales`` (one fp32 scale per
    ``quant_size`` channels; value = code * scale).  ``shared`` (bf16 [T, H]) is
    a shared expert's output the sum starts from.
    """
    _need_cuda(topk_weights, "topk_weights", torch.float32)
    h = handle
    if y.dim() == 3:                      # the low-latency layout [E, R*M, H]
        y = y.reshape(-1, y.shape[-1])
    if y.dtype == torch.bfloat16:
        yq, qs = 0, 0
    elif y.dtype in (torch.float8_e4m3fn, torch.int8):
        if y_scales is None:
            raise ValueError("quantised y needs y_scales")
        _need_cuda(y_scales, "y_scales", torch.float32)
        yq, qs = (1 if y.dtype == torch.float8_e4m3fn else 2), quant_size
    else:
        raise ValueError(f"unsupported y dtype {y.dtype}")
    _need_cuda(y, "y")
    if y.shape[1] != h.hidden or y.shape[0] > h.recv_capacity:
        raise ValueError("y must be [rows <= recv_capacity, hidden] in received-row order")
    if tuple(topk_weights.shape) != (h.num_tokens, h.num_topk):
        raise ValueError("topk_weights shape does not match the handle")
    if shared is not None:
        _need_cuda(shared, "shared", torch.bfloat16)
        if tuple(shared.shape) != (h.num_tokens, h.hidden):
            raise ValueError("shared must be [num_tokens, hidden]")
    if out is None:
        out = torch.empty((h.num_tokens, h.hidden), dtype=torch.bfloat16, device=y.device)
    ch = h._c()
    ch.recv_capacity = y.shape[0]
    if yq == 0 and shared is None:
        st = _lib.ep_combine(_ptr(y), C.byref(ch), _ptr(topk_weights), _ptr(out), _stream(y.device))
        _check(st, "ep_combine")
    else:
        st = _lib.ep_combine_ex(_ptr(y), _ptr(y_scales), yq, qs, C.byref(ch), _ptr(topk_weights), _ptr(shared),
                                _ptr(out), _stream(y.device))
        _check(st, "ep_combine_ex")
    return out


@_on_tensor_device
def ep_dispatch_low_latency(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                            num_max_dispatch_tokens_per_rank: int, num_experts: int, num_ranks: int,
                            quant: Optional[str] = None, *, quant_size: int = 128, round_scale: bool = False,
                            workspace: Optional[torch.Tensor] = None, buffers: Optional[dict] = None,
                            cumulative_local_expert_recv_stats: Optional[torch.Tensor] = None,
                            scale_ue8m0: bool = False, events: Optional[tuple] = None):
    """Low-latency (decode) dispatch into fixed-capacity per-expert buffers.

    Returns (recv_x [E, R*M, H], recv_scales [E, R*M, H/quant_size] or None,
    packed_recv_count [E], packed_recv_layout_range [E, R] int64, handle);
    entry (t,k) of source rank r for expert e is row r*M + p of expert e's
    block, p its position among rank r's entries for e.  ``events`` (two
    recorded torch.cuda.Event) bracket the pack kernel, as in ep_dispatch.
    """
    _need_cuda(x, "x", torch.bfloat16)
    _need_cuda(topk_idx, "topk_idx", torch.int64)
    _need_cuda(topk_weights, "topk_weights", torch.float32)
    T, H = x.shape
    K = topk_idx.shape[1]
    E, R, M = num_experts, num_ranks, num_max_dispatch_tokens_per_rank
    rows = E * R * M
    q = None if quant in (None, "none") else quant
    dev = x.device
    b = buffers
    if b is None:
        i32 = dict(dtype=torch.int32, device=dev)
        rx, rs = _recv_tensors(rows, H, q, quant_size, scale_ue8m0, dev)
        b = {"recv_x": rx, "recv_scales": rs,
             "recv_topk_idx": torch.empty((rows, K), **i32),
             "recv_topk_weights": torch.empty((rows, K), dtype=torch.float32, device=dev),
             "count": torch.empty((E,), **i32),
             "layout_range": torch.empty((E, R), dtype=torch.int64, device=dev),
             "handle": EPHandle(T, K, E, R, H, 1, 1, rows, torch.empty((T, K), **i32), torch.empty((E,), **i32),
                                torch.empty((E,), **i32), torch.empty((rows, 2), **i32),
                                torch.empty((T, K), **i32), torch.zeros((1,), **i32), low_latency=1)}
    h = b["handle"]
    nbytes = workspace_bytes(T, K, E, R)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=dev)
    opts = _Opts(1, _QUANT[q], quant_size if q else 0, int(bool(round_scale)), 1, int(bool(scale_ue8m0)),
                 None if cumulative_local_expert_recv_stats is None
                 else cumulative_local_expert_recv_stats.data_ptr(),
                 None if events is None else events[0].cuda_event,
                 None if events is None else events[1].cuda_event)
    ch = h._c()
    st = _lib.ep_dispatch_low_latency(_ptr(x), T, H, _ptr(topk_idx), _ptr(topk_weights), K, E, R, M, C.byref(opts),
                                      _ptr(b["recv_x"]), _ptr(b["recv_scales"]), _ptr(b["recv_topk_idx"]),
                                      _ptr(b["recv_topk_weights"]), _ptr(b["count"]), _ptr(b["layout_range"]),
                                      C.byref(ch), _ptr(workspace), workspace.numel(), _stream(dev))
    _check(st, "ep_dispatch_low_latency")
    h.recv_capacity, h.low_latency, h.expert_alignment = ch.recv_capacity, 1, 1
    rs = b["recv_scales"]
    return (b["recv_x"].view(E, R * M, -1), None if rs is None else rs.view(E, R * M, -1), b["count"],
            b["layout_range"], h)


@_on_tensor_device
def ep_group_limited_gating(logits: torch.Tensor, n_group: int = 32, topk_group: int = 4, per_group: int = 2, *,
                            out: Optional[tuple] = None, err: Optional[torch.Tensor] = None, check: bool = True):
    """Group-limited gating (DeepSeek-V3): router logits fp32 [T, E] ->
    (topk_idx int64 [T, K], topk_weights fp32 [T, K]), K = topk_group * per_group,
    ready for ep_dispatch.  The defaults are the DeepSeek-V3 setting (32 groups,
    top-4 groups, top-2 experts per group).  ``out`` = (topk_idx, topk_weights)
    preallocated; ``err`` an int32 [1] status word; with ``check`` the call
    waits and raises on a device error (EP_ERR_NONFINITE)."""
    _need_cuda(logits, "logits", torch.float32)
    T, E = logits.shape
    K = topk_group * per_group
    dev = logits.device
    if out is None:
        out = (torch.empty((T, K), dtype=torch.int64, device=dev), torch.empty((T, K), dtype=torch.float32, device=dev))
    idx, w = out
    _need_cuda(idx, "topk_idx", torch.int64)
    _need_cuda(w, "topk_weights", torch.float32)
    if tuple(idx.shape) != (T, K) or tuple(w.shape) != (T, K):
        raise ValueError("out tensors must be [T, topk_group * per_group]")
    if err is None:
        err = torch.zeros((1,), dtype=torch.int32, device=dev)
    st = _lib.ep_group_limited_gating(_ptr(logits), T, E, n_group, topk_group, per_group, _ptr(idx), _ptr(w),
                                      _ptr(err), _stream(dev))
    _check(st, "ep_group_limited_gating")
    if check:
        s = C.c_int32(0)
        _check(_lib.ep_read_error(_ptr(err), _stream(dev), C.byref(s)), "ep_read_error")
        if s.value:
            raise EPError(s.value, "ep_group_limited_gating")
    return idx, w


@_on_tensor_device
def ep_write_padding_rows(psum: torch.Tensor, counts: torch.Tensor, recv_x: torch.Tensor,
                          recv_scales: Optional[torch.Tensor] = None, recv_topk_idx: Optional[torch.Tensor] = None,
                          recv_topk_weights: Optional[torch.Tensor] = None,
                          recv_src_metadata: Optional[torch.Tensor] = None):
    """Writes the alignment padding rows of a receive layout (psum / counts per
    expert segment) as ep_dispatch writes them: zero rows and scales,
    recv_topk_idx -1, weight 0, metadata (-1, -1)."""
    _need_cuda(psum, "psum", torch.int32)
    _need_cuda(counts, "counts", torch.int32)
    _need_cuda(recv_x, "recv_x")
    cap = recv_x.shape[0]
    row_bytes = recv_x[0].numel() * recv_x.element_size() if cap else 16
    srb = 0 if recv_scales is None else recv_scales[0].numel() * recv_scales.element_size()
    K = recv_topk_idx.shape[1] if recv_topk_idx is not None else 1
    st = _lib.ep_write_padding_rows(_ptr(psum), _ptr(counts), psum.numel(), _ptr(recv_x), row_bytes,
                                    _ptr(recv_scales), srb, _ptr(recv_topk_idx), _ptr(recv_topk_weights), K,
                                    _ptr(recv_src_metadata), cap, _stream(recv_x.device))
    _check(st, "ep_write_padding_rows")


# ----------------------------------------------- multi-GPU through peer memory

@_on_tensor_device
def ep_route(topk_idx: torch.Tensor, topk_weights: torch.Tensor, num_experts: int, num_ranks: int, hidden: int,
             expert_alignment: int = 1, token_offset: int = 0, recv_capacity: Optional[int] = None):
    """Routing without the pack (ep_dispatch's handle, recv_topk_idx / weights
    and metadata): (recv_topk_idx, recv_topk_weights, handle)."""
    _need_cuda(topk_idx, "topk_idx", torch.int64)
    _need_cuda(topk_weights, "topk_weights", torch.float32)
    T, K = topk_idx.shape
    E, R, A = num_experts, num_ranks, expert_alignment
    dev = topk_idx.device
    cap = recv_capacity_bound(T, K, E, A) if recv_capacity is None else int(recv_capacity)
    i32 = dict(dtype=torch.int32, device=dev)
    h = EPHandle(T, K, E, R, hidden, A, 1, cap, torch.empty((T, K), **i32), torch.empty((E,), **i32),
                 torch.empty((E,), **i32), torch.empty((max(cap, 1), 2), **i32), torch.empty((T, K), **i32),
                 torch.zeros((1,), **i32))
    rti = torch.empty((max(cap, 1), K), **i32)
    rtw = torch.empty((max(cap, 1), K), dtype=torch.float32, device=dev)
    ws = torch.empty((max(workspace_bytes(T, K, E, R), 256),), dtype=torch.uint8, device=dev)
    ch = h._c()
    st = _lib.ep_route(_ptr(topk_idx), _ptr(topk_weights), T, K, E, R, A, int(token_offset), _ptr(rti), _ptr(rtw),
                       cap, C.byref(ch), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ep_route")
    h.workspace_keepalive = ws
    return rti, rtw, h


def pointer_table(tensors, device) -> torch.Tensor:
    """A device array of the given tensors' (or raw addresses') data pointers."""
    addrs = [t if isinstance(t, int) else (0 if t is None else t.data_ptr()) for t in tensors]
    return torch.tensor(addrs, dtype=torch.int64, device=device)


@_on_tensor_device
def ep_pack_peer(x: torch.Tensor, handle: EPHandle, send_topk_idx: torch.Tensor, send_topk_weights: torch.Tensor,
                 counts_all: torch.Tensor, G: int, g: int, expert_alignment: int, peer_recv_x: torch.Tensor,
                 peer_recv_scales: Optional[torch.Tensor], peer_recv_topk_idx: torch.Tensor,
                 peer_recv_topk_weights: torch.Tensor, peer_recv_metadata: torch.Tensor, peer_capacity: int,
                 quant: Optional[str] = None, quant_size: int = 128, round_scale: bool = False,
                 scale_ue8m0: bool = False):
    """Stores this GPU's rows straight into the receivers' layouts (peer_* are
    device pointer tables from pointer_table)."""
    q = None if quant in (None, "none") else quant
    opts = _Opts(1, _QUANT[q], quant_size if q else 0, int(bool(round_scale)), 1, int(bool(scale_ue8m0)),
                 None, None, None, 0)
    st = _lib.ep_pack_peer(_ptr(x), C.byref(handle._c()), _ptr(send_topk_idx), _ptr(send_topk_weights),
                           _ptr(counts_all), G, g, expert_alignment, C.byref(opts), _ptr(peer_recv_x),
                           _ptr(peer_recv_scales), _ptr(peer_recv_topk_idx), _ptr(peer_recv_topk_weights),
                           _ptr(peer_recv_metadata), int(peer_capacity), _stream(x.device))
    _check(st, "ep_pack_peer")


@_on_tensor_device
def ep_receiver_layout(counts_all: torch.Tensor, G: int, g: int, expert_alignment: int):
    """(psum [E/G], counts [E/G]) of this GPU's receive layout."""
    E = counts_all.shape[1]
    dev = counts_all.device
    psum = torch.empty((E // G,), dtype=torch.int32, device=dev)
    cnt = torch.empty((E // G,), dtype=torch.int32, device=dev)
    st = _lib.ep_receiver_layout(_ptr(counts_all), G, g, E, expert_alignment, _ptr(psum), _ptr(cnt), _stream(dev))
    _check(st, "ep_receiver_layout")
    return psum, cnt


@_on_tensor_device
def ep_combine_peer(peer_y: torch.Tensor, handle: EPHandle, counts_all: torch.Tensor, G: int, g: int,
                    expert_alignment: int, topk_weights: torch.Tensor, peer_capacity: int,
                    out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Each of this GPU's tokens reduced from its rows in the receivers' y."""
    if out is None:
        out = torch.empty((handle.num_tokens, handle.hidden), dtype=torch.bfloat16, device=topk_weights.device)
    st = _lib.ep_combine_peer(_ptr(peer_y), C.byref(handle._c()), _ptr(counts_all), G, g, expert_alignment,
                              _ptr(topk_weights), _ptr(out), int(peer_capacity), _stream(out.device))
    _check(st, "ep_combine_peer")
    return out


def ipc_export(t: torch.Tensor):
    """(64-byte handle, offset) of the allocation holding t, for another process."""
    h = C.create_string_buffer(64)
    off = C.c_int64(0)
    with torch.cuda.device(t.device):
        _check(_lib.ep_ipc_export(_ptr(t), h, C.byref(off)), "ep_ipc_export")
    return bytes(h.raw), off.value


def ipc_import(handle: bytes, offset: int, device) -> int:
    """The address, in this process, of an exported allocation plus offset."""
    base = C.c_void_p(0)
    with torch.cuda.device(device):
        _check(_lib.ep_ipc_import(C.create_string_buffer(handle, 64), C.byref(base)), "ep_ipc_import")
    return base.value + offset
