"""CPU oracle for MoE expert-parallel dispatch / combine (numpy front end).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product path.  The arithmetic lives
in ep_oracle.c (plain C, single-threaded); this module only marshals numpy
arrays.  It imports nothing from the CUDA package.

``use_threads(n)`` with n > 1 routes the row functions (dispatch rows and
combine) to the OpenMP build of the same source, which splits their token
loops across n threads; every token's arithmetic is unchanged.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import numpy as np

from . import build as _build

OK, INVALID_ARG, BAD_EXPERT_ID, CAPACITY, NONFINITE = 0, 1, 2, 3, 4
QUANT = {"none": 0, "fp8": 1, "int8": 2, "mxfp4": 3}


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"oracle {what}: status {status}")
        self.status = status


_lib = None
_lib_omp = None
_threads = 1


def lib():
    global _lib
    if _lib is None:
        _lib = _setup(C.CDLL(_build.build()))
    return _lib


def _rowlib():
    """The library the row functions call: the OpenMP build once use_threads(n > 1)."""
    global _lib_omp
    if _threads <= 1:
        return lib()
    if _lib_omp is None:
        _lib_omp = _setup(C.CDLL(_build.build_omp()))
    _lib_omp.oracle_threads(_threads)
    return _lib_omp


def use_threads(n: int) -> int:
    """Row functions run on n threads (1 = the single-threaded build); returns n."""
    global _threads
    _threads = max(1, int(n))
    return _rowlib().oracle_threads(0) if _threads > 1 else 1


def threads() -> int:
    return _threads


def _setup(L):
    """Declares the argument and result types of every oracle function."""
    p = C.c_void_p
    i32, i64 = C.c_int32, C.c_int64
    L.oracle_bf16_to_f32.argtypes = [C.c_uint16]
    L.oracle_bf16_to_f32.restype = C.c_float
    L.oracle_f32_to_bf16.argtypes = [C.c_float]
    L.oracle_f32_to_bf16.restype = C.c_uint16
    L.oracle_e4m3_to_f64.argtypes = [C.c_uint8]
    L.oracle_e4m3_to_f64.restype = C.c_double
    L.oracle_f32_to_e4m3.argtypes = [C.c_float]
    L.oracle_f32_to_e4m3.restype = C.c_uint8
    L.oracle_pow2_ceil.argtypes = [C.c_float]
    L.oracle_pow2_ceil.restype = C.c_float
    L.oracle_layout.argtypes = [p, i32, i32, i32, i32, p, p, p]
    L.oracle_layout.restype = C.c_int
    L.oracle_slots.argtypes = [p, p, i32, i32, i32, i32, i32, i64, p, p, p, p, p, p, p]
    L.oracle_slots.restype = C.c_int
    L.oracle_quantize_row.argtypes = [p, i32, i32, i32, i32, p, p]
    L.oracle_quantize_row.restype = C.c_int
    L.oracle_dispatch_rows.argtypes = [p, i32, i32, i32, p, i32, i32, i32, p, i64, p, p, i64]
    L.oracle_dispatch_rows.restype = C.c_int
    L.oracle_combine_rows.argtypes = [p, i64, i32, i32, i32, p, p, p, i64, p]
    L.oracle_combine_rows.restype = C.c_int
    L.oracle_round_tokens.argtypes = [i32, i32, i32, i32, p]
    L.oracle_round_tokens.restype = i64
    L.oracle_ll_slots.argtypes = [p, p, i32, i32, i32, i32, i32, p, p, p, p, p, p]
    L.oracle_ll_slots.restype = C.c_int
    L.oracle_combine_rows_q.argtypes = [p, p, i32, i32, i64, i32, i32, i32, p, p, p, p, i64, p]
    L.oracle_combine_rows_q.restype = C.c_int
    L.oracle_e2m1_to_f64.argtypes = [C.c_uint8]
    L.oracle_e2m1_to_f64.restype = C.c_double
    L.oracle_f32_to_e2m1.argtypes = [C.c_float]
    L.oracle_f32_to_e2m1.restype = C.c_uint8
    L.oracle_quantize_row_mx.argtypes = [p, i32, i32, i32, i32, i32, p, p]
    L.oracle_quantize_row_mx.restype = C.c_int
    L.oracle_dispatch_rows_mx.argtypes = [p, i32, i32, i32, p, i32, i32, i32, i32, p, i64, p, p, i64]
    L.oracle_dispatch_rows_mx.restype = C.c_int
    L.oracle_f32_to_e4m3_n.argtypes = [p, i64, p]
    L.oracle_f32_to_e4m3_n.restype = None
    L.oracle_f32_to_bf16_n.argtypes = [p, i64, p]
    L.oracle_f32_to_bf16_n.restype = None
    L.oracle_e4m3_to_f64_n.argtypes = [p, i64, p]
    L.oracle_e4m3_to_f64_n.restype = None
    L.oracle_group_limited_gating.argtypes = [p, i32, i32, i32, i32, i32, p, p]
    L.oracle_group_limited_gating.restype = C.c_int
    L.oracle_threads.argtypes = [C.c_int]
    L.oracle_threads.restype = C.c_int
    return L


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ numbers

def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    f = lib().oracle_bf16_to_f32
    return np.array([f(int(v)) for v in np.asarray(b).ravel()], dtype=np.float32).reshape(np.shape(b))


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    a = _c(x, np.float32)
    out = np.zeros(a.shape, np.uint16)
    lib().oracle_f32_to_bf16_n(_ptr(a), a.size, _ptr(out))
    return out


def e4m3_to_f64(c: np.ndarray) -> np.ndarray:
    a = _c(c, np.uint8)
    out = np.zeros(a.shape, np.float64)
    lib().oracle_e4m3_to_f64_n(_ptr(a), a.size, _ptr(out))
    return out


def f32_to_e4m3(x: np.ndarray) -> np.ndarray:
    a = _c(x, np.float32)
    out = np.zeros(a.shape, np.uint8)
    lib().oracle_f32_to_e4m3_n(_ptr(a), a.size, _ptr(out))
    return out


def pow2_ceil(s: float) -> float:
    return lib().oracle_pow2_ceil(float(s))


# ------------------------------------------------------------------- layout

def layout(topk_idx: np.ndarray, num_experts: int, num_ranks: int):
    ti = _c(topk_idx, np.int64)
    T, K = ti.shape
    ntpr = np.zeros(num_ranks, np.int32)
    ntpe = np.zeros(num_experts, np.int32)
    itr = np.zeros((T, num_ranks), np.uint8)
    st = lib().oracle_layout(_ptr(ti), T, K, num_experts, num_ranks, _ptr(ntpr), _ptr(ntpe), _ptr(itr))
    if st:
        raise OracleError(st, "layout")
    return {"num_tokens_per_rank": ntpr, "num_tokens_per_expert": ntpe,
            "is_token_in_rank": itr.astype(bool)}


def capacity_bound(T: int, K: int, E: int, A: int) -> int:
    return T * K + E * (A - 1)


def slots(topk_idx, topk_weights, num_experts: int, num_ranks: int, expert_alignment: int = 1,
          capacity: Optional[int] = None):
    ti = _c(topk_idx, np.int64)
    tw = _c(topk_weights, np.float32)
    T, K = ti.shape
    E, A = num_experts, expert_alignment
    cap = capacity_bound(T, K, E, A) if capacity is None else capacity
    psum = np.zeros(E, np.int32)
    cnt = np.zeros(E, np.int32)
    dst = np.zeros((T, K), np.int32)
    meta = np.zeros((max(cap, 1), 2), np.int32)
    rti = np.zeros((max(cap, 1), K), np.int32)
    rtw = np.zeros((max(cap, 1), K), np.float32)
    n = C.c_int64(0)
    st = lib().oracle_slots(_ptr(ti), _ptr(tw), T, K, E, num_ranks, A, cap, _ptr(psum), _ptr(cnt),
                            _ptr(dst), _ptr(meta), _ptr(rti), _ptr(rtw), C.byref(n))
    if st:
        raise OracleError(st, "slots")
    nr = n.value
    return {"psum_num_recv_tokens_per_expert": psum, "num_recv_tokens_per_expert": cnt,
            "dst_buffer_slot_idx": dst, "recv_src_metadata": meta[:nr],
            "recv_topk_idx": rti[:nr], "recv_topk_weights": rtw[:nr], "num_recv_rows": nr}


def quantize_row(x_row: np.ndarray, quant: str, quant_size: int, round_scale: bool):
    xr = _c(x_row, np.uint16)
    H = xr.shape[0]
    q = np.zeros(H, np.uint8)
    sc = np.zeros(H // quant_size, np.float32)
    st = lib().oracle_quantize_row(_ptr(xr), H, QUANT[quant], quant_size, int(round_scale), _ptr(q), _ptr(sc))
    if st:
        raise OracleError(st, "quantize_row")
    return q, sc


def dispatch_rows(x, dst_buffer_slot_idx, quant: str = "none", quant_size: int = 128,
                  round_scale: bool = False, tokens=None, num_rows: Optional[int] = None,
                  out=None):
    """recv_x (and recv_scales) rows of the listed tokens.

    Rows of tokens not listed keep their previous content (zero when the
    buffers are allocated here, or the caller's ``out`` = (recv_x, recv_scales)).
    """
    xs = _c(x, np.uint16)
    dst = _c(dst_buffer_slot_idx, np.int32)
    T, H = xs.shape
    K = dst.shape[1]
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tok = _c(tokens, np.int32)
    if out is None:
        rows = int(dst.max()) + 1 if num_rows is None else num_rows
        rows = max(rows, 0)
        if quant == "none":
            recv_x = np.zeros((rows, H), np.uint16)
            recv_scales = None
        else:
            recv_x = np.zeros((rows, H), np.uint8)
            recv_scales = np.zeros((rows, H // quant_size), np.float32)
    else:
        recv_x, recv_scales = out
        rows = recv_x.shape[0]
    st = _rowlib().oracle_dispatch_rows(_ptr(xs), T, H, K, _ptr(dst), QUANT[quant], quant_size,
                                    int(round_scale), _ptr(tok), tok.shape[0], _ptr(recv_x),
                                    _ptr(recv_scales), rows)
    if st:
        raise OracleError(st, "dispatch_rows")
    return recv_x, recv_scales


def combine_rows(y, dst_buffer_slot_idx, topk_weights, tokens=None):
    ys = _c(y, np.uint16)
    dst = _c(dst_buffer_slot_idx, np.int32)
    tw = _c(topk_weights, np.float32)
    T, K = dst.shape
    H = ys.shape[1]
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tok = _c(tokens, np.int32)
    out = np.zeros((tok.shape[0], H), np.uint16)
    st = _rowlib().oracle_combine_rows(_ptr(ys), ys.shape[0], H, T, K, _ptr(dst), _ptr(tw), _ptr(tok),
                                   tok.shape[0], _ptr(out))
    if st:
        raise OracleError(st, "combine_rows")
    return out


def round_tokens(T: int, R: int, rounds: int, j: int) -> np.ndarray:
    out = np.zeros(max(T // max(rounds, 1), 1), np.int32)
    n = lib().oracle_round_tokens(T, R, rounds, j, _ptr(out))
    if n < 0:
        raise OracleError(INVALID_ARG, "round_tokens")
    return out[:n]


def dispatch(x, topk_idx, topk_weights, num_experts: int, num_ranks: int,
             expert_alignment: int = 1, quant: str = "none", quant_size: int = 128,
             round_scale: bool = False, num_rounds: int = 1):
    """Full dispatch: slots over all tokens, then the rows, round by round."""
    s = slots(topk_idx, topk_weights, num_experts, num_ranks, expert_alignment)
    T = np.asarray(topk_idx).shape[0]
    recv_x, recv_scales = dispatch_rows(x, s["dst_buffer_slot_idx"], quant, quant_size,
                                        round_scale, tokens=np.zeros(0, np.int32),
                                        num_rows=s["num_recv_rows"])
    for j in range(num_rounds):
        tok = round_tokens(T, num_ranks, num_rounds, j) if num_rounds > 1 else None
        dispatch_rows(x, s["dst_buffer_slot_idx"], quant, quant_size, round_scale,
                      tokens=tok, out=(recv_x, recv_scales))
    s["recv_x"] = recv_x
    s["recv_scales"] = recv_scales
    return s


def combine(y, dst_buffer_slot_idx, topk_weights, num_ranks: int = 1, num_rounds: int = 1):
    T = np.asarray(dst_buffer_slot_idx).shape[0]
    if num_rounds == 1:
        return combine_rows(y, dst_buffer_slot_idx, topk_weights)
    H = np.asarray(y).shape[1]
    out = np.zeros((T, H), np.uint16)
    for j in range(num_rounds):
        tok = round_tokens(T, num_ranks, num_rounds, j)
        out[tok] = combine_rows(y, dst_buffer_slot_idx, topk_weights, tokens=tok)
    return out


# ---------------------------------------------------------- low latency

def ll_slots(topk_idx, topk_weights, num_experts: int, num_ranks: int, max_tokens_per_rank: int):
    """Low-latency fixed-capacity layout: rows e*R*M + r*M + p (see ep_oracle.c)."""
    ti = _c(topk_idx, np.int64)
    tw = _c(topk_weights, np.float32)
    T, K = ti.shape
    E, R, M = num_experts, num_ranks, max_tokens_per_rank
    rows = E * R * M
    dst = np.zeros((T, K), np.int32)
    cnt = np.zeros(E, np.int32)
    rng = np.zeros((E, R), np.int64)
    meta = np.full((rows, 2), -7, np.int32)          # untouched rows keep this marker
    rti = np.full((rows, K), -7, np.int32)
    rtw = np.full((rows, K), -7.0, np.float32)
    st = lib().oracle_ll_slots(_ptr(ti), _ptr(tw), T, K, E, R, M, _ptr(dst), _ptr(cnt), _ptr(rng),
                               _ptr(meta), _ptr(rti), _ptr(rtw))
    if st:
        raise OracleError(st, "ll_slots")
    return {"dst_buffer_slot_idx": dst, "recv_count": cnt, "layout_range": rng, "recv_src_metadata": meta,
            "recv_topk_idx": rti, "recv_topk_weights": rtw}


def combine_rows_q(y, y_scales, quant: str, quant_size: int, dst_buffer_slot_idx, topk_weights,
                   shared=None, tokens=None):
    """Combine of quantised (or bf16) expert outputs, optionally starting from a shared-expert row."""
    dst = _c(dst_buffer_slot_idx, np.int32)
    tw = _c(topk_weights, np.float32)
    T, K = dst.shape
    if quant == "none":
        ys = _c(y, np.uint16)
        sc = None
    else:
        ys = _c(y, np.uint8)
        sc = _c(y_scales, np.float32)
    H = ys.shape[1]
    sh = None if shared is None else _c(shared, np.uint16)
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tok = _c(tokens, np.int32)
    out = np.zeros((tok.shape[0], H), np.uint16)
    st = _rowlib().oracle_combine_rows_q(_ptr(ys), _ptr(sc), QUANT[quant], quant_size, ys.shape[0], H, T, K,
                                     _ptr(dst), _ptr(tw), _ptr(sh), _ptr(tok), tok.shape[0], _ptr(out))
    if st:
        raise OracleError(st, "combine_rows_q")
    return out


# ------------------------------------------------------- MXFP4 and UE8M0

def e2m1_to_f64(codes) -> np.ndarray:
    f = lib().oracle_e2m1_to_f64
    return np.array([f(int(c)) for c in np.asarray(codes).ravel()], np.float64).reshape(np.shape(codes))


def f32_to_e2m1(x) -> np.ndarray:
    f = lib().oracle_f32_to_e2m1
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()], np.uint8).reshape(np.shape(x))


def row_layout(H: int, quant: str, quant_size: int, scale_ue8m0: bool):
    """(code bytes per row, scale dtype, scales per row) of a received row."""
    if quant == "none":
        return 2 * H, None, 0
    ue8 = scale_ue8m0 or quant == "mxfp4"
    return (H // 2 if quant == "mxfp4" else H), (np.uint8 if ue8 else np.float32), H // quant_size


def quantize_row_mx(x_row, quant: str, quant_size: int, round_scale: bool = False, scale_ue8m0: bool = False):
    xr = _c(x_row, np.uint16)
    H = xr.shape[0]
    nb, sdt, ns = row_layout(H, quant, quant_size, scale_ue8m0)
    q = np.zeros(nb, np.uint8)
    sc = np.zeros(ns, sdt)
    st = lib().oracle_quantize_row_mx(_ptr(xr), H, QUANT[quant], quant_size, int(round_scale), int(scale_ue8m0),
                                      _ptr(q), _ptr(sc))
    if st:
        raise OracleError(st, "quantize_row_mx")
    return q, sc


def dispatch_rows_mx(x, dst_buffer_slot_idx, quant: str, quant_size: int, round_scale: bool = False,
                     scale_ue8m0: bool = False, tokens=None, num_rows: Optional[int] = None):
    """recv_x code bytes [rows, row_bytes] and scales [rows, H/quant_size] (fp32 or UE8M0 bytes)."""
    xs = _c(x, np.uint16)
    dst = _c(dst_buffer_slot_idx, np.int32)
    T, H = xs.shape
    K = dst.shape[1]
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tok = _c(tokens, np.int32)
    rows = (int(dst.max()) + 1 if dst.size else 0) if num_rows is None else num_rows
    nb, sdt, ns = row_layout(H, quant, quant_size, scale_ue8m0)
    recv_x = np.zeros((rows, nb), np.uint8)
    recv_scales = None if sdt is None else np.zeros((rows, ns), sdt)
    st = _rowlib().oracle_dispatch_rows_mx(_ptr(xs), T, H, K, _ptr(dst), QUANT[quant], quant_size, int(round_scale),
                                       int(scale_ue8m0), _ptr(tok), tok.shape[0], _ptr(recv_x),
                                       _ptr(recv_scales), rows)
    if st:
        raise OracleError(st, "dispatch_rows_mx")
    return recv_x, recv_scales


# -------------------------------------------------- group-limited gating

def group_limited_gating(logits, n_group: int, topk_group: int, per_group: int):
    """(topk_idx int64 [T, K], topk_weights fp32 [T, K]) of group-limited
    gating over router logits fp32 [T, E]: K = topk_group * per_group
    (see ep_oracle.c for the definition and its readings)."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    K = topk_group * per_group
    idx = np.zeros((T, K), np.int64)
    w = np.zeros((T, K), np.float32)
    st = lib().oracle_group_limited_gating(_ptr(lg), T, E, n_group, topk_group, per_group, _ptr(idx), _ptr(w))
    if st:
        raise OracleError(st, "group_limited_gating")
    return idx, w
