"""CPU oracle of the MoE dispatch/combine path (ctypes wrapper over plain C).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package; the CUDA library
never does, and shares no code with it.  The arithmetic lives in
``ep_oracle.c`` (its header states the definitions it follows); this module
only marshals numpy/torch CPU arrays in and out.
"""
from __future__ import annotations

import ctypes
from typing import Dict

import numpy as np
import torch

from . import build as _build

_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)

ORACLE_OK = 0
ORACLE_ERR_INVALID_ARG = 1
ORACLE_ERR_INDEX = 4


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        L.ep_oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.ep_oracle_bf16_to_f32.restype = ctypes.c_float
        L.ep_oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.ep_oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.ep_oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.ep_oracle_f32_to_e4m3.restype = ctypes.c_uint8
        L.ep_oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.ep_oracle_e4m3_to_f32.restype = ctypes.c_float
        L.ep_oracle_f32_to_bf16_n.argtypes = [_f32p, ctypes.c_long, _u16p]
        L.ep_oracle_f32_to_bf16_n.restype = None
        L.ep_oracle_f32_to_e4m3_n.argtypes = [_f32p, ctypes.c_long, _u8p]
        L.ep_oracle_f32_to_e4m3_n.restype = None
        L.ep_oracle_layout.argtypes = [
            _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, _i32p, _u8p, _i32p, _i32p, _i32p, _i32p]
        L.ep_oracle_layout.restype = ctypes.c_int
        L.ep_oracle_rank_layout.argtypes = [_u8p, ctypes.c_int, ctypes.c_int, _i32p, _i32p,
                                            _i32p, _i32p]
        L.ep_oracle_rank_layout.restype = ctypes.c_int
        L.ep_oracle_dispatch_bf16.argtypes = [
            _u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p,
            ctypes.c_long, _u16p]
        L.ep_oracle_dispatch_bf16.restype = ctypes.c_int
        L.ep_oracle_dispatch_fp8.argtypes = [
            _u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p,
            ctypes.c_long, _u8p, _f32p]
        L.ep_oracle_dispatch_fp8.restype = ctypes.c_int
        L.ep_oracle_combine.argtypes = [
            _u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, _f32p, _u16p]
        L.ep_oracle_combine.restype = ctypes.c_int
        L.ep_oracle_layout_aligned.argtypes = [
            _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, _i32p, _i32p]
        L.ep_oracle_layout_aligned.restype = ctypes.c_int
        L.ep_oracle_combine_fp8.argtypes = [
            _u8p, _f32p, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, _f32p, _u16p]
        L.ep_oracle_combine_fp8.restype = ctypes.c_int
        L.ep_oracle_map_replicas.argtypes = [
            _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _i32p, _i32p]
        L.ep_oracle_map_replicas.restype = ctypes.c_int
        _lib = L
    return _lib


def _np(a, dtype) -> np.ndarray:
    """Contiguous numpy view of a CPU tensor/array with the given dtype."""
    if isinstance(a, torch.Tensor):
        if a.dtype == torch.bfloat16:
            a = a.view(torch.int16)
        elif a.dtype == torch.float8_e4m3fn:
            a = a.view(torch.uint8)
        a = a.detach().cpu().contiguous().numpy()
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        if a.dtype.itemsize == np.dtype(dtype).itemsize and a.dtype.kind in "iu" \
                and np.dtype(dtype).kind in "iu":
            a = a.view(dtype)
        else:
            a = a.astype(dtype)
    return a


def _ptr(a: np.ndarray, typ):
    return a.ctypes.data_as(typ)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor."""
    return _np(t, np.uint16)


def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


# ------------------------------------------------------------------ numbers

def f32_to_bf16(v: float) -> int:
    return int(lib().ep_oracle_f32_to_bf16(float(v)))


def bf16_to_f32(h: int) -> float:
    return float(lib().ep_oracle_bf16_to_f32(int(h)))


def f32_to_e4m3(v: float) -> int:
    return int(lib().ep_oracle_f32_to_e4m3(float(v)))


def e4m3_to_f32(q: int) -> float:
    return float(lib().ep_oracle_e4m3_to_f32(int(q)))


def f32_to_bf16_array(v) -> np.ndarray:
    a = _np(v, np.float32).reshape(-1)
    out = np.empty(a.size, np.uint16)
    lib().ep_oracle_f32_to_bf16_n(_ptr(a, _f32p), a.size, _ptr(out, _u16p))
    return out


def f32_to_e4m3_array(v) -> np.ndarray:
    a = _np(v, np.float32).reshape(-1)
    out = np.empty(a.size, np.uint8)
    lib().ep_oracle_f32_to_e4m3_n(_ptr(a, _f32p), a.size, _ptr(out, _u8p))
    return out


# ------------------------------------------------------------------- layout

def layout(idx, E: int, R: int) -> Dict[str, np.ndarray]:
    """Dispatch layout of expert ids idx [T, k] (int64; -1 = dropped).

    Returns cnt_e[E], cnt_r[R], in_rank[T, R] (u8), off_e[E+1], off_r[R+1],
    slot_pos[T, k], recv_src[T*k] (all int32 but in_rank) and 'status'
    (0, or 4 when an id lay outside [-1, E)).
    """
    ids = _np(idx, np.int64)
    T, k = ids.shape
    out = dict(cnt_e=np.zeros(E, np.int32), cnt_r=np.zeros(R, np.int32),
               in_rank=np.zeros((T, R), np.uint8),
               off_e=np.zeros(E + 1, np.int32), off_r=np.zeros(R + 1, np.int32),
               slot_pos=np.zeros((T, k), np.int32),
               recv_src=np.zeros(T * k, np.int32))
    st = lib().ep_oracle_layout(
        _ptr(ids, _i64p), T, k, E, R, _ptr(out["cnt_e"], _i32p),
        _ptr(out["cnt_r"], _i32p), _ptr(out["in_rank"], _u8p),
        _ptr(out["off_e"], _i32p), _ptr(out["off_r"], _i32p),
        _ptr(out["slot_pos"], _i32p), _ptr(out["recv_src"], _i32p))
    if st == ORACLE_ERR_INVALID_ARG:
        raise ValueError("oracle layout: invalid arguments")
    out["status"] = st
    return out


def rank_layout(in_rank) -> Dict[str, np.ndarray]:
    """Rank rows of the token-in-rank mask in_rank [T, R] (uint8):
    cnt_r[R], off_r[R+1], rank_row[T, R], rank_src[T*R]."""
    m = np.ascontiguousarray(_np(in_rank, np.uint8))
    T, R = m.shape
    out = dict(cnt_r=np.zeros(R, np.int32), off_r=np.zeros(R + 1, np.int32),
               rank_row=np.zeros((T, R), np.int32), rank_src=np.zeros(T * R, np.int32))
    st = lib().ep_oracle_rank_layout(_ptr(m, _u8p), T, R, _ptr(out["cnt_r"], _i32p),
                                     _ptr(out["off_r"], _i32p), _ptr(out["rank_row"], _i32p),
                                     _ptr(out["rank_src"], _i32p))
    if st:
        raise ValueError("oracle rank_layout: invalid arguments")
    return out


# ----------------------------------------------------------------- dispatch

def dispatch_bf16(x, slot_pos, n_rows: int, recv: np.ndarray = None) -> np.ndarray:
    """recv[slot_pos[t, j]] = x[t] as uint16 bf16 bits [n_rows, H].

    Rows no slot points at keep the contents of ``recv`` (zeros if None)."""
    xb = _np(x, np.uint16)
    sp = _np(slot_pos, np.int32)
    T, H = xb.shape
    k = sp.shape[1]
    if recv is None:
        recv = np.zeros((n_rows, H), np.uint16)
    assert recv.dtype == np.uint16 and recv.flags.c_contiguous
    st = lib().ep_oracle_dispatch_bf16(_ptr(xb, _u16p), T, H, k,
                                       _ptr(sp, _i32p), n_rows,
                                       _ptr(recv, _u16p))
    if st:
        raise ValueError("oracle dispatch_bf16: invalid arguments")
    return recv


def dispatch_fp8(x, slot_pos, n_rows: int, recv_q: np.ndarray = None,
                 recv_scale: np.ndarray = None):
    """FP8 dispatch: (recv_q uint8 [n_rows, H], recv_scale f32 [n_rows, H/128])."""
    xb = _np(x, np.uint16)
    sp = _np(slot_pos, np.int32)
    T, H = xb.shape
    k = sp.shape[1]
    if recv_q is None:
        recv_q = np.zeros((n_rows, H), np.uint8)
    if recv_scale is None:
        recv_scale = np.zeros((n_rows, H // 128), np.float32)
    st = lib().ep_oracle_dispatch_fp8(_ptr(xb, _u16p), T, H, k,
                                      _ptr(sp, _i32p), n_rows,
                                      _ptr(recv_q, _u8p),
                                      _ptr(recv_scale, _f32p))
    if st:
        raise ValueError("oracle dispatch_fp8: invalid arguments")
    return recv_q, recv_scale


# ------------------------------------------------------------------ combine

def combine(y, slot_pos, w) -> np.ndarray:
    """out[t] = bf16(fma chain over slots of w[t, j] * y[slot_pos[t, j]]),
    as uint16 bf16 bits [T, H]; w=None means every weight is 1."""
    yb = _np(y, np.uint16)
    sp = _np(slot_pos, np.int32)
    wf = np.ones(sp.shape, np.float32) if w is None else _np(w, np.float32)
    n_rows, H = yb.shape
    T, k = sp.shape
    out = np.zeros((T, H), np.uint16)
    st = lib().ep_oracle_combine(_ptr(yb, _u16p), n_rows, T, H, k,
                                 _ptr(sp, _i32p), _ptr(wf, _f32p),
                                 _ptr(out, _u16p))
    if st:
        raise ValueError("oracle combine: invalid arguments")
    return out


# ------------------------------------------------------- aligned layout

def padded_rows(T: int, k: int, E: int, align: int) -> int:
    """Receive rows an aligned layout may use: T*k + E*(align-1)."""
    return T * k + E * (align - 1)


def layout_aligned(idx, E: int, align: int) -> Dict[str, np.ndarray]:
    """Receive rows with every expert segment starting on a multiple of
    ``align``: off_pad [E+1], slot_pos [T,k], recv_src [T*k + E*(align-1)]
    (-1 for padding and unused rows) and the status."""
    ix = _np(idx, np.int64)
    T, k = ix.shape
    out = {"off_pad": np.zeros(E + 1, np.int32),
           "slot_pos": np.zeros((T, k), np.int32),
           "recv_src": np.zeros(padded_rows(T, k, E, align), np.int32)}
    st = lib().ep_oracle_layout_aligned(
        _ptr(ix, _i64p), T, k, E, align, _ptr(out["off_pad"], _i32p),
        _ptr(out["slot_pos"], _i32p), _ptr(out["recv_src"], _i32p))
    if st == ORACLE_ERR_INVALID_ARG:
        raise ValueError("oracle layout_aligned: invalid arguments")
    out["status"] = st
    return out


# ---------------------------------------------------------- FP8 combine

def combine_fp8(yq, ys, slot_pos, w) -> np.ndarray:
    """out[t] = bf16(fma chain over slots of w[t, j] * (e4m3(yq) * ys)), as
    uint16 bf16 bits [T, H]; w=None means every weight is 1."""
    q = _np(yq, np.uint8)
    sc = _np(ys, np.float32)
    sp = _np(slot_pos, np.int32)
    wf = np.ones(sp.shape, np.float32) if w is None else _np(w, np.float32)
    n_rows, H = q.shape
    T, k = sp.shape
    assert sc.shape == (n_rows, H // 128)
    out = np.zeros((T, H), np.uint16)
    st = lib().ep_oracle_combine_fp8(_ptr(q, _u8p), _ptr(sc, _f32p), n_rows, T, H, k,
                                     _ptr(sp, _i32p), _ptr(wf, _f32p), _ptr(out, _u16p))
    if st:
        raise ValueError("oracle combine_fp8: invalid arguments")
    return out


# ------------------------------------------------------------- replicas

def map_replicas(idx, rep_off, rep_ids):
    """Physical expert of every slot [T, k] (int32, -1 dropped) and the
    status: logical expert e's slots, in token-major order, dealt
    round-robin over its copies rep_ids[rep_off[e]:rep_off[e+1]]."""
    ix = _np(idx, np.int64)
    off = _np(rep_off, np.int32)
    ids = _np(rep_ids, np.int32)
    T, k = ix.shape
    E = off.shape[0] - 1
    phys = np.zeros((T, k), np.int32)
    st = lib().ep_oracle_map_replicas(_ptr(ix, _i64p), T, k, E, _ptr(off, _i32p),
                                      _ptr(ids, _i32p), _ptr(phys, _i32p))
    if st == ORACLE_ERR_INVALID_ARG:
        raise ValueError("oracle map_replicas: invalid arguments")
    return phys, st
