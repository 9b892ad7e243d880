"""B200-native MoE expert-parallel dispatch/combine (DeepEP's hot path, with
the ranks as logical partitions of one GPU's memory).

Thin Python binding over the C ABI of ``libep.so`` (``include/ep.h``): it
only marshals torch tensors (device memory and the current CUDA stream) into
the C calls; every step runs in the library's CUDA kernels.  There is no
CPU path: if the library is missing, calls raise ``EPLibraryError``.

    layout = ep_get_layout(idx, E, R)                 # counts, offsets, rows
    recv = ep_dispatch(x, layout.slot_pos)            # bf16 rows
    q, scale = ep_dispatch(x, layout.slot_pos, fp8=True)
    out = ep_combine(y, layout.slot_pos, w)           # gate-weighted sum
    layout, (q, scale) = ep_layout_dispatch(idx, E, R, x, fp8=True)  # one launch
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

__all__ = ["EPError", "EPLibraryError", "Layout", "RankLayout", "ep_get_layout",
           "ep_get_rank_layout", "ep_rank_layout_workspace_bytes",
           "ep_get_layout_noalloc", "EP_NOALLOC_SCRATCH_BYTES",
           "ep_dispatch", "ep_combine", "ep_read_error", "ep_layout_dispatch",
           "ep_combine_fp8", "ep_aligned_rows", "ep_pad_layout", "PaddedLayout",
           "ep_map_replicas",
           "ep_layout_workspace_bytes", "ep_kernel_launches", "lib",
           "EP_OK", "EP_ERR_INVALID_ARG", "EP_ERR_UNSUPPORTED", "EP_ERR_CUDA",
           "EP_ERR_INDEX", "EP_ERR_TIMEOUT", "LIB_PATH"]

EP_OK = 0
EP_ERR_INVALID_ARG = 1
EP_ERR_UNSUPPORTED = 2
EP_ERR_CUDA = 3
EP_ERR_INDEX = 4
EP_ERR_TIMEOUT = 5
EP_NOALLOC_SCRATCH_BYTES = 256 * 1024

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libep.so")

_lib = None

# e4m3 buffers may be given as torch's float8 type or as their raw bytes
E4M3_BYTES = (torch.float8_e4m3fn, torch.uint8)


class EPError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"[ep status {status}] {msg}")
        self.status = status


class EPLibraryError(ImportError):
    pass


_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

_SIGNATURES = {
    "ep_abi_version": ([], _i),
    "ep_last_error_string": ([], ctypes.c_char_p),
    "ep_kernel_launches": ([], ctypes.c_uint64),
    "ep_debug_expire_first_wait": ([_i], None),
    "ep_layout_workspace_bytes": ([_i, _i, _i, _i], _sz),
    "ep_get_layout": ([_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp,
                       _vp, _vp, _sz, _vp, _vp], _i),
    "ep_dispatch": ([_vp, _i, _i, _i, _vp, _i, _vp, _vp, _i, _i, _vp, _vp], _i),
    "ep_combine": ([_vp, _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp], _i),
    "ep_combine_fp8": ([_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp], _i),
    "ep_aligned_rows": ([_i, _i, _i, _i], _sz),
    "ep_map_replicas": ([_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i),
    "ep_pad_layout": ([_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp], _i),
    "ep_read_error": ([_vp, _vp], _i),
    "ep_get_layout_noalloc": ([_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                               _vp, _vp, _vp, _vp], _i),
    "ep_rank_layout_workspace_bytes": ([_i, _i], _sz),
    "ep_get_rank_layout": ([_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i),
    "ep_layout_dispatch": ([_vp, _i, _i, _i, _i, _i, _vp, _i, _i, _vp, _vp, _vp, _vp,
                            _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i, _vp, _vp], _i),
}


def lib() -> ctypes.CDLL:
    """The loaded libep.so (raises EPLibraryError when it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise EPLibraryError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m combine_ep_get_09_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(status: int):
    if status != EP_OK:
        raise EPError(status, lib().ep_last_error_string().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _need_cuda(name: str, t: torch.Tensor):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need(name: str, t: Optional[torch.Tensor], dtype, shape=None, min_rows=None):
    """A CUDA, contiguous tensor of `dtype` and `shape` (or, with min_rows,
    at least that many rows of shape[1:]): the library writes through the
    raw pointer, so a wrong size would write out of bounds."""
    if t is None:
        raise ValueError(f"{name} is missing")
    _need_cuda(name, t)
    allowed = dtype if isinstance(dtype, tuple) else (dtype,)
    if t.dtype not in allowed:
        raise ValueError(f"{name} must be {' or '.join(map(str, allowed))}, not {t.dtype}")
    if shape is not None:
        if min_rows is not None:
            if t.dim() != len(shape) or t.shape[0] < min_rows or tuple(t.shape[1:]) != tuple(shape[1:]):
                raise ValueError(f"{name} must have shape [>= {min_rows}, "
                                 f"{', '.join(map(str, shape[1:]))}], not {tuple(t.shape)}")
        elif tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")


def _need_err(d_err: Optional[torch.Tensor]):
    if d_err is not None:
        _need("d_err", d_err, torch.int32)
        if d_err.numel() < 1:
            raise ValueError("d_err needs one element")


def _check_layout(L, T: int, k: int, E: int, R: int):
    i32 = torch.int32
    _need("cnt_e", L.cnt_e, i32, (E,))
    _need("cnt_r", L.cnt_r, i32, (R,))
    _need("in_rank", L.in_rank, torch.uint8, (T, R))
    _need("off_e", L.off_e, i32, (E + 1,))
    _need("off_r", L.off_r, i32, (R + 1,))
    _need("slot_pos", L.slot_pos, i32, (T, k))
    _need("recv_src", L.recv_src, i32, (T * k,))


class Layout(NamedTuple):
    cnt_e: torch.Tensor     # [E] int32
    cnt_r: torch.Tensor     # [R] int32
    in_rank: torch.Tensor   # [T, R] uint8
    off_e: torch.Tensor     # [E+1] int32
    off_r: torch.Tensor     # [R+1] int32
    slot_pos: torch.Tensor  # [T, k] int32
    recv_src: torch.Tensor  # [T*k] int32


def ep_layout_workspace_bytes(T: int, k: int, E: int, R: int) -> int:
    return int(lib().ep_layout_workspace_bytes(T, k, E, R))


def ep_kernel_launches() -> int:
    return int(lib().ep_kernel_launches())


def ep_debug_expire_first_wait(on: bool) -> None:
    """Testing switch: while on, the first bounded copy wait of every CTA of
    the bulk-copy kernels gives up at once, so their time-out path
    (EP_ERR_TIMEOUT in d_err, drain, early return) runs; off restores the
    normal limit.  Process-wide."""
    lib().ep_debug_expire_first_wait(1 if on else 0)


def empty_layout(T: int, k: int, E: int, R: int, device) -> Layout:
    i32 = dict(dtype=torch.int32, device=device)
    return Layout(torch.empty(E, **i32), torch.empty(R, **i32),
                  torch.empty((T, R), dtype=torch.uint8, device=device),
                  torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                  torch.empty((T, k), **i32), torch.empty(T * k, **i32))


def ep_get_layout(idx: torch.Tensor, E: int, R: int, *,
                  out: Optional[Layout] = None,
                  ws: Optional[torch.Tensor] = None,
                  d_err: Optional[torch.Tensor] = None,
                  stream=None) -> Layout:
    """Dispatch layout of expert ids ``idx`` [T, k] (int64 or int32, -1 =
    dropped slot).  ``ws`` (uint8, zero-filled before first use, reused
    across stream-ordered calls) is allocated zeroed when not given."""
    _need_cuda("idx", idx)
    if idx.dtype not in (torch.int64, torch.int32) or idx.dim() != 2:
        raise ValueError("idx must be a 2-D int64 or int32 tensor")
    T, k = idx.shape
    if out is None:
        out = empty_layout(T, k, E, R, idx.device)
    _check_layout(out, T, k, E, R)
    _need_err(d_err)
    need = ep_layout_workspace_bytes(T, k, E, R)
    if ws is None and need > 0:
        ws = torch.zeros(need, dtype=torch.uint8, device=idx.device)
    _check(lib().ep_get_layout(
        _ptr(idx), int(idx.dtype == torch.int64), T, k, E, R,
        _ptr(out.cnt_e), _ptr(out.cnt_r), _ptr(out.in_rank), _ptr(out.off_e),
        _ptr(out.off_r), _ptr(out.slot_pos), _ptr(out.recv_src),
        _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _ptr(d_err), _stream(stream)))
    return out


def ep_get_layout_noalloc(idx: torch.Tensor, E: int, R: int, *,
                          out: Optional[Layout] = None,
                          d_err: Optional[torch.Tensor] = None,
                          stream=None) -> Layout:
    """ep_get_layout for callers that cannot allocate device memory: the
    library's fixed scratch array (EP_NOALLOC_SCRATCH_BYTES per device)
    replaces the workspace.  The array used is the current device's, so
    ``idx``, the outputs and ``stream`` must be on the current device.
    Calls that overlap on the GPU race on that array; the first call on a
    device loads the library's module there, so make it before any stream
    capture.  Outputs are allocated here only when ``out`` is not given."""
    _need_cuda("idx", idx)
    cur = torch.cuda.current_device()
    if idx.device.index != cur:
        raise ValueError(f"idx is on cuda:{idx.device.index} but the current device is "
                         f"cuda:{cur}; the scratch array used is the current device's")
    if isinstance(stream, torch.cuda.Stream) and stream.device.index != cur:
        raise ValueError(f"stream belongs to cuda:{stream.device.index} but the current "
                         f"device is cuda:{cur}")
    if idx.dtype not in (torch.int64, torch.int32) or idx.dim() != 2:
        raise ValueError("idx must be a 2-D int64 or int32 tensor")
    T, k = idx.shape
    if out is None:
        out = empty_layout(T, k, E, R, idx.device)
    _check_layout(out, T, k, E, R)
    _need_err(d_err)
    _check(lib().ep_get_layout_noalloc(
        _ptr(idx), int(idx.dtype == torch.int64), T, k, E, R,
        _ptr(out.cnt_e), _ptr(out.cnt_r), _ptr(out.in_rank), _ptr(out.off_e),
        _ptr(out.off_r), _ptr(out.slot_pos), _ptr(out.recv_src),
        _ptr(d_err), _stream(stream)))
    return out


class RankLayout(NamedTuple):
    cnt_r: torch.Tensor     # [R] int32
    off_r: torch.Tensor     # [R+1] int32
    rank_row: torch.Tensor  # [T, R] int32
    rank_src: torch.Tensor  # [T*R] int32


def ep_rank_layout_workspace_bytes(T: int, R: int) -> int:
    return int(lib().ep_rank_layout_workspace_bytes(T, R))


def ep_get_rank_layout(in_rank: torch.Tensor, *, out: Optional[RankLayout] = None,
                       ws: Optional[torch.Tensor] = None, stream=None) -> RankLayout:
    """Rows of the rank-deduplicated dispatch from the token-in-rank mask
    ``in_rank`` [T, R] (uint8) of ep_get_layout: one row per (token, rank)
    pair.  Dispatch with ``ep_dispatch(x, rank_row)``; combine per-rank
    partial outputs with ``ep_combine(z, rank_row, None)``."""
    _need_cuda("in_rank", in_rank)
    if in_rank.dtype != torch.uint8 or in_rank.dim() != 2:
        raise ValueError("in_rank must be a 2-D uint8 tensor")
    T, R = in_rank.shape
    dev = in_rank.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = RankLayout(torch.empty(R, **i32), torch.empty(R + 1, **i32),
                         torch.empty((T, R), **i32), torch.empty(T * R, **i32))
    _need("cnt_r", out.cnt_r, torch.int32, (R,))
    _need("off_r", out.off_r, torch.int32, (R + 1,))
    _need("rank_row", out.rank_row, torch.int32, (T, R))
    _need("rank_src", out.rank_src, torch.int32, (T * R,))
    need = ep_rank_layout_workspace_bytes(T, R)
    if ws is None and need > 0:
        ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    _check(lib().ep_get_rank_layout(
        _ptr(in_rank), T, R, _ptr(out.cnt_r), _ptr(out.off_r), _ptr(out.rank_row),
        _ptr(out.rank_src), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def ep_dispatch(x: torch.Tensor, slot_pos: torch.Tensor, fp8: bool = False, *,
                recv: Optional[torch.Tensor] = None,
                recv_scale: Optional[torch.Tensor] = None,
                num_sms: int = 0, d_err: Optional[torch.Tensor] = None,
                stream=None):
    """Rows of ``x`` [T, H] bf16 to their receive rows.  Returns ``recv``
    [T*k, H] (bf16), or ``(recv_q [T*k, H] float8_e4m3fn, recv_scale
    [T*k, H/128] fp32)`` when ``fp8``.  A given ``recv`` may have more rows
    (an aligned layout's ep_aligned_rows); slot rows past it are skipped."""
    _need_cuda("x", x)
    _need_cuda("slot_pos", slot_pos)
    if x.dtype != torch.bfloat16 or slot_pos.dtype != torch.int32:
        raise ValueError("x must be bf16 and slot_pos int32")
    T, H = x.shape
    if slot_pos.dim() != 2 or slot_pos.shape[0] != T:
        raise ValueError("slot_pos must be [T, k] with x's T")
    k = slot_pos.shape[1]
    rdt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    if recv is None:
        recv = torch.empty((T * k, H), device=x.device, dtype=rdt)
    _need("recv", recv, E4M3_BYTES if fp8 else rdt, (0, H), min_rows=0)
    if fp8:
        if recv_scale is None:
            recv_scale = torch.empty((recv.shape[0], H // 128), device=x.device,
                                     dtype=torch.float32)
        _need("recv_scale", recv_scale, torch.float32, (0, H // 128), min_rows=recv.shape[0])
    if recv.shape[0] == 0 and T * k > 0:
        raise ValueError("recv has no rows")   # 0 would mean T*k rows to the library
    _need_err(d_err)
    _check(lib().ep_dispatch(_ptr(x), T, H, k, _ptr(slot_pos), int(bool(fp8)),
                             _ptr(recv), _ptr(recv_scale) if fp8 else None,
                             recv.shape[0], num_sms, _ptr(d_err), _stream(stream)))
    return (recv, recv_scale) if fp8 else recv


def ep_layout_dispatch(idx: torch.Tensor, E: int, R: int, x: torch.Tensor,
                       fp8: bool = False, *, out: Optional[Layout] = None,
                       recv: Optional[torch.Tensor] = None,
                       recv_scale: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, num_sms: int = 0,
                       d_err: Optional[torch.Tensor] = None, stream=None):
    """ep_get_layout then ep_dispatch, in one kernel launch for small
    batches (a decode step).  Returns ``(layout, recv)`` or, with ``fp8``,
    ``(layout, (recv_q, recv_scale))``, bit-identical to the two calls."""
    _need_cuda("idx", idx)
    _need_cuda("x", x)
    if idx.dtype not in (torch.int64, torch.int32) or idx.dim() != 2:
        raise ValueError("idx must be a 2-D int64 or int32 tensor")
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[0] != idx.shape[0]:
        raise ValueError("x must be a bf16 [T, H] tensor with idx's T")
    T, k = idx.shape
    H = x.shape[1]
    if out is None:
        out = empty_layout(T, k, E, R, idx.device)
    _check_layout(out, T, k, E, R)
    rdt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    if recv is None:
        recv = torch.empty((T * k, H), device=x.device, dtype=rdt)
    _need("recv", recv, E4M3_BYTES if fp8 else rdt, (T * k, H), min_rows=T * k)
    if fp8:
        if recv_scale is None:
            recv_scale = torch.empty((T * k, H // 128), device=x.device, dtype=torch.float32)
        _need("recv_scale", recv_scale, torch.float32, (T * k, H // 128), min_rows=T * k)
    _need_err(d_err)
    need = ep_layout_workspace_bytes(T, k, E, R)
    if ws is None and need > 0:
        ws = torch.zeros(need, dtype=torch.uint8, device=idx.device)
    _check(lib().ep_layout_dispatch(
        _ptr(idx), int(idx.dtype == torch.int64), T, k, E, R, _ptr(x), H, int(bool(fp8)),
        _ptr(out.cnt_e), _ptr(out.cnt_r), _ptr(out.in_rank), _ptr(out.off_e),
        _ptr(out.off_r), _ptr(out.slot_pos), _ptr(out.recv_src), _ptr(recv),
        _ptr(recv_scale) if fp8 else None, _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), num_sms, _ptr(d_err),
        _stream(stream)))
    return out, ((recv, recv_scale) if fp8 else recv)


def ep_combine(y: torch.Tensor, slot_pos: torch.Tensor, w: Optional[torch.Tensor], *,
               out: Optional[torch.Tensor] = None, num_sms: int = 0,
               d_err: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Gate-weighted combine of expert outputs ``y`` [T*k, H] bf16 into
    ``out`` [T, H] bf16 (fp32 fma chain in slot order).  ``w=None`` sums
    the slot rows with unit weights."""
    for name, t in (("y", y), ("slot_pos", slot_pos)):
        _need_cuda(name, t)
    if w is not None:
        _need_cuda("w", w)
    if y.dtype != torch.bfloat16 or (w is not None and w.dtype != torch.float32):
        raise ValueError("y must be bf16 and w fp32")
    T, k = slot_pos.shape
    H = y.shape[1]
    if w is not None and tuple(w.shape) != (T, k):
        raise ValueError(f"w must have shape {(T, k)}")
    if out is None:
        out = torch.empty((T, H), device=y.device, dtype=torch.bfloat16)
    _need("out", out, torch.bfloat16, (T, H))
    _need_err(d_err)
    if y.shape[0] == 0 and T > 0:
        raise ValueError("y has no rows")   # 0 would mean T*k rows to the library
    _check(lib().ep_combine(_ptr(y), y.shape[0], T, H, k, _ptr(slot_pos), _ptr(w),
                            _ptr(out), num_sms, _ptr(d_err), _stream(stream)))
    return out


def ep_combine_fp8(y_q: torch.Tensor, y_scale: torch.Tensor, slot_pos: torch.Tensor,
                   w: Optional[torch.Tensor], *, out: Optional[torch.Tensor] = None,
                   num_sms: int = 0, d_err: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Gate-weighted combine of FP8 expert outputs (``y_q`` [rows, H]
    float8_e4m3fn codes, ``y_scale`` [rows, H/128] fp32) into ``out`` [T, H]
    bf16: each value decoded and scaled in fp32, then the fp32 fma chain in
    slot order."""
    for name, t in (("y_q", y_q), ("y_scale", y_scale), ("slot_pos", slot_pos)):
        _need_cuda(name, t)
    if w is not None:
        _need_cuda("w", w)
    if y_q.dtype not in E4M3_BYTES or y_scale.dtype != torch.float32:
        raise ValueError("y_q must be float8_e4m3fn (or its uint8 bytes) and y_scale fp32")
    T, k = slot_pos.shape
    rows, H = y_q.shape
    if (rows == 0 and T > 0) or y_scale.shape != (rows, H // 128):
        raise ValueError("y_scale must be [rows, H/128] and y_q hold rows")
    if w is not None and tuple(w.shape) != (T, k):
        raise ValueError(f"w must have shape {(T, k)}")
    if out is None:
        out = torch.empty((T, H), device=y_q.device, dtype=torch.bfloat16)
    _need("out", out, torch.bfloat16, (T, H))
    _need_err(d_err)
    _check(lib().ep_combine_fp8(_ptr(y_q), _ptr(y_scale), rows, T, H, k, _ptr(slot_pos),
                                _ptr(w), _ptr(out), num_sms, _ptr(d_err), _stream(stream)))
    return out


class PaddedLayout(NamedTuple):
    off_pad: torch.Tensor       # [E+1] int32
    slot_pos: torch.Tensor      # [T, k] int32, rows of the aligned buffer
    recv_src: torch.Tensor      # [ep_aligned_rows(T, k, E, align)] int32


def ep_aligned_rows(T: int, k: int, E: int, align: int) -> int:
    return int(lib().ep_aligned_rows(T, k, E, align))


def ep_pad_layout(layout: Layout, align: int, *, out: Optional[PaddedLayout] = None,
                  stream=None) -> PaddedLayout:
    """Expert segments of ``layout`` (from ep_get_layout) moved to start on
    multiples of ``align`` rows, for a grouped GEMM with row tiles of that
    size.  Dispatch into and combine from a buffer of
    ``ep_aligned_rows(T, k, E, align)`` rows with the returned slot_pos."""
    T, k = layout.slot_pos.shape
    E = layout.cnt_e.shape[0]
    dev = layout.slot_pos.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = PaddedLayout(torch.empty(E + 1, **i32), torch.empty((T, k), **i32),
                           torch.empty(max(1, ep_aligned_rows(T, k, E, align)), **i32))
    _need("off_pad", out.off_pad, torch.int32, (E + 1,))
    _need("slot_pos", out.slot_pos, torch.int32, (T, k))
    _need("recv_src", out.recv_src, torch.int32, (0,),
          min_rows=ep_aligned_rows(T, k, E, align))
    _check(lib().ep_pad_layout(_ptr(layout.cnt_e), _ptr(layout.slot_pos), T, k, E, align,
                               _ptr(out.off_pad), _ptr(out.slot_pos), _ptr(out.recv_src),
                               _stream(stream)))
    return out


def ep_read_error(d_err: torch.Tensor, stream=None) -> int:
    """Waits for the stream and returns the device error word."""
    st = lib().ep_read_error(_ptr(d_err), _stream(stream))
    if st == EP_ERR_CUDA:
        _check(st)
    return int(st)


def ep_map_replicas(idx: torch.Tensor, layout: Layout, rep_off: torch.Tensor,
                    rep_ids: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                    d_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Physical expert ids [T, k] (int32) for logical ids ``idx`` with
    ``layout`` = ep_get_layout(idx, E, R): expert e's slots, in the layout's
    order, dealt round-robin over its copies ``rep_ids[rep_off[e]:rep_off[e+1]]``."""
    for name, t in (("idx", idx), ("rep_off", rep_off), ("rep_ids", rep_ids)):
        _need_cuda(name, t)
    if rep_off.dtype != torch.int32 or rep_ids.dtype != torch.int32:
        raise ValueError("rep_off and rep_ids must be int32")
    T, k = idx.shape
    E = rep_off.shape[0] - 1
    if layout.cnt_e.shape[0] != E:
        raise ValueError("rep_off needs E + 1 entries for the layout's E experts")
    if out is None:
        out = torch.empty((T, k), dtype=torch.int32, device=idx.device)
    _need("out", out, torch.int32, (T, k))
    _need_err(d_err)
    _check(lib().ep_map_replicas(_ptr(idx), int(idx.dtype == torch.int64), T, k, E,
                                 _ptr(layout.slot_pos), _ptr(layout.off_e), _ptr(rep_off),
                                 _ptr(rep_ids), _ptr(out), _ptr(d_err), _stream(stream)))
    return out
