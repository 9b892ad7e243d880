"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/ep.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

import combine_ep_get_09_b200 as ep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "ep.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert "ep_get_layout" in names and "ep_dispatch" in names and "ep_combine" in names
    L = ctypes.CDLL(ep.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) <= set(ep._SIGNATURES), "binding lacks a declared symbol"


def test_abi_version():
    assert ep.lib().ep_abi_version() == 5


def test_workspace_sizes():
    # the single-CTA and cluster paths (T*k < 65536) need none; the grid
    # path (65536 <= T*k <= 2^19) three 4-byte barrier counters padded to 16
    # bytes plus an [E + R][160] count matrix and E + R totals, when that is
    # at most 256 KiB (else the cluster path again); the tiled path one row
    # of E + R counts per tile (at most 296 tiles of >= 128 tokens) plus a
    # 16-byte ticket
    assert ep.ep_layout_workspace_bytes(128, 8, 256, 8) == 0
    assert ep.ep_layout_workspace_bytes(0, 8, 256, 8) == 0
    assert ep.ep_layout_workspace_bytes(4096, 8, 256, 8) == 0
    assert ep.ep_layout_workspace_bytes(8191, 8, 256, 8) == 0
    assert ep.ep_layout_workspace_bytes(8192, 8, 256, 8) == 16 + (264 * 160 + 264) * 4
    assert ep.ep_layout_workspace_bytes(65536, 8, 256, 8) == 16 + (264 * 160 + 264) * 4
    assert ep.ep_layout_workspace_bytes(32768, 8, 128, 16) == 16 + (144 * 160 + 144) * 4
    assert ep.ep_layout_workspace_bytes(32768, 8, 1024, 64) == 0   # 696 KiB: cluster path
    assert ep.ep_layout_workspace_bytes(65537, 8, 256, 8) == 16 + 296 * 264 * 4
    assert ep.ep_layout_workspace_bytes(70000, 8, 128, 16) == 16 + 296 * 144 * 4
    assert ep.ep_layout_workspace_bytes(300000, 2, 16, 16) == 16 + 296 * 32 * 4
    # invalid sizes report 0
    assert ep.ep_layout_workspace_bytes(4096, 8, 250, 8) == 0


def _layout_call(**kw):
    a = dict(idx=16, idx_is_int64=1, T=4, k=2, E=8, R=2, cnt_e=16, cnt_r=16,
             in_rank=16, off_e=16, off_r=16, slot_pos=16, recv_src=16, ws=None,
             ws_bytes=0, d_err=None, stream=None)
    a.update(kw)
    return ep.lib().ep_get_layout(*a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), ep.EP_ERR_INVALID_ARG),
    (dict(k=0), ep.EP_ERR_INVALID_ARG),
    (dict(E=0), ep.EP_ERR_INVALID_ARG),
    (dict(R=0), ep.EP_ERR_INVALID_ARG),
    (dict(E=9), ep.EP_ERR_INVALID_ARG),          # E % R != 0
    (dict(k=9), ep.EP_ERR_INVALID_ARG),          # k > E
    (dict(k=33, E=64), ep.EP_ERR_UNSUPPORTED),
    (dict(E=2048), ep.EP_ERR_UNSUPPORTED),
    (dict(E=128, R=128), ep.EP_ERR_UNSUPPORTED),
    (dict(T=1 << 30, k=4), ep.EP_ERR_UNSUPPORTED),
    (dict(cnt_e=None), ep.EP_ERR_INVALID_ARG),
    (dict(idx=None), ep.EP_ERR_INVALID_ARG),
    (dict(idx=20), ep.EP_ERR_INVALID_ARG),       # int64 ids need 8-byte alignment
    (dict(slot_pos=18), ep.EP_ERR_INVALID_ARG),
    (dict(T=65537, k=8, E=256, R=8), ep.EP_ERR_INVALID_ARG),   # tiled path, no ws
    (dict(T=65537, k=8, E=256, R=8, ws=16, ws_bytes=100), ep.EP_ERR_INVALID_ARG),
    (dict(T=65537, k=8, E=256, R=8, ws=24, ws_bytes=1 << 20), ep.EP_ERR_INVALID_ARG),
])
def test_layout_rejects(kw, status):
    assert _layout_call(**kw) == status
    assert ep.lib().ep_last_error_string().decode()


@pytest.mark.parametrize("args,status", [
    ((16, -1, 64, 2, 16, 0, 16, None, 0, 0, None, None), ep.EP_ERR_INVALID_ARG),
    ((16, 4, 0, 2, 16, 0, 16, None, 0, 0, None, None), ep.EP_ERR_INVALID_ARG),
    ((16, 4, 12, 2, 16, 0, 16, None, 0, 0, None, None), ep.EP_ERR_UNSUPPORTED),   # H % 8
    ((16, 4, 64, 2, 16, 1, 16, 16, 0, 0, None, None), ep.EP_ERR_UNSUPPORTED),     # fp8, H % 128
    ((16, 4, 64, 33, 16, 0, 16, None, 0, 0, None, None), ep.EP_ERR_UNSUPPORTED),  # k > 32
    ((16, 4, 64, 2, 16, 0, 16, None, 0, -1, None, None), ep.EP_ERR_INVALID_ARG),  # num_sms
    ((None, 4, 64, 2, 16, 0, 16, None, 0, 0, None, None), ep.EP_ERR_INVALID_ARG),
    ((24, 4, 64, 2, 16, 0, 16, None, 0, 0, None, None), ep.EP_ERR_INVALID_ARG),   # x misaligned
    ((16, 4, 128, 2, 16, 1, 16, None, 0, 0, None, None), ep.EP_ERR_INVALID_ARG),  # fp8, no scale
    ((16, 4, 64, 2, 16, 0, 8, None, 0, 0, None, None), ep.EP_ERR_INVALID_ARG),    # recv misaligned
    ((16, 4, 64, 2, 16, 0, 16, None, 0, 0, 18, None), ep.EP_ERR_INVALID_ARG),     # d_err misaligned
    ((16, 4, 64, 2, 16, 0, 16, None, -1, 0, None, None), ep.EP_ERR_INVALID_ARG),  # recv_rows
])
def test_dispatch_rejects(args, status):
    assert ep.lib().ep_dispatch(*args) == status


def test_dispatch_combine_empty_batch_is_a_no_op():
    # T = 0: valid, nothing to do, nothing touched (no device needed)
    assert ep.lib().ep_dispatch(None, 0, 64, 2, None, 0, None, None, 0, 0, None, None) == ep.EP_OK
    assert ep.lib().ep_combine(None, 0, 0, 64, 2, None, None, None, 0, None, None) == ep.EP_OK


@pytest.mark.parametrize("args,status", [
    ((None, 0, 4, 64, 2, 16, None, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),  # no y
    ((16, 0, 4, 64, 2, 16, 18, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),    # w misaligned
    ((16, 0, 4, 60, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_UNSUPPORTED),
    ((16, 0, 4, 64, 2, 16, 16, 40, 0, None, None), ep.EP_ERR_INVALID_ARG),    # out misaligned
    ((16, 0, 4, 64, 2, 16, 16, 16, 0, 2, None), ep.EP_ERR_INVALID_ARG),       # d_err misaligned
    ((16, -1, 4, 64, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),  # y_rows
])
def test_combine_rejects(args, status):
    assert ep.lib().ep_combine(*args) == status


@pytest.mark.parametrize("args,status", [
    ((16, -1, 8, 16, 16, 16, 16, None, 0, None), ep.EP_ERR_INVALID_ARG),
    ((16, 4, 0, 16, 16, 16, 16, None, 0, None), ep.EP_ERR_INVALID_ARG),
    ((16, 4, 65, 16, 16, 16, 16, None, 0, None), ep.EP_ERR_UNSUPPORTED),
    ((None, 4, 8, 16, 16, 16, 16, None, 0, None), ep.EP_ERR_INVALID_ARG),
    ((16, 4, 8, None, 16, 16, 16, None, 0, None), ep.EP_ERR_INVALID_ARG),
    ((16, 4, 8, 16, 16, 18, 16, None, 0, None), ep.EP_ERR_INVALID_ARG),   # rank_row
    ((16, 70000, 8, 16, 16, 16, 16, None, 0, None), ep.EP_ERR_INVALID_ARG),  # tiled, no ws
])
def test_rank_layout_rejects(args, status):
    assert ep.lib().ep_get_rank_layout(*args) == status


def test_rank_layout_workspace_sizes():
    assert ep.ep_rank_layout_workspace_bytes(4096, 8) == 0
    assert ep.ep_rank_layout_workspace_bytes(70000, 8) == ep.ep_layout_workspace_bytes(70000, 8, 8, 1)
    assert ep.ep_rank_layout_workspace_bytes(70000, 8) > 0


def _layout_dispatch_call(**kw):
    a = dict(idx=16, idx_is_int64=1, T=4, k=2, E=8, R=2, x=16, H=512, fp8=0, cnt_e=16,
             cnt_r=16, in_rank=16, off_e=16, off_r=16, slot_pos=16, recv_src=16, recv=16,
             recv_scale=None, ws=None, ws_bytes=0, num_sms=0, d_err=None, stream=None)
    a.update(kw)
    return ep.lib().ep_layout_dispatch(*a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), ep.EP_ERR_INVALID_ARG),
    (dict(E=9), ep.EP_ERR_INVALID_ARG),                     # E % R != 0
    (dict(k=33, E=64), ep.EP_ERR_UNSUPPORTED),
    (dict(idx=None), ep.EP_ERR_INVALID_ARG),
    (dict(slot_pos=None), ep.EP_ERR_INVALID_ARG),
    (dict(x=None), ep.EP_ERR_INVALID_ARG),
    (dict(x=24), ep.EP_ERR_INVALID_ARG),                    # x misaligned
    (dict(recv=None), ep.EP_ERR_INVALID_ARG),
    (dict(H=12), ep.EP_ERR_UNSUPPORTED),                    # H % 8
    (dict(H=0), ep.EP_ERR_INVALID_ARG),
    (dict(fp8=1, H=64, recv_scale=16), ep.EP_ERR_UNSUPPORTED),   # fp8, H % 128
    (dict(fp8=1), ep.EP_ERR_INVALID_ARG),                   # fp8, no scales
    (dict(num_sms=-1), ep.EP_ERR_INVALID_ARG),
    (dict(d_err=2), ep.EP_ERR_INVALID_ARG),
    (dict(T=65537, k=8, E=256, R=8), ep.EP_ERR_INVALID_ARG),     # two-kernel path, no ws
])
def test_layout_dispatch_rejects(kw, status):
    assert _layout_dispatch_call(**kw) == status
    assert ep.lib().ep_last_error_string().decode()


@pytest.mark.parametrize("args,status", [
    ((None, 16, 0, 4, 128, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),   # no codes
    ((16, None, 0, 4, 128, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),   # no scales
    ((16, 16, 0, 4, 64, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_UNSUPPORTED),      # H % 128
    ((16, 16, -1, 4, 128, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),    # y_rows
    ((24, 16, 0, 4, 128, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),     # codes align
    ((16, 18, 0, 4, 128, 2, 16, 16, 16, 0, None, None), ep.EP_ERR_INVALID_ARG),     # scale align
    ((16, 16, 0, 4, 128, 33, 16, 16, 16, 0, None, None), ep.EP_ERR_UNSUPPORTED),    # k > 32
    ((16, 16, 0, 4, 128, 2, 16, 16, 40, 0, None, None), ep.EP_ERR_INVALID_ARG),     # out align
])
def test_combine_fp8_rejects(args, status):
    assert ep.lib().ep_combine_fp8(*args) == status
    assert ep.lib().ep_last_error_string().decode()


def test_combine_fp8_empty_batch_is_a_no_op():
    assert ep.lib().ep_combine_fp8(None, None, 0, 0, 128, 2, None, None, None, 0, None,
                                   None) == ep.EP_OK


def test_aligned_rows():
    assert ep.ep_aligned_rows(4096, 8, 256, 128) == 4096 * 8 + 256 * 127
    assert ep.ep_aligned_rows(10, 2, 4, 1) == 20
    assert ep.ep_aligned_rows(0, 2, 4, 3) == 8
    assert ep.ep_aligned_rows(10, 2, 4, 0) == 0
    assert ep.ep_aligned_rows(1 << 30, 4, 4, 2) == 0      # does not fit int32


@pytest.mark.parametrize("args,status", [
    ((16, 16, -1, 2, 4, 2, 16, 16, 16, None), ep.EP_ERR_INVALID_ARG),
    ((16, 16, 4, 0, 4, 2, 16, 16, 16, None), ep.EP_ERR_INVALID_ARG),
    ((16, 16, 4, 2, 0, 2, 16, 16, 16, None), ep.EP_ERR_INVALID_ARG),
    ((16, 16, 4, 2, 4, 0, 16, 16, 16, None), ep.EP_ERR_INVALID_ARG),         # align
    ((16, 16, 4, 2, 2048, 2, 16, 16, 16, None), ep.EP_ERR_UNSUPPORTED),      # E
    ((16, 16, 1 << 29, 8, 4, 2, 16, 16, 16, None), ep.EP_ERR_UNSUPPORTED),   # rows overflow
    ((None, 16, 4, 2, 4, 2, 16, 16, 16, None), ep.EP_ERR_INVALID_ARG),       # cnt_e
    ((16, None, 4, 2, 4, 2, 16, 16, 16, None), ep.EP_ERR_INVALID_ARG),       # slot_pos
    ((16, 16, 4, 2, 4, 2, None, 16, 16, None), ep.EP_ERR_INVALID_ARG),       # off_pad
    ((16, 16, 4, 2, 4, 2, 16, 18, 16, None), ep.EP_ERR_INVALID_ARG),         # slot_pos_pad
    ((16, 16, 4, 2, 4, 2, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),       # recv_src_pad
])
def test_pad_layout_rejects(args, status):
    assert ep.lib().ep_pad_layout(*args) == status


@pytest.mark.parametrize("args,status", [
    ((16, 1, -1, 2, 4, 16, 16, 16, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),
    ((16, 1, 4, 0, 4, 16, 16, 16, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),
    ((16, 1, 4, 2, 0, 16, 16, 16, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),
    ((None, 1, 4, 2, 4, 16, 16, 16, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),  # idx
    ((20, 1, 4, 2, 4, 16, 16, 16, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),    # int64 align
    ((16, 1, 4, 2, 4, None, 16, 16, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),  # slot_pos
    ((16, 1, 4, 2, 4, 16, None, 16, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),  # off_e
    ((16, 1, 4, 2, 4, 16, 16, None, 16, 16, None, None), ep.EP_ERR_INVALID_ARG),  # rep_off
    ((16, 1, 4, 2, 4, 16, 16, 16, None, 16, None, None), ep.EP_ERR_INVALID_ARG),  # rep_ids
    ((16, 1, 4, 2, 4, 16, 16, 16, 16, None, None, None), ep.EP_ERR_INVALID_ARG),  # phys_idx
    ((16, 1, 4, 2, 4, 16, 16, 16, 16, 16, 2, None), ep.EP_ERR_INVALID_ARG),       # d_err
])
def test_map_replicas_rejects(args, status):
    assert ep.lib().ep_map_replicas(*args) == status


def test_read_error_rejects_null():
    assert ep.lib().ep_read_error(None, None) == ep.EP_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ep, "_lib", None)
    monkeypatch.setattr(ep, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ep.EPLibraryError):
        ep.lib()
