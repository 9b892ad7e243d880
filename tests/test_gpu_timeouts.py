"""The bounded waits of the bulk-copy kernels, made to run out on purpose.

Every wait of a kernel for its own asynchronous copies is bounded; when the
bound runs out the kernel records EP_ERR_TIMEOUT in d_err, waits (bounded)
for the copies it still has in flight and returns.  No copy here ever
fails, so the testing switch ep_debug_expire_first_wait makes the first
wait of every CTA give up at once while its copy still lands at a valid
address.  Each test checks the status, then that the GPU is still usable:
the same call with the switch off matches the oracle."""
import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads
from _parity import (assert_layout_equal, assert_scales_equal, gpu_layout, tensor_bits16,
                     tensor_bytes)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ep.lib()
    yield
    ep.ep_debug_expire_first_wait(False)


def _expired(call):
    """Status of `call(d_err)` with every CTA's first wait expired."""
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ep.ep_debug_expire_first_wait(True)
    try:
        call(d_err)
    finally:
        ep.ep_debug_expire_first_wait(False)
    return ep.ep_read_error(d_err)


def _normal(call):
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = call(d_err)
    assert ep.ep_read_error(d_err) == ep.EP_OK
    return res


def _setup(name, seed, T, H):
    cfg = workloads.CONFIGS[name]
    b = workloads.make_batch(cfg, seed, T=T, H=H)
    L, g = gpu_layout(b.idx, cfg.E, cfg.R)
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    assert_layout_equal(g, ref)
    return cfg, b, L, ref


# the bf16 combine's bulk-copy pipeline runs under an SM budget once the
# items outgrow one wave of the register kernel (which has no asynchronous
# copies to wait for): T = 200 on 148 SMs, about two items per CTA;
# T = 3000 on 4 SMs, CTAs walking many items each
@pytest.mark.parametrize("T,num_sms", [(200, 148), (3000, 4)])
def test_combine_wait_times_out_then_recovers(T, num_sms):
    cfg, b, L, ref = _setup("decode", 31, T, 7168)
    y = b.x.cuda()[torch.from_numpy(np.maximum(ref["recv_src"], 0)).long().cuda()]
    w = b.w.cuda()
    call = lambda e: ep.ep_combine(y, L.slot_pos, w, num_sms=num_sms, d_err=e)  # noqa: E731
    assert _expired(call) == ep.EP_ERR_TIMEOUT
    out = _normal(call)
    want = oracle.combine(y.cpu(), ref["slot_pos"], b.w)
    np.testing.assert_array_equal(tensor_bits16(out), want)


def test_combine_fp8_wait_times_out_then_recovers():
    # the bulk-copy pipeline of the FP8 combine runs under an SM budget
    cfg, b, L, ref = _setup("decode", 32, 300, 7168)
    T, H, k = b.T, b.H, cfg.k
    q, s = ep.ep_dispatch(b.x.cuda(), L.slot_pos, fp8=True)
    w = b.w.cuda()
    call = lambda e: ep.ep_combine_fp8(q, s, L.slot_pos, w, num_sms=148, d_err=e)  # noqa: E731
    assert _expired(call) == ep.EP_ERR_TIMEOUT
    out = _normal(call)
    want = oracle.combine_fp8(tensor_bytes(q), s.cpu().numpy(), ref["slot_pos"], b.w)
    np.testing.assert_array_equal(tensor_bits16(out), want)


# all SMs: one token per CTA (a single wait each); under an SM budget:
# CTAs walking token ranges with two rows in flight
@pytest.mark.parametrize("num_sms", [0, 7])
def test_dispatch_fp8_wait_times_out_then_recovers(num_sms):
    cfg, b, L, ref = _setup("prefill", 33, 1000, 7168)
    T, H, k = b.T, b.H, cfg.k
    x = b.x.cuda()
    q = torch.empty((T * k, H), dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.empty((T * k, H // 128), dtype=torch.float32, device="cuda")
    call = lambda e: ep.ep_dispatch(x, L.slot_pos, fp8=True, recv=q,  # noqa: E731
                                    recv_scale=s, num_sms=num_sms, d_err=e)
    assert _expired(call) == ep.EP_ERR_TIMEOUT
    _normal(call)
    wq, ws_ = oracle.dispatch_fp8(b.x, ref["slot_pos"], T * k)
    np.testing.assert_array_equal(tensor_bytes(q), wq)
    assert_scales_equal(s.cpu().numpy(), ws_)


# all SMs: the one-token-per-CTA fused kernel; one SM: the token-range one
@pytest.mark.parametrize("num_sms", [0, 1])
@pytest.mark.parametrize("fp8", [True, False])
def test_fused_layout_dispatch_wait_times_out_then_recovers(num_sms, fp8):
    cfg = workloads.CONFIGS["decode"]
    b = workloads.make_batch(cfg, 34)
    T, H, k = b.T, b.H, cfg.k
    idx, x = b.idx.cuda(), b.x.cuda()
    out = ep.empty_layout(T, k, cfg.E, cfg.R, "cuda")
    if fp8:
        recv = torch.empty((T * k, H), dtype=torch.float8_e4m3fn, device="cuda")
        scale = torch.empty((T * k, H // 128), dtype=torch.float32, device="cuda")
    else:
        recv = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
        scale = None
    launches = []

    def call(e):
        n0 = ep.ep_kernel_launches()
        ep.ep_layout_dispatch(idx, cfg.E, cfg.R, x, fp8, out=out, recv=recv,
                              recv_scale=scale, num_sms=num_sms, d_err=e)
        launches.append(ep.ep_kernel_launches() - n0)

    assert _expired(call) == ep.EP_ERR_TIMEOUT
    _normal(call)
    assert launches == [1, 1]
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    host = {key: getattr(out, key).cpu().numpy() for key in ref if key != "status"}
    host["status"] = ref["status"]
    assert_layout_equal(host, ref)
    if fp8:
        wq, ws_ = oracle.dispatch_fp8(b.x, ref["slot_pos"], T * k)
        np.testing.assert_array_equal(tensor_bytes(recv), wq)
        assert_scales_equal(scale.cpu().numpy(), ws_)
    else:
        want = oracle.dispatch_bf16(b.x, ref["slot_pos"], T * k)
        np.testing.assert_array_equal(tensor_bits16(recv), want)


def test_grid_layout_barrier_times_out_then_recovers():
    # the grid layout kernel (one CTA per SM) meets at two barriers between
    # its CTAs; the switch makes the first give up in every CTA that has not
    # seen all arrive, and the workspace's counters must still be left at 0
    cfg = workloads.CONFIGS["large"]
    b = workloads.make_batch(cfg, 35, H=8)
    idx = b.idx.cuda()
    ws = torch.zeros(ep.ep_layout_workspace_bytes(b.T, cfg.k, cfg.E, cfg.R),
                     dtype=torch.uint8, device="cuda")
    out = ep.empty_layout(b.T, cfg.k, cfg.E, cfg.R, "cuda")
    call = lambda e: ep.ep_get_layout(idx, cfg.E, cfg.R, out=out, ws=ws, d_err=e)  # noqa: E731
    assert _expired(call) == ep.EP_ERR_TIMEOUT
    assert not ws[:12].view(torch.int32).any()
    _normal(call)
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    host = {key: getattr(out, key).cpu().numpy() for key in ref if key != "status"}
    host["status"] = ref["status"]
    assert_layout_equal(host, ref)
