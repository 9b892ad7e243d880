"""ep_get_layout_noalloc: the layout entry point for callers that cannot
allocate device memory -- a runtime whose device memory all belongs to its
own pool (an extra cudaMalloc would fail or break its accounting), or a
loop that must not pay the implicit synchronisation of cudaMalloc and
cudaFree.  It uses a fixed scratch array inside the library instead of a
caller workspace.  These tests check, through the C ABI, that calls in a
row on that shared array give exactly what the oracle and ep_get_layout
(with a fresh workspace) give, that a call allocates no device memory,
that it works on a side stream, and that a batch too big for the array, or
an input the current device cannot use, is refused up front.  (This file
sorts last so that a run stopping at the first failure has run every other
test already.)"""
import ctypes

import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads

KEYS = ("cnt_e", "cnt_r", "in_rank", "off_e", "off_r", "slot_pos", "recv_src")


def test_noalloc_refuses_batches_larger_than_its_scratch():
    # 100000 tokens, top-8 over 1024 experts in 64 ranks needs ~1.2 MiB of
    # scratch; the call must say so before touching the device
    T, k, E, R = 100000, 8, 1024, 64
    assert ep.ep_layout_workspace_bytes(T, k, E, R) > ep.EP_NOALLOC_SCRATCH_BYTES
    st = ep.lib().ep_get_layout_noalloc(16, 1, T, k, E, R, 16, 16, 16, 16, 16,
                                        16, 16, None, None)
    assert st == ep.EP_ERR_UNSUPPORTED
    assert "scratch" in ep.lib().ep_last_error_string().decode()


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check_against(got, want: dict, name: str):
    for key in KEYS:
        np.testing.assert_array_equal(getattr(got, key).cpu().numpy().reshape(-1),
                                      np.asarray(want[key]).reshape(-1),
                                      err_msg=f"{name}: {key}")


# batches of the large workload's routing (128 experts in 16 ranks, top-8)
# whose layouts use the scratch: two for the tiled kernels (T*k > 2^19),
# then one for the grid kernel (65536 <= T*k <= 2^19, barrier counters
# in the scratch), after a tiled one on the same array
BATCHES = ((70000, 0), (66000, 1), (32768, 2))


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_workspace_entry_point_two_calls_in_a_row():
    _need_gpu()
    dev = torch.device("cuda")
    cfg = workloads.CONFIGS["large"]
    for T, seed in BATCHES:
        assert 0 < ep.ep_layout_workspace_bytes(T, cfg.k, cfg.E, cfg.R) \
            <= ep.EP_NOALLOC_SCRATCH_BYTES
        b = workloads.make_batch(cfg, seed, T=T, H=8)
        idx = b.idx.to(dev)
        ref = oracle.layout(b.idx, cfg.E, cfg.R)
        want = ep.ep_get_layout(idx, cfg.E, cfg.R)
        # the second batch finds the first one's counters in the array
        got = ep.ep_get_layout_noalloc(idx, cfg.E, cfg.R)
        torch.cuda.synchronize()
        _check_against(got, ref, f"T={T} vs oracle")
        _check_against(got, {k: getattr(want, k).cpu().numpy() for k in KEYS},
                       f"T={T} vs ep_get_layout")


@pytest.mark.gpu
def test_noalloc_allocates_nothing_and_runs_on_a_side_stream():
    _need_gpu()
    dev = torch.device("cuda")
    cfg = workloads.CONFIGS["large"]
    T, seed = BATCHES[0]
    b = workloads.make_batch(cfg, seed, T=T, H=8)
    idx = b.idx.to(dev)
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    out = ep.empty_layout(T, cfg.k, cfg.E, cfg.R, dev)
    side = torch.cuda.Stream(dev)
    ep.ep_get_layout_noalloc(idx, cfg.E, cfg.R, out=out)   # first call: set-up
    torch.cuda.synchronize()
    for stream in (None, side):
        for key in KEYS:
            getattr(out, key).fill_(-7 if key != "in_rank" else 7)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info(dev)
        ep.ep_get_layout_noalloc(idx, cfg.E, cfg.R, out=out, stream=stream)
        if stream is not None:
            stream.synchronize()
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info(dev)
        assert free1 == free0, f"device memory changed by {free0 - free1} bytes"
        _check_against(out, ref, "side stream" if stream is not None else "current stream")


@pytest.mark.gpu
def test_noalloc_refuses_input_the_current_device_cannot_use():
    # the scratch is the current device's: ids in plain host memory (or on
    # another device) are refused before anything is enqueued
    _need_gpu()
    dev = torch.device("cuda")
    cfg = workloads.CONFIGS["large"]
    T = BATCHES[0][0]
    host_idx = workloads.make_batch(cfg, 0, T=T, H=8).idx.contiguous()
    out = ep.empty_layout(T, cfg.k, cfg.E, cfg.R, dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = ep.lib().ep_get_layout_noalloc(
        p(host_idx), 1, T, cfg.k, cfg.E, cfg.R, p(out.cnt_e), p(out.cnt_r), p(out.in_rank),
        p(out.off_e), p(out.off_r), p(out.slot_pos), p(out.recv_src), None, None)
    assert st == ep.EP_ERR_INVALID_ARG
    assert "idx" in ep.lib().ep_last_error_string().decode()
    # and the binding says so for a tensor on the wrong device
    with pytest.raises(ValueError):
        ep.ep_get_layout_noalloc(host_idx, cfg.E, cfg.R, out=out)
