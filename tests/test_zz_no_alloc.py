"""ep_get_layout_noalloc: the layout entry point for callers that cannot
allocate device memory (a runtime whose memory all belongs to its own pool,
or a loop that must not pay cudaMalloc's implicit synchronisation).  It uses
a fixed scratch array inside the library instead of a caller workspace, so
these tests check that two calls in a row on that shared array give exactly
what ep_get_layout gives with a fresh workspace, and that a batch too big
for the array is refused up front.  (This file sorts last so that a run
stopping at the first failure has run every other test already.)"""
import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
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


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    # two different batches big enough for the tiled (scratch-using) layout,
    # back to back: the second call finds the first one's counters in the
    # shared array
    cfg = workloads.CONFIGS["large"]
    for T, seed in ((70000, 0), (66000, 1)):
        assert 0 < ep.ep_layout_workspace_bytes(T, cfg.k, cfg.E, cfg.R) \
            <= ep.EP_NOALLOC_SCRATCH_BYTES
        name = f"T={T}"
        idx = workloads.make_batch(cfg, seed, T=T, H=8).idx.to(dev)
        want = ep.ep_get_layout(idx, cfg.E, cfg.R)
        got = ep.ep_get_layout_noalloc(idx, cfg.E, cfg.R)
        torch.cuda.synchronize()
        for key in KEYS:
            np.testing.assert_array_equal(getattr(got, key).cpu().numpy(),
                                          getattr(want, key).cpu().numpy(),
                                          err_msg=f"{name}: {key}")
