"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
the oracle on the same seeded batch, and compare."""
import numpy as np
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads

LAYOUT_KEYS = ("cnt_e", "cnt_r", "in_rank", "off_e", "off_r", "slot_pos", "recv_src")


def gpu_layout(idx_cpu: torch.Tensor, E: int, R: int, int32_ids: bool = False):
    dev = torch.device("cuda")
    idx = idx_cpu.to(torch.int32 if int32_ids else torch.int64).to(dev)
    d_err = torch.zeros(1, dtype=torch.int32, device=dev)
    L = ep.ep_get_layout(idx, E, R, d_err=d_err)
    status = ep.ep_read_error(d_err)
    host = {k: getattr(L, k).cpu().numpy() for k in LAYOUT_KEYS}
    host["status"] = status
    return L, host


def assert_layout_equal(gpu: dict, ref: dict):
    for key in LAYOUT_KEYS:
        np.testing.assert_array_equal(np.asarray(gpu[key]).reshape(-1),
                                      np.asarray(ref[key]).reshape(-1),
                                      err_msg=key)
    assert gpu["status"] == ref["status"]


def bf16_ulp_dist(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns
    (patterns mapped to a monotone integer line; +0 and -0 are 1 apart)."""
    def ordered(h):
        h = h.astype(np.int32)
        return np.where(h & 0x8000, 0x8000 - (h & 0x7FFF), 0x8000 + h)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def tensor_bits16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def tensor_bytes(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def assert_scales_equal(got: np.ndarray, want: np.ndarray):
    """Scale bits equal, except that a NaN scale only has to be a NaN: the
    reading makes a block with a NaN get a NaN scale, and its payload bits
    are not part of it (C division keeps the operand's payload, the GPU
    returns its canonical NaN)."""
    nan = np.isnan(want)
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got.view(np.uint32)[~nan], want.view(np.uint32)[~nan])


def nan_inf_batch(cfg, seed, T, H):
    """A batch whose blocks hold NaNs and infinities (reading c7): a NaN
    makes its block's amax NaN (it sorts above inf), hence a NaN scale and
    all codes 0x7f; an infinite amax gives an infinite scale, under which
    finite values become signed zeros and the infinities NaN (inf / inf)."""
    b = workloads.make_batch(cfg, seed, T=T, H=H)
    x = b.x.float()
    nan, inf = float("nan"), float("inf")
    x[0, 5] = nan                     # one NaN in block 0
    x[1, 130] = inf                   # +inf in block 1
    x[2, 300] = -inf                  # -inf in block 2
    x[3] = nan                        # a whole row of NaN
    x[4, 10], x[4, 20] = inf, nan     # both in one block
    x[6, :128] = inf                  # a block of +inf, then one of -inf
    x[6, 128:256] = -inf
    b.x = x.to(torch.bfloat16)
    b.x.view(torch.int16)[5, H - 7] = -64   # 0xffc0: a NaN with its sign bit set
    return b
