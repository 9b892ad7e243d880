"""GPU parity of the rank-deduplicated path (one receive row per (token,
rank) pair): rank rows bit-exact against the oracle on the workloads'
token-in-rank masks (cluster and tiled layouts), bf16 and FP8 dispatch into
rank rows bit-exact, and the unit-weight combine of per-rank partial
outputs bit-exact."""
import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads
from _parity import tensor_bits16, tensor_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ep.lib()


def _mask(name, seed, T=None, H=8, drop=0.0):
    cfg = workloads.CONFIGS[name]
    b = workloads.make_batch(cfg, seed, T=T, H=H, drop_frac=drop)
    L = ep.ep_get_layout(b.idx.cuda(), cfg.E, cfg.R)
    return cfg, b, L


def _check_rank_layout(in_rank_dev):
    RL = ep.ep_get_rank_layout(in_rank_dev)
    ref = oracle.rank_layout(in_rank_dev.cpu().numpy())
    for key in ("cnt_r", "off_r", "rank_row", "rank_src"):
        np.testing.assert_array_equal(getattr(RL, key).cpu().numpy().reshape(-1),
                                      ref[key].reshape(-1), err_msg=key)
    return RL, ref


@pytest.mark.parametrize("name", list(workloads.CONFIGS))
def test_rank_layout_workloads(name):
    cfg, b, L = _mask(name, 0)
    RL, ref = _check_rank_layout(L.in_rank)
    np.testing.assert_array_equal(RL.cnt_r.cpu().numpy(), L.cnt_r.cpu().numpy())


@pytest.mark.parametrize("T", [0, 1, 255, 2049, 8192, 65536, 70001])
def test_rank_layout_ragged_and_tiled(T):
    # T * R from 65536 (8192 x 8) to 2^19 (65536 x 8) takes the grid
    # kernel, above 2^19 (70001 x 8) the tiled layout, both with a workspace
    cfg, b, L = _mask("prefill", 1, T=T, drop=0.2)
    _check_rank_layout(L.in_rank)


def test_rank_layout_64_ranks_random_mask():
    rng = np.random.default_rng(5)
    m = torch.from_numpy((rng.random((3000, 64)) < 0.1).astype(np.uint8)).cuda()
    _check_rank_layout(m)


@pytest.mark.parametrize("fp8", [False, True])
def test_dedup_dispatch_and_combine(fp8):
    cfg, b, L = _mask("prefill", 2, T=700, H=1024, drop=0.05)
    T, H, R = b.T, b.H, cfg.R
    RL, ref = _check_rank_layout(L.in_rank)
    x = b.x.cuda()
    n = T * R
    if fp8:
        q = torch.full((n, H), 0x5A, dtype=torch.uint8, device="cuda")
        s = torch.full((n, H // 128), -1.0, dtype=torch.float32, device="cuda")
        ep.ep_dispatch(x, RL.rank_row, fp8=True, recv=q, recv_scale=s)
        wq, ws_ = oracle.dispatch_fp8(b.x, ref["rank_row"], n,
                                      np.full((n, H), 0x5A, np.uint8),
                                      np.full((n, H // 128), -1.0, np.float32))
        np.testing.assert_array_equal(tensor_bytes(q), wq)
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), ws_.view(np.uint32))
    else:
        recv = torch.full((n, H), -23131, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        ep.ep_dispatch(x, RL.rank_row, recv=recv)
        want = oracle.dispatch_bf16(b.x, ref["rank_row"], n, np.full((n, H), 0xA5A5, np.uint16))
        np.testing.assert_array_equal(tensor_bits16(recv), want)
    # combine: per-rank partial outputs z, summed with unit weights
    z = workloads.expert_outputs(b.x, torch.from_numpy(ref["rank_src"]),
                                 torch.from_numpy(ref["off_r"]), "scale")
    out = ep.ep_combine(z.cuda(), RL.rank_row, None)
    want = oracle.combine(z, ref["rank_row"], None)
    np.testing.assert_array_equal(tensor_bits16(out), want)


def test_dedup_rows_fewer_than_expert_rows():
    # group-limited routing (4 of 8 groups): at most 4 rank rows per token
    cfg, b, L = _mask("prefill", 0)
    RL = ep.ep_get_rank_layout(L.in_rank)
    rows = int(RL.off_r[-1])
    assert rows <= 4 * b.T < b.T * cfg.k
