"""Pins of the oracle's rank layout (rows of the rank-deduplicated dispatch)
and of the unit-weight combine: a hand-worked case, numpy cumulative sums,
the invariants of the definition, and the identity with the expert layout of
the mask."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _golden import GOLDEN


def _hand():
    d = {}
    with open(f"{GOLDEN}/rank_layout_hand.txt") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, vals = line.split(":", 1)
                d[key.strip()] = [int(v) for v in vals.split()]
    return d


def test_hand_worked():
    d = _hand()
    T, R = d["T"][0], d["R"][0]
    out = oracle.rank_layout(np.array(d["in_rank"], np.uint8).reshape(T, R))
    for key in ("cnt_r", "off_r", "rank_row", "rank_src"):
        np.testing.assert_array_equal(out[key].reshape(-1), d[key], err_msg=key)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_vs_numpy_cumsum(seed):
    rng = np.random.default_rng(seed)
    m = (rng.random((500, 16)) < 0.3).astype(np.uint8)
    out = oracle.rank_layout(m)
    cnt = m.sum(axis=0).astype(np.int64)
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)
    before = np.cumsum(m.astype(np.int64), axis=0) - m   # earlier tokens, same rank
    want = np.where(m == 1, off[:-1][None, :] + before, -1)
    np.testing.assert_array_equal(out["cnt_r"], cnt)
    np.testing.assert_array_equal(out["off_r"], off)
    np.testing.assert_array_equal(out["rank_row"], want)
    # rank_src inverts rank_row; rows past the last are -1
    n = off[-1]
    t_of = np.full(m.size, -1)
    rows = want[m == 1]
    t_of[rows] = np.nonzero(m)[0]
    np.testing.assert_array_equal(out["rank_src"][:n], t_of[:n])
    assert np.all(out["rank_src"][n:] == -1)


def test_matches_expert_layout_of_the_mask():
    # the rank rows are the expert layout of "slot (t, r) chooses expert r"
    cfg = workloads.CONFIGS["prefill"]
    b = workloads.make_batch(cfg, 3, T=300, H=8, drop_frac=0.1)
    L = oracle.layout(b.idx, cfg.E, cfg.R)
    m = L["in_rank"]
    R = cfg.R
    ids = np.where(m == 1, np.arange(R)[None, :], -1).astype(np.int64)
    via_experts = oracle.layout(ids, R, 1)
    out = oracle.rank_layout(m)
    np.testing.assert_array_equal(out["rank_row"], via_experts["slot_pos"])
    np.testing.assert_array_equal(out["rank_src"], via_experts["recv_src"])
    np.testing.assert_array_equal(out["cnt_r"], L["cnt_r"])
    np.testing.assert_array_equal(out["off_r"], L["off_r"])
    # rows per token = distinct ranks <= min(k, R)
    assert out["off_r"][-1] == m.sum() <= 300 * min(cfg.k, R)


def test_unit_weight_combine_is_plain_sum():
    rng = np.random.default_rng(4)
    y = torch.from_numpy(rng.standard_normal((12, 16)).astype(np.float32)).to(torch.bfloat16)
    sp = np.array([[0, 3, -1], [5, -1, -1], [-1, -1, -1], [7, 8, 11]], np.int32)
    got = oracle.bits_to_bf16(oracle.combine(y, sp, None)).float()
    yf = y.float()
    for t in range(4):
        acc = torch.zeros(16)
        for r in sp[t]:
            if r >= 0:
                acc = acc + yf[r]                   # fp32 adds in slot order
        assert torch.equal(got[t], acc.to(torch.bfloat16).float())
