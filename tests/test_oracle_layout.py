"""Pins of the oracle's layout step against things other than itself:
hand-worked cases, a library stable sort, exhaustive tiny inputs and the
invariants the layout's definition fixes (counts sum to the kept slots,
offsets are an exclusive scan, placement is a bijection)."""
import itertools

import numpy as np
import pytest

import oracle
import workloads
from _golden import layout_cases


def _by_library(idx, E, R):
    """Layout recomputed with numpy primitives: a stable argsort of the
    expert ids over the token-major slot order gives the receive order."""
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < E)
    order = np.flatnonzero(valid)[np.argsort(flat[valid], kind="stable")]
    n = order.size
    slot = np.full(T * k, -1, np.int64)
    slot[order] = np.arange(n)
    src = np.full(T * k, -1, np.int64)
    src[:n] = order // k
    cnt_e = np.bincount(flat[valid], minlength=E)
    G = E // R
    in_rank = np.zeros((T, R), np.uint8)
    tok = np.repeat(np.arange(T), k)[valid]
    in_rank[tok, flat[valid] // G] = 1
    cnt_r = in_rank.sum(axis=0)
    return dict(cnt_e=cnt_e, off_e=np.concatenate([[0], np.cumsum(cnt_e)]),
                slot_pos=slot.reshape(T, k), recv_src=src, in_rank=in_rank,
                cnt_r=cnt_r, off_r=np.concatenate([[0], np.cumsum(cnt_r)]))


def _same(a, b):
    for key in ("cnt_e", "off_e", "slot_pos", "recv_src", "in_rank", "cnt_r",
                "off_r"):
        np.testing.assert_array_equal(np.asarray(a[key]).reshape(-1),
                                      np.asarray(b[key]).reshape(-1), err_msg=key)


@pytest.mark.parametrize("case", layout_cases(), ids=lambda c: f"T{c['T']}k{c['k']}")
def test_hand_worked(case):
    idx = np.array(case["idx"], np.int64).reshape(case["T"], case["k"])
    L = oracle.layout(idx, case["E"], case["R"])
    assert L["status"] == 0
    _same(L, case)


def test_exhaustive_tiny():
    # every id assignment of 3 tokens x 2 slots over {-1, 0, 1, 2, 3}
    E, R, T, k = 4, 2, 3, 2
    for ids in itertools.product(range(-1, E), repeat=T * k):
        idx = np.array(ids, np.int64).reshape(T, k)
        _same(oracle.layout(idx, E, R), _by_library(idx, E, R))


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skewed"])
@pytest.mark.parametrize("seed", [0, 1])
def test_workloads_vs_library(name, seed):
    cfg = workloads.CONFIGS[name]
    T = min(cfg.T, 2048)
    b = workloads.make_batch(cfg, seed, T=T, H=128)
    L = oracle.layout(b.idx, cfg.E, cfg.R)
    assert L["status"] == 0
    _same(L, _by_library(b.idx.numpy(), cfg.E, cfg.R))


@pytest.mark.parametrize("drop,dup", [(0.0, 0.0), (0.2, 0.0), (0.0, 0.5),
                                      (0.3, 0.3), (1.0, 0.0)])
def test_invariants(drop, dup):
    cfg = workloads.CONFIGS["large"]
    b = workloads.make_batch(cfg, 3, T=1000, H=8, drop_frac=drop, dup_frac=dup)
    idx = b.idx.numpy()
    T, k = idx.shape
    L = oracle.layout(idx, cfg.E, cfg.R)
    n_valid = int((idx >= 0).sum())
    # counts sum to the kept slots; offsets are the exclusive scan
    assert L["cnt_e"].sum() == n_valid
    assert L["off_e"][0] == 0 and L["off_e"][-1] == n_valid
    np.testing.assert_array_equal(np.diff(L["off_e"]), L["cnt_e"])
    np.testing.assert_array_equal(np.diff(L["off_r"]), L["cnt_r"])
    # placement is a bijection between kept slots and rows [0, n_valid)
    sp = L["slot_pos"].reshape(-1)
    kept = sp[idx.reshape(-1) >= 0]
    assert np.all(sp[idx.reshape(-1) < 0] == -1)
    np.testing.assert_array_equal(np.sort(kept), np.arange(n_valid))
    # each row lies inside its expert's segment and points back to its token
    for i in np.flatnonzero(idx.reshape(-1) >= 0):
        e, row = idx.reshape(-1)[i], sp[i]
        assert L["off_e"][e] <= row < L["off_e"][e + 1]
        assert L["recv_src"][row] == i // k
    assert np.all(L["recv_src"][n_valid:] == -1)
    # rows of one expert come in ascending token order (stable)
    for e in range(cfg.E):
        seg = L["recv_src"][L["off_e"][e]:L["off_e"][e + 1]]
        assert np.all(np.diff(seg) >= 0)
    # per-rank counts: deduplicated tokens, bounded by T * min(k, R)
    assert L["cnt_r"].sum() <= T * min(k, cfg.R)
    G = cfg.E // cfg.R
    for t in range(0, T, 37):
        ranks = {int(e) // G for e in idx[t] if e >= 0}
        assert set(np.flatnonzero(L["in_rank"][t])) == ranks


def test_invalid_ids_reported_and_skipped():
    idx = np.array([[0, 5], [-2, 1], [3, -1]], np.int64)
    L = oracle.layout(idx, 4, 2)
    assert L["status"] == oracle.ORACLE_ERR_INDEX
    np.testing.assert_array_equal(L["slot_pos"], [[0, -1], [-1, 1], [2, -1]])
    np.testing.assert_array_equal(L["cnt_e"], [1, 1, 0, 1])


def test_empty():
    L = oracle.layout(np.zeros((0, 4), np.int64), 16, 4)
    assert L["status"] == 0
    assert L["cnt_e"].sum() == 0 and L["off_e"][-1] == 0 and L["off_r"][-1] == 0
