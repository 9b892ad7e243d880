"""Pins of the oracle's aligned layout and FP8 combine against what fixes
them independently of the oracle's own code: hand-worked layouts, the
plain layout (align = 1), properties of every expert segment on brute-force
inputs, torch's float8 decoding, and the pinned bf16 combine on values that
bf16 holds exactly."""
import itertools

import numpy as np
import pytest
import torch

import oracle
from _golden import layout_aligned_cases


@pytest.mark.parametrize("case", layout_aligned_cases(), ids=lambda c: f"T{c['T']}a{c['align']}")
def test_aligned_layout_hand_cases(case):
    idx = torch.tensor(case["idx"], dtype=torch.int64).view(case["T"], case["k"])
    got = oracle.layout_aligned(idx, case["E"], case["align"])
    assert got["off_pad"].tolist() == case["off_pad"]
    assert got["slot_pos"].reshape(-1).tolist() == case["slot_pos"]
    assert got["recv_src"].tolist() == case["recv_src"]
    assert got["status"] == oracle.ORACLE_OK


@pytest.mark.parametrize("seed", range(4))
def test_align_one_is_the_plain_layout(seed):
    rng = np.random.default_rng(seed)
    T, k, E, R = 50, 4, 16, 4
    idx = torch.from_numpy(rng.integers(-1, E, (T, k)).astype(np.int64))
    plain = oracle.layout(idx, E, R)
    al = oracle.layout_aligned(idx, E, 1)
    np.testing.assert_array_equal(al["off_pad"], plain["off_e"])
    np.testing.assert_array_equal(al["slot_pos"], plain["slot_pos"])
    np.testing.assert_array_equal(al["recv_src"], plain["recv_src"])


def _check_segments(idx, E, align, got):
    """Every expert segment from the definition, by enumeration."""
    ix = idx.numpy()
    T, k = ix.shape
    off = got["off_pad"]
    src = got["recv_src"]
    assert len(src) == T * k + E * (align - 1)
    assert off[0] == 0
    for e in range(E):
        tokens = [t for t in range(T) for j in range(k) if ix[t, j] == e]
        seg = off[e + 1] - off[e]
        assert off[e] % align == 0
        assert seg % align == 0 and len(tokens) <= seg < len(tokens) + align
        assert src[off[e]:off[e] + len(tokens)].tolist() == tokens
        assert (src[off[e] + len(tokens):off[e + 1]] == -1).all()
    assert (src[off[E]:] == -1).all()
    for t in range(T):
        for j in range(k):
            r = got["slot_pos"][t, j]
            if 0 <= ix[t, j] < E:
                assert off[ix[t, j]] <= r < off[ix[t, j] + 1] and src[r] == t
                # the slot's place among its expert's slots in token-major order
                before = sum(1 for t2 in range(T) for j2 in range(k)
                             if ix[t2, j2] == ix[t, j] and (t2, j2) < (t, j))
                assert r == off[ix[t, j]] + before
            else:
                assert r == -1


def test_aligned_layout_brute_force_tiny():
    # every id assignment of 3 tokens x 2 slots over {-1, 0, 1, 2}, E = 3
    E, T, k = 3, 3, 2
    for align in (1, 2, 3, 5):
        for flat in itertools.product(range(-1, E), repeat=T * k):
            idx = torch.tensor(flat, dtype=torch.int64).view(T, k)
            _check_segments(idx, E, align, oracle.layout_aligned(idx, E, align))


@pytest.mark.parametrize("align", [2, 7, 128])
def test_aligned_layout_random(align):
    rng = np.random.default_rng(align)
    T, k, E = 40, 8, 32
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int64)
    idx[rng.random(idx.shape) < 0.1] = -1
    idx = torch.from_numpy(idx)
    _check_segments(idx, E, align, oracle.layout_aligned(idx, E, align))


def test_aligned_layout_bad_id_reported():
    idx = torch.tensor([[0, 5], [1, -3]], dtype=torch.int64)
    got = oracle.layout_aligned(idx, 4, 2)
    assert got["status"] == oracle.ORACLE_ERR_INDEX
    assert got["slot_pos"].tolist() == [[0, -1], [2, -1]]


# ----------------------------------------------------------- FP8 combine

def _fp8_rows(rng, n, H, scale_exp=None):
    q = torch.from_numpy(rng.integers(0, 256, (n, H), dtype=np.uint8))
    q[(q & 0x7F) == 0x7F] = 0x10           # no NaN codes
    if scale_exp is None:
        s = torch.from_numpy((rng.random((n, H // 128)) * 0.1 + 1e-3).astype(np.float32))
    else:
        s = torch.from_numpy(np.ldexp(1.0, rng.integers(-scale_exp, scale_exp,
                                                          (n, H // 128))).astype(np.float32))
    return q, s


def _decode(q, s):
    """torch's float8 decoding times the block scale, in fp32."""
    v = q.view(torch.float8_e4m3fn).float()
    return v * s.repeat_interleave(128, dim=1)


def test_fp8_combine_single_slot_is_the_decoded_row():
    rng = np.random.default_rng(1)
    T, H = 6, 256
    q, s = _fp8_rows(rng, T, H)
    slot = torch.arange(T, dtype=torch.int32).view(T, 1)
    out = oracle.combine_fp8(q, s, slot, torch.ones(T, 1))
    # the chain starts from +0, so a -0 code (0x80) comes out as +0
    want = (_decode(q, s) + 0.0).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(out, want)


def test_fp8_combine_equals_bf16_combine_on_exact_values():
    # with power-of-two scales every decoded value has at most 4 significant
    # bits, so bf16 holds it exactly: the FP8 combine must then equal the
    # (separately pinned) bf16 combine of those values, slot for slot
    rng = np.random.default_rng(2)
    T, k, H = 9, 4, 384
    n = T * k + 5
    q, s = _fp8_rows(rng, n, H, scale_exp=8)
    y = _decode(q, s).to(torch.bfloat16)
    assert torch.equal(y.float(), _decode(q, s))
    slot = torch.from_numpy(rng.permutation(n)[:T * k].astype(np.int32)).view(T, k)
    slot[0, 1] = -1
    slot[3, 0] = n + 4                      # outside the buffer: skipped
    w = torch.from_numpy(rng.random((T, k)).astype(np.float32))
    np.testing.assert_array_equal(oracle.combine_fp8(q, s, slot, w),
                                  oracle.combine(y, slot, w))
    np.testing.assert_array_equal(oracle.combine_fp8(q, s, slot, None),
                                  oracle.combine(y, slot, None))


def test_fp8_dispatch_then_combine_round_trip():
    # identity experts on the FP8 receive rows, weights summing to 1: out is
    # x within the e4m3 error (2^-4 relative on normal codes, plus the
    # subnormal step s * 2^-9 and the bf16 rounding of out)
    rng = np.random.default_rng(3)
    T, k, H = 16, 4, 512
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16)
    slot = torch.arange(T * k, dtype=torch.int32).view(T, k)
    q, s = oracle.dispatch_fp8(x, slot, T * k)
    w = torch.from_numpy(rng.dirichlet(np.ones(k), T).astype(np.float32))
    out = oracle.combine_fp8(q, s, slot, w)
    got = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).float()
    xf = x.float()
    srow = torch.from_numpy(s[::k].copy()).repeat_interleave(128, dim=1)
    bound = xf.abs() * (2.0 ** -4) * 1.01 + srow * 2.0 ** -9 + got.abs() * 2.0 ** -8
    assert ((got - xf).abs() <= bound).all()


# -------------------------------------------------------------- replicas

def test_replicas_one_copy_each_is_a_relabelling():
    rng = np.random.default_rng(4)
    T, k, E = 60, 4, 12
    idx = torch.from_numpy(rng.integers(-1, E, (T, k)).astype(np.int64))
    perm = rng.permutation(E).astype(np.int32)
    phys, st = oracle.map_replicas(idx, np.arange(E + 1, dtype=np.int32), perm)
    want = np.where(idx.numpy() >= 0, perm[np.clip(idx.numpy(), 0, None)], -1)
    np.testing.assert_array_equal(phys, want)
    assert st == oracle.ORACLE_OK


def test_replicas_hand_case():
    # expert 0 has copies {5, 3}, expert 1 the single copy {4}; slots of
    # expert 0 in token-major order: (0,0) (1,1) (2,0) (3,1) -> 5 3 5 3
    idx = torch.tensor([[0, 1], [1, 0], [0, -1], [1, 0]], dtype=torch.int64)
    phys, st = oracle.map_replicas(idx, np.array([0, 2, 3], np.int32),
                                   np.array([5, 3, 4], np.int32))
    assert phys.tolist() == [[5, 4], [4, 3], [5, -1], [4, 3]]
    assert st == oracle.ORACLE_OK


def test_replicas_balance_and_order_brute_force():
    # every copy of a logical expert gets floor or ceil of its share, and the
    # copies are dealt in the order the slots come (checked by enumeration)
    rng = np.random.default_rng(5)
    T, k, E = 200, 6, 10
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int64)
    idx[rng.random(idx.shape) < 0.1] = -1
    n_rep = rng.integers(1, 5, E)
    rep_off = np.concatenate([[0], np.cumsum(n_rep)]).astype(np.int32)
    rep_ids = rng.permutation(int(rep_off[-1])).astype(np.int32)
    phys, st = oracle.map_replicas(torch.from_numpy(idx), rep_off, rep_ids)
    assert st == oracle.ORACLE_OK
    for e in range(E):
        slots = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e]
        copies = rep_ids[rep_off[e]:rep_off[e + 1]]
        got = [phys[t, j] for t, j in slots]
        assert got == [copies[i % len(copies)] for i in range(len(slots))]
        counts = [got.count(c) for c in copies]
        assert max(counts) - min(counts) <= 1
    assert ((phys == -1) == (idx == -1)).all()


def test_replicas_bad_ids_and_experts_without_copies():
    idx = torch.tensor([[0, 7], [1, 2]], dtype=torch.int64)
    phys, st = oracle.map_replicas(idx, np.array([0, 1, 1, 2], np.int32),
                                   np.array([9, 8], np.int32))
    assert st == oracle.ORACLE_ERR_INDEX
    assert phys.tolist() == [[9, -1], [-1, 8]]        # expert 1 has no copy
