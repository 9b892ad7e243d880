"""Pins of the oracle's number conversions: fp32 -> bf16 (RNE) and
fp32 -> FP8 E4M3 (RNE, saturating), against torch's casts, a brute-force
nearest-code search over all 256 codes, and hand-worked encodings."""
import math

import numpy as np
import torch

import oracle
from _golden import e4m3_codes

F448 = 0x43E00000  # bit pattern of 448.0f


def _f32(bits):
    return np.asarray(bits, np.uint32).view(np.float32)


def test_bf16_vs_torch_all_upper_halves():
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x1234], np.uint32)
    bits = (hi[:, None] | lows[None, :]).reshape(-1)
    v = _f32(bits)
    finite = ~np.isnan(v)
    ours = oracle.f32_to_bf16_array(v[finite])
    ref = torch.from_numpy(v[finite]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    nan_out = oracle.f32_to_bf16_array(v[~finite])
    assert np.all((nan_out & 0x7F80) == 0x7F80) and np.all(nan_out & 0x007F)


def test_bf16_roundtrip():
    # bf16 -> fp32 -> bf16 is the identity on non-NaN values (NaN payloads
    # do not survive the trip through a Python float)
    h = np.arange(0, 1 << 16, 97, dtype=np.uint32)
    h = h[(h & 0x7F80) != 0x7F80]
    f = np.array([oracle.bf16_to_f32(int(x)) for x in h], np.float32)
    assert np.array_equal(f.view(np.uint32), h << 16)
    assert np.array_equal(oracle.f32_to_bf16_array(f), h.astype(np.uint16))


def _torch_e4m3(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def test_e4m3_vs_torch_all_bf16_in_range():
    # every bf16 value with |v| <= 448 (torch's cast does not saturate above)
    h = np.arange(1 << 16, dtype=np.uint32)
    v = _f32(h << 16)
    v = v[np.isfinite(v) & (np.abs(v) <= 448)]
    np.testing.assert_array_equal(oracle.f32_to_e4m3_array(v), _torch_e4m3(v))


def test_e4m3_vs_torch_fp32_stride():
    bits = np.arange(0, F448 + 1, 1237, dtype=np.uint32)
    bits = np.concatenate([bits, bits | 0x80000000])
    v = _f32(bits)
    np.testing.assert_array_equal(oracle.f32_to_e4m3_array(v), _torch_e4m3(v))


def test_e4m3_nearest_code_brute_force():
    # decode every finite code; the oracle must pick the nearest one, ties
    # to the even code (lowest mantissa bit 0), and saturate past 448.
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    vals = np.array([oracle.e4m3_to_f32(int(c)) for c in codes], np.float64)
    pos = np.unique(vals[vals > 0])
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)  # exact in fp32
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.uniform(-470, 470, 4000), rng.standard_normal(4000) * 0.01,
        vals, mids, -mids, [2.0 ** -10, -(2.0 ** -10), 447.9, 448.1],
    ]).astype(np.float32)
    got = oracle.f32_to_e4m3_array(xs)
    for x, g in zip(xs.astype(np.float64), got):
        if abs(x) > 448:
            assert g == (0xFE if x < 0 else 0x7E), (x, hex(g))
            continue
        if x == 0:
            continue
        d = np.abs(vals - x)
        cand = codes[d == d.min()]
        cand = cand[[np.sign(oracle.e4m3_to_f32(int(c))) in (0, np.sign(x)) for c in cand]]
        if len(cand) > 1:  # a tie: keep the even code(s)
            cand = cand[(cand & 1) == 0]
        assert g in cand, (x, hex(g), [hex(c) for c in cand])


def test_e4m3_hand_worked_codes():
    for v, code in e4m3_codes():
        assert oracle.f32_to_e4m3(v) == code, (v, hex(code))


def test_e4m3_decode_definition():
    assert oracle.e4m3_to_f32(0x7E) == 448.0
    assert oracle.e4m3_to_f32(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_f32(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_f32(0x38) == 1.0
    assert math.isnan(oracle.e4m3_to_f32(0x7F))
    # decode(encode(c)) == c for every finite code
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.f32_to_e4m3(oracle.e4m3_to_f32(c)) == c
