"""Pins of the oracle's dispatch (bf16, FP8) and combine steps.

Against: numpy fancy indexing (dispatch is a row permutation), torch's own
fp32 division and float8_e4m3fn cast (FP8 dispatch on in-range values),
hand-worked blocks and combines, an fp64 reduction (combine within the fp32
chain's error plus one bf16 rounding), and the round trip
combine(dispatch(x)) = x for identity experts with weights summing to 1."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _golden import combine_case, fp8_block

CANARY16 = 0xA5A5
CANARY8 = 0x5A


def _setup(name, seed, T, H, **kw):
    cfg = workloads.CONFIGS[name]
    b = workloads.make_batch(cfg, seed, T=T, H=H, **kw)
    L = oracle.layout(b.idx, cfg.E, cfg.R)
    return cfg, b, L


@pytest.mark.parametrize("drop", [0.0, 0.25])
def test_dispatch_bf16_is_row_gather(drop):
    cfg, b, L = _setup("prefill", 0, 300, 136, drop_frac=drop)
    n = 300 * cfg.k
    recv = np.full((n, 136), CANARY16, np.uint16)
    oracle.dispatch_bf16(b.x, L["slot_pos"], n, recv)
    xb = oracle.bf16_bits(b.x)
    nv = L["off_e"][-1]
    np.testing.assert_array_equal(recv[:nv], xb[L["recv_src"][:nv]])
    assert np.all(recv[nv:] == CANARY16)


def _torch_fp8(x: torch.Tensor):
    """FP8 dispatch payload of each token computed with torch CPU ops:
    fp32 amax per 128-block, clamp 1e-4, s = a / 448 and q = cast(x / s)."""
    T, H = x.shape
    xf = x.to(torch.float32).view(T, H // 128, 128)
    a = xf.abs().amax(dim=2).clamp_min(1e-4)
    s = a / 448.0
    q = (xf / s[:, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return q.reshape(T, H).numpy(), s.numpy()


@pytest.mark.parametrize("name,T,H", [("decode", 128, 7168), ("tiny", 128, 256),
                                      ("skewed", 200, 1024)])
def test_dispatch_fp8_vs_torch(name, T, H):
    cfg, b, L = _setup(name, 1, T, H, drop_frac=0.05)
    n = T * cfg.k
    q, s = oracle.dispatch_fp8(b.x, L["slot_pos"], n,
                               np.full((n, H), CANARY8, np.uint8),
                               np.full((n, H // 128), -1.0, np.float32))
    tq, ts = _torch_fp8(b.x)
    nv = L["off_e"][-1]
    src = L["recv_src"][:nv]
    np.testing.assert_array_equal(q[:nv], tq[src])
    np.testing.assert_array_equal(s[:nv].view(np.uint32), ts[src].view(np.uint32))
    assert np.all(q[nv:] == CANARY8) and np.all(s[nv:] == -1.0)


def test_dispatch_fp8_hand_worked_block():
    chans, scale = fp8_block()
    x = torch.zeros(1, 128, dtype=torch.float32)
    for c, v, _ in chans:
        x[0, c] = v
    xb = x.to(torch.bfloat16)
    assert torch.equal(xb.float(), x)          # fixture values are bf16-exact
    q, s = oracle.dispatch_fp8(xb, np.array([[0]], np.int32), 1)
    assert s[0, 0] == scale
    for c, _, code in chans:
        assert q[0, c] == code, (c, hex(q[0, c]), hex(code))
    listed = {c for c, _, _ in chans}
    assert all(q[0, c] == 0 for c in range(128) if c not in listed)


def test_dispatch_fp8_properties():
    cfg, b, L = _setup("skewed", 2, 64, 2048)
    T, H = 64, 2048
    sp = np.arange(T, dtype=np.int32)[:, None]        # one row per token
    q, s = oracle.dispatch_fp8(b.x, sp, T)
    x = b.x.to(torch.float64).numpy().reshape(T, H // 128, 128)
    deq = np.vectorize(oracle.e4m3_to_f32, otypes=[np.float64])(
        np.arange(256, dtype=np.uint8))[q].reshape(T, H // 128, 128)
    deq = deq * s[:, :, None]
    # the element at the block's amax lands on +-448
    amax_code = (q.reshape(T, H // 128, 128) & 0x7F).max(axis=2)
    assert np.all(amax_code == 0x7E)
    # dequantisation error: half an e4m3 ulp (2^-4 relative) for normals,
    # half the subnormal step 2^-10 * s below 2^-6 * s; slack for x / s
    err = np.abs(deq - x)
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s[:, :, None]) * (1 + 2 ** -20)
    assert np.all(err <= bound)


def test_dispatch_fp8_zero_and_tiny_blocks():
    x = torch.zeros(2, 256, dtype=torch.bfloat16)
    x[1, 128:] = 1e-6                                  # amax below the clamp
    q, s = oracle.dispatch_fp8(x, np.array([[0], [1]], np.int32), 2)
    clamp = np.float32(np.float32(1e-4) / np.float32(448.0))
    assert np.all(s == clamp)
    assert np.all(q[0] == 0) and np.all(q[1, :128] == 0)
    expect = oracle.f32_to_e4m3(float(np.float32(x[1, 200].float().item()) / clamp))
    assert np.all(q[1, 128:] == expect)


def test_dispatch_fp8_nan_propagates():
    x = torch.randn(1, 256).to(torch.bfloat16)
    x[0, 5] = float("nan")
    q, s = oracle.dispatch_fp8(x, np.array([[0]], np.int32), 1)
    assert np.isnan(s[0, 0]) and np.all(q[0, :128] == 0x7F)
    assert np.isfinite(s[0, 1]) and not np.any(q[0, 128:] == 0x7F)


def test_dispatch_fp8_infinite_amax():
    # IEEE arithmetic of the stated steps: amax = inf gives s = inf / 448 =
    # inf; a finite value over inf is a zero of its own sign (e4m3 0x00 /
    # 0x80) and inf / inf is NaN (0x7f); the next block is untouched
    x = torch.randn(1, 256).to(torch.bfloat16)
    x[0, 0] = 2.5
    x[0, 1] = -3.0
    x[0, 7] = float("inf")
    x[0, 9] = float("-inf")
    q, s = oracle.dispatch_fp8(x, np.array([[0]], np.int32), 1)
    assert np.isposinf(s[0, 0]) and np.isfinite(s[0, 1])
    assert q[0, 0] == 0x00 and q[0, 1] == 0x80
    assert q[0, 7] == 0x7F and q[0, 9] == 0x7F
    signs = (x[0, :128].float().numpy() < 0)
    finite = np.isfinite(x[0, :128].float().numpy())
    assert np.all(q[0, :128][finite] == np.where(signs[finite], 0x80, 0x00))


# ------------------------------------------------------------------ combine

def test_combine_hand_worked():
    d = combine_case()
    y = torch.tensor(d["y"], dtype=torch.float32).view(-1, 2).to(torch.bfloat16)
    sp = np.array(d["slot_pos"], np.int32).reshape(2, 2)
    w = np.array(d["w"], np.float32).reshape(2, 2)
    out = oracle.bits_to_bf16(oracle.combine(y, sp, w)).float()
    assert out.flatten().tolist() == d["out"]


def _bf16_ulp_dist(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    def ordered(h):
        h = h.astype(np.int32)
        return np.where(h & 0x8000, 0x8000 - (h & 0x7FFF), 0x8000 + h)
    return np.abs(ordered(a_bits) - ordered(b_bits))


@pytest.mark.parametrize("name,drop", [("prefill", 0.0), ("large", 0.1),
                                       ("skewed", 0.0)])
def test_combine_vs_fp64(name, drop):
    T, H = 256, 512
    cfg, b, L = _setup(name, 4, T, H, drop_frac=drop)
    y = workloads.expert_outputs(b.x, torch.from_numpy(L["recv_src"]),
                                 torch.from_numpy(L["off_e"]), cfg.expert)
    out = oracle.combine(y, L["slot_pos"], b.w)
    # fp64 reference: index_add of w * y over the kept slots
    sp = torch.from_numpy(L["slot_pos"]).long()
    keep = sp >= 0
    tok = torch.arange(T).repeat_interleave(cfg.k).view(T, cfg.k)
    ref = torch.zeros(T, H, dtype=torch.float64)
    contrib = b.w.double()[keep][:, None] * y.double()[sp[keep]]
    ref.index_add_(0, tok[keep], contrib)
    mag = torch.zeros(T, H, dtype=torch.float64).index_add_(0, tok[keep], contrib.abs())
    got = oracle.bits_to_bf16(out).double()
    # fp32 chain: <= k roundings of 2^-24 relative to the running magnitude;
    # then one bf16 rounding: <= 2^-9 relative
    bound = cfg.k * 2.0 ** -24 * mag + 2.0 ** -8 * ref.abs() + 1e-30
    assert torch.all((got - ref).abs() <= bound)
    # tokens with every slot dropped give exactly +0
    dead = ~keep.any(dim=1)
    assert torch.all(got[dead] == 0)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill"])
def test_combine_dispatch_roundtrip_identity(name):
    # identity experts, weights summing to 1: combine(dispatch(x)) = x to
    # within one bf16 ulp
    cfg = workloads.CONFIGS[name]
    T = min(cfg.T, 512)
    cfg, b, L = _setup(name, 5, T, min(cfg.H, 1024))
    n = T * cfg.k
    recv = oracle.dispatch_bf16(b.x, L["slot_pos"], n)
    out = oracle.combine(recv, L["slot_pos"], b.w)
    assert np.abs(b.w.double().sum(1).numpy() - 1).max() < 1e-6
    assert _bf16_ulp_dist(out, oracle.bf16_bits(b.x)).max() <= 1


def test_combine_fp8_roundtrip_within_e4m3_error():
    cfg, b, L = _setup("decode", 6, 64, 1024)
    n = 64 * cfg.k
    q, s = oracle.dispatch_fp8(b.x, L["slot_pos"], n)
    lut = np.vectorize(oracle.e4m3_to_f32, otypes=[np.float32])(np.arange(256, dtype=np.uint8))
    deq = torch.from_numpy(lut[q] * np.repeat(s, 128, axis=1)).to(torch.bfloat16)
    out = oracle.bits_to_bf16(oracle.combine(deq, L["slot_pos"], b.w)).double()
    x = b.x.double()
    sblk = torch.from_numpy(np.repeat(s[L["slot_pos"][:, 0]], 128, axis=1)).double()
    bound = 2.0 ** -4 * x.abs() + 2.0 ** -10 * sblk + 2.0 ** -7 * x.abs() + 1e-12
    assert torch.all((out - x).abs() <= bound)


def test_combine_weighting_scaled_experts():
    # experts scale by (1 + 0.01 e): out ~ x * sum_j w_j (1 + 0.01 e_j)
    cfg, b, L = _setup("large", 7, 128, 256)
    y = workloads.expert_outputs(b.x, torch.from_numpy(L["recv_src"]),
                                 torch.from_numpy(L["off_e"]), "scale")
    out = oracle.bits_to_bf16(oracle.combine(y, L["slot_pos"], b.w)).double()
    f = (b.w.double() * (1 + 0.01 * b.idx.double())).sum(1, keepdim=True)
    ref = b.x.double() * f
    assert torch.all((out - ref).abs() <= 2.0 ** -6 * ref.abs() + 1e-6)
    # and the factor is not the unweighted mean
    g = (1 + 0.01 * b.idx.double()).mean(1, keepdim=True)
    assert (f - g).abs().max() > 1e-3
