"""GPU parity of ep_layout_dispatch (layout and dispatch in one launch for
small batches) against the CPU oracle: every layout array, the bf16 rows,
the FP8 payload and the FP8 scales bit-exact, on the decode and tiny
workloads at full size and on ragged token counts, both id types,
duplicated and dropped slots, bad ids, the largest fused shapes and the
sizes that fall back to the two-kernel path.  Every output buffer starts
filled with a canary so an entry the kernel forgets to write shows up."""
import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads
from _parity import (LAYOUT_KEYS, assert_layout_equal, assert_scales_equal,
                     nan_inf_batch, tensor_bits16, tensor_bytes)

pytestmark = pytest.mark.gpu

CANARY32 = 0x5A5A5A5A
CANARY16 = -23131   # 0xA5A5 as int16
CANARY8 = 0x5A


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ep.lib()
    yield
    torch.cuda.empty_cache()


def _canary_layout(T, k, E, R):
    L = ep.empty_layout(T, k, E, R, "cuda")
    return ep.Layout(*[t.fill_(CANARY8 if t.dtype == torch.uint8 else CANARY32) for t in L])


def _run(idx, x, E, R, fp8, *, int32_ids=False, num_sms=0, scale_offset=0):
    """One ep_layout_dispatch call; returns host copies and the number of
    kernels it launched."""
    T, k = idx.shape
    H = x.shape[1]
    dev = torch.device("cuda")
    idx_d = idx.to(torch.int32 if int32_ids else torch.int64).to(dev)
    x_d = x.to(dev)
    out = _canary_layout(T, k, E, R)
    d_err = torch.zeros(1, dtype=torch.int32, device=dev)
    if fp8:
        recv = torch.full((T * k, H), CANARY8, dtype=torch.uint8, device=dev)
        s_buf = torch.full((T * k * (H // 128) + scale_offset,), -1.0,
                           dtype=torch.float32, device=dev)
        scale = s_buf[scale_offset:].view(T * k, H // 128)
    else:
        recv = torch.full((T * k, H), CANARY16, dtype=torch.int16, device=dev)
        scale = None
    before = ep.ep_kernel_launches()
    L, _ = ep.ep_layout_dispatch(
        idx_d, E, R, x_d, fp8, out=out,
        recv=recv.view(torch.float8_e4m3fn) if fp8 else recv.view(torch.bfloat16),
        recv_scale=scale, num_sms=num_sms, d_err=d_err)
    launches = ep.ep_kernel_launches() - before
    host = {key: getattr(L, key).cpu().numpy() for key in LAYOUT_KEYS}
    host["status"] = ep.ep_read_error(d_err)
    got = {"recv": tensor_bytes(recv) if fp8 else tensor_bits16(recv)}
    if fp8:
        got["scale"] = scale.cpu().numpy().view(np.uint32)
    return host, got, launches


def _check(idx, x, E, R, fp8, **kw):
    T, k = idx.shape
    H = x.shape[1]
    host, got, launches = _run(idx, x, E, R, fp8, **kw)
    ref = oracle.layout(idx, E, R)
    assert_layout_equal(host, ref)
    if fp8:
        wq, ws_ = oracle.dispatch_fp8(x, ref["slot_pos"], T * k,
                                      np.full((T * k, H), CANARY8, np.uint8),
                                      np.full((T * k, H // 128), -1.0, np.float32))
        np.testing.assert_array_equal(got["recv"], wq)
        assert_scales_equal(got["scale"].view(np.float32), ws_)
    else:
        want = oracle.dispatch_bf16(x, ref["slot_pos"], T * k,
                                    np.full((T * k, H), 0xA5A5, np.uint16))
        np.testing.assert_array_equal(got["recv"], want)
    return launches


def _batch(name, seed=0, **kw):
    cfg = workloads.CONFIGS[name]
    return cfg, workloads.make_batch(cfg, seed, **kw)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_fp8_full_size_one_launch(seed):
    cfg, b = _batch("decode", seed)
    assert _check(b.idx, b.x, cfg.E, cfg.R, True) == 1


@pytest.mark.parametrize("name,fp8", [("tiny", False), ("decode", False)])
def test_bf16_full_size_one_launch(name, fp8):
    cfg, b = _batch(name, 0)
    assert _check(b.idx, b.x, cfg.E, cfg.R, fp8) == 1


@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 127, 129, 300, 1000, 1024])
@pytest.mark.parametrize("fp8", [False, True])
def test_ragged_tokens_with_drops_and_duplicates(T, fp8):
    # dup_frac: slot 1 repeats slot 0's expert (two slots of one expert in
    # one token), which switches the kernel to counting ranks over slots
    cfg, b = _batch("decode", 11, T=T, H=512, drop_frac=0.1, dup_frac=0.05 if T > 2 else 0.0)
    assert _check(b.idx, b.x, cfg.E, cfg.R, fp8) == 1


@pytest.mark.parametrize("fp8", [False, True])
def test_int32_ids(fp8):
    cfg, b = _batch("decode", 12, T=200, H=1024, drop_frac=0.05)
    assert _check(b.idx, b.x, cfg.E, cfg.R, fp8, int32_ids=True) == 1


def test_every_token_duplicated():
    cfg, b = _batch("decode", 13, T=100, H=512, dup_frac=1.0)
    assert _check(b.idx, b.x, cfg.E, cfg.R, True) == 1


def test_all_slots_dropped():
    cfg, b = _batch("decode", 14, T=64, H=512)
    idx = torch.full_like(b.idx, -1)
    assert _check(idx, b.x, cfg.E, cfg.R, True) == 1


@pytest.mark.parametrize("T,k,E,R", [
    (256, 32, 1024, 64),   # T*k = 8192 slots, the largest fused batch; 64 ranks
    (128, 8, 1024, 64),    # mask 1024 experts x 4 words
    (1024, 8, 256, 8),     # mask 256 x 32 words = 32 KiB, the largest
    (300, 1, 1, 1),        # one expert, one rank
    (500, 16, 16, 16),     # one expert per rank
])
def test_extreme_fused_shapes(T, k, E, R):
    rng = np.random.default_rng(T * 7 + k + E)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int64)
    x = torch.from_numpy(rng.standard_normal((T, 512)).astype(np.float32)).to(torch.bfloat16)
    assert _check(torch.from_numpy(idx), x, E, R, True) == 1
    assert _check(torch.from_numpy(idx), x, E, R, False) == 1


def test_bad_ids_reported_and_dropped():
    cfg, b = _batch("decode", 15, T=128, H=512)
    idx = b.idx.clone()
    idx[64, 3] = 256          # == E: out of range
    idx[127, 0] = -7
    idx[0, 7] = 1 << 40       # int64 only
    host, _, _ = _run(idx, b.x, cfg.E, cfg.R, True)
    assert host["status"] == ep.EP_ERR_INDEX
    assert _check(idx, b.x, cfg.E, cfg.R, True) == 1


@pytest.mark.parametrize("num_sms", [0, 1, 2])
@pytest.mark.parametrize("fp8", [False, True])
def test_both_fused_kernels_on_the_decode_shape(num_sms, fp8):
    # all SMs: one token per CTA (T + 1 CTAs fit at once); one or two SMs:
    # the token-range kernel, each CTA walking many tokens through its
    # two-stage row pipeline -- with dropped, duplicated and bad ids
    cfg, b = _batch("decode", 22, drop_frac=0.05, dup_frac=0.1)
    idx = b.idx.clone()
    idx[5, 2] = 999
    host, _, _ = _run(idx, b.x, cfg.E, cfg.R, fp8, num_sms=num_sms)
    assert host["status"] == ep.EP_ERR_INDEX
    assert _check(idx, b.x, cfg.E, cfg.R, fp8, num_sms=num_sms) == 1


@pytest.mark.parametrize("H,fused", [(8, True), (136, True), (7176, True), (16384, True),
                                     (16392, False)])
def test_bf16_hidden_sizes(H, fused):
    cfg, b = _batch("decode", 16, T=60, H=H, drop_frac=0.1)
    assert _check(b.idx, b.x, cfg.E, cfg.R, False) == (1 if fused else 2)


@pytest.mark.parametrize("H,fused", [(128, False), (384, False), (512, True), (1536, True),
                                     (16384, True), (7296, False)])
def test_fp8_hidden_sizes(H, fused):
    # the fused kernel stores whole scale rows with bulk copies: H % 512 == 0
    cfg, b = _batch("decode", 17, T=60, H=H, drop_frac=0.1)
    assert _check(b.idx, b.x, cfg.E, cfg.R, True) == (1 if fused else 2)


def test_misaligned_scales_take_two_kernels():
    cfg, b = _batch("decode", 18, T=50, H=1024)
    assert _check(b.idx, b.x, cfg.E, cfg.R, True, scale_offset=1) == 2


@pytest.mark.parametrize("num_sms", [0, 1])
def test_fp8_nan_and_inf(num_sms):
    # all SMs: the one-token-per-CTA kernel; one SM: the token-range kernel
    cfg = workloads.CONFIGS["decode"]
    b = nan_inf_batch(cfg, 23, 40, 1024)
    assert _check(b.idx, b.x, cfg.E, cfg.R, True, num_sms=num_sms) == 1


@pytest.mark.parametrize("num_sms", [1, 7, 148])
def test_sm_budget(num_sms):
    # fewer CTAs than tokens: each CTA walks several tokens through the
    # two-stage row pipeline
    cfg, b = _batch("decode", 19, T=700, H=1024, drop_frac=0.05, dup_frac=0.05)
    assert _check(b.idx, b.x, cfg.E, cfg.R, True, num_sms=num_sms) == 1
    assert _check(b.idx, b.x, cfg.E, cfg.R, False, num_sms=num_sms) == 1


@pytest.mark.parametrize("T", [1025, 4096])
def test_large_batches_take_two_kernels(T):
    cfg, b = _batch("prefill", 20, T=T, H=512)
    assert _check(b.idx, b.x, cfg.E, cfg.R, True) == 2


def test_matches_separate_calls_and_combines():
    # the decode step end to end: fused layout + FP8 dispatch, then combine
    # of the dequantised rows, against the unfused calls on the same inputs
    cfg, b = _batch("decode", 21)
    idx, x, w = b.idx.cuda(), b.x.cuda(), b.w.cuda()
    L1, (q1, s1) = ep.ep_layout_dispatch(idx, cfg.E, cfg.R, x, True)
    L2 = ep.ep_get_layout(idx, cfg.E, cfg.R)
    q2, s2 = ep.ep_dispatch(x, L2.slot_pos, fp8=True)
    for key in LAYOUT_KEYS:
        assert torch.equal(getattr(L1, key), getattr(L2, key)), key
    assert torch.equal(q1.view(torch.uint8), q2.view(torch.uint8))
    assert torch.equal(s1, s2)
    y = (q1.float().view(q1.shape[0], -1, 128) * s1.unsqueeze(-1)).view(q1.shape)
    y = y.to(torch.bfloat16)
    out = ep.ep_combine(y, L1.slot_pos, w)
    want = oracle.combine(y.cpu(), L1.slot_pos.cpu().numpy(), b.w)
    np.testing.assert_array_equal(tensor_bits16(out), want)


def test_empty_batch():
    dev = torch.device("cuda")
    idx = torch.empty((0, 8), dtype=torch.int64, device=dev)
    x = torch.empty((0, 512), dtype=torch.bfloat16, device=dev)
    L, (q, s) = ep.ep_layout_dispatch(idx, 256, 8, x, True)
    torch.cuda.synchronize()
    assert int(L.off_e[-1]) == 0 and int(L.off_r[-1]) == 0
    assert L.cnt_e.abs().sum().item() == 0 and q.numel() == 0 and s.numel() == 0
