"""GPU parity of the combine variants against the CPU oracle: the aligned
layout (expert segments padded for a grouped GEMM), dispatch into and
combine from the padded receive buffer, and the FP8 expert-output combine.
Layout arrays, bf16 rows and FP8 bytes bit-exact; the combines follow the
oracle's fp32 chain, so they are compared bit for bit as well (the bar is
1 bf16 ulp)."""
import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads
from _parity import tensor_bits16, tensor_bytes

pytestmark = pytest.mark.gpu

CANARY32 = 0x5A5A5A5A
CANARY16 = -23131
CANARY8 = 0x5A


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ep.lib()
    yield
    torch.cuda.empty_cache()


def _batch(name, seed=0, **kw):
    cfg = workloads.CONFIGS[name]
    return cfg, workloads.make_batch(cfg, seed, **kw)


def _padded(idx, E, R, align, in_place=False):
    L = ep.ep_get_layout(idx.cuda(), E, R)
    T, k = idx.shape
    cap = ep.ep_aligned_rows(T, k, E, align)
    out = ep.PaddedLayout(torch.full((E + 1,), CANARY32, dtype=torch.int32, device="cuda"),
                          L.slot_pos if in_place else
                          torch.full((T, k), CANARY32, dtype=torch.int32, device="cuda"),
                          torch.full((max(cap, 1),), CANARY32, dtype=torch.int32, device="cuda"))
    P = ep.ep_pad_layout(L, align, out=out)
    return P, cap


def _assert_padded(P, cap, ref):
    np.testing.assert_array_equal(P.off_pad.cpu().numpy(), ref["off_pad"])
    np.testing.assert_array_equal(P.slot_pos.cpu().numpy(), ref["slot_pos"])
    np.testing.assert_array_equal(P.recv_src[:cap].cpu().numpy(), ref["recv_src"])


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skewed"])
@pytest.mark.parametrize("align", [1, 8, 128])
def test_pad_layout_full_size(name, align):
    cfg, b = _batch(name, 1, H=8)
    P, cap = _padded(b.idx, cfg.E, cfg.R, align)
    _assert_padded(P, cap, oracle.layout_aligned(b.idx, cfg.E, align))


@pytest.mark.parametrize("T", [0, 1, 77, 1000, 70001])
@pytest.mark.parametrize("align", [3, 64])
def test_pad_layout_ragged_drops_duplicates_in_place(T, align):
    cfg, b = _batch("prefill", 2, T=T, H=8, drop_frac=0.1, dup_frac=0.1)
    P, cap = _padded(b.idx, cfg.E, cfg.R, align, in_place=True)
    _assert_padded(P, cap, oracle.layout_aligned(b.idx, cfg.E, align))


def test_pad_layout_empty_experts_and_one_hot_expert():
    T, k, E, R = 3000, 4, 1024, 64
    idx = torch.full((T, k), -1, dtype=torch.int64)
    idx[:, 0] = 513
    idx[::7, 1] = 0
    idx[::5, 2] = 1023
    P, cap = _padded(idx, E, R, 128)
    _assert_padded(P, cap, oracle.layout_aligned(idx, E, 128))


@pytest.mark.parametrize("fp8", [False, True])
def test_dispatch_and_combine_through_padded_buffer(fp8):
    # layout -> pad -> dispatch into the aligned buffer -> identity experts
    # -> combine (bf16) from it, against the oracle's aligned chain
    cfg, b = _batch("prefill", 3, T=600, H=1024, drop_frac=0.05)
    align = 128
    T, H, k = b.T, b.H, cfg.k
    P, cap = _padded(b.idx, cfg.E, cfg.R, align)
    ref = oracle.layout_aligned(b.idx, cfg.E, align)
    x = b.x.cuda()
    if fp8:
        q = torch.full((cap, H), CANARY8, dtype=torch.uint8, device="cuda")
        s = torch.full((cap, H // 128), -1.0, dtype=torch.float32, device="cuda")
        ep.ep_dispatch(x, P.slot_pos, fp8=True, recv=q.view(torch.float8_e4m3fn), recv_scale=s)
        wq, ws_ = oracle.dispatch_fp8(b.x, ref["slot_pos"], cap,
                                      np.full((cap, H), CANARY8, np.uint8),
                                      np.full((cap, H // 128), -1.0, np.float32))
        np.testing.assert_array_equal(tensor_bytes(q), wq)
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), ws_.view(np.uint32))
        out = ep.ep_combine_fp8(q.view(torch.float8_e4m3fn), s, P.slot_pos, b.w.cuda())
        want = oracle.combine_fp8(wq, ws_, ref["slot_pos"], b.w)
    else:
        recv = torch.full((cap, H), CANARY16, dtype=torch.int16, device="cuda")
        ep.ep_dispatch(x, P.slot_pos, recv=recv.view(torch.bfloat16))
        want_recv = oracle.dispatch_bf16(b.x, ref["slot_pos"], cap,
                                         np.full((cap, H), 0xA5A5, np.uint16))
        np.testing.assert_array_equal(tensor_bits16(recv), want_recv)
        # padding rows hold canaries; combine never reads them
        out = ep.ep_combine(recv.view(torch.bfloat16), P.slot_pos, b.w.cuda())
        want = oracle.combine(torch.from_numpy(want_recv.view(np.int16)).view(torch.bfloat16),
                              ref["slot_pos"], b.w)
    np.testing.assert_array_equal(tensor_bits16(out), want)


# ---------------------------------------------------------- FP8 combine

def _fp8_expert_rows(rng, n, H):
    q = rng.integers(0, 256, (n, H), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x3C            # no NaN codes
    s = (rng.random((n, H // 128)) * 0.05 + 1e-3).astype(np.float32)
    return q, s


def _combine_fp8_check(T, H, k, seed, drop=0.0, w_none=False, scale_offset=0, num_sms=0,
                       extra_rows=0):
    rng = np.random.default_rng(seed)
    n = T * k + extra_rows
    q, s = _fp8_expert_rows(rng, n, H)
    slot = rng.permutation(n)[:T * k].astype(np.int32).reshape(T, k) if T * k else \
        np.zeros((T, k), np.int32)
    slot[rng.random(slot.shape) < drop] = -1
    w = None if w_none else rng.random((T, k)).astype(np.float32)
    s_buf = torch.full((n * (H // 128) + scale_offset,), -1.0, dtype=torch.float32, device="cuda")
    s_d = s_buf[scale_offset:].view(n, H // 128)
    s_d.copy_(torch.from_numpy(s))
    out = ep.ep_combine_fp8(torch.from_numpy(q).cuda().view(torch.float8_e4m3fn), s_d,
                            torch.from_numpy(slot).cuda(),
                            None if w is None else torch.from_numpy(w).cuda(), num_sms=num_sms)
    want = oracle.combine_fp8(q, s, slot, w)
    np.testing.assert_array_equal(tensor_bits16(out), want)


def test_combine_fp8_prefill_full_size():
    _combine_fp8_check(4096, 7168, 8, 0)


def test_combine_fp8_decode_full_size():
    _combine_fp8_check(128, 7168, 8, 1)


@pytest.mark.parametrize("num_sms", [0, 9])
@pytest.mark.parametrize("H", [128, 384, 512, 1536, 4096, 7296, 16384])
def test_combine_fp8_ragged_hidden_and_drops(H, num_sms):
    # all SMs: the item kernel at every H; under an SM budget H % 512 == 0
    # takes the bulk-copy kernel, other multiples of 128 the register kernel
    _combine_fp8_check(97, H, 8, H, drop=0.1, num_sms=num_sms)


@pytest.mark.parametrize("k", [1, 3, 16, 32])
def test_combine_fp8_k(k):
    _combine_fp8_check(50, 1024, k, k, drop=0.05)


def test_combine_fp8_unit_weights_extra_rows_misaligned_scales():
    _combine_fp8_check(200, 2048, 8, 5, w_none=True, extra_rows=300)
    _combine_fp8_check(200, 2048, 8, 6, scale_offset=1)     # item kernel
    _combine_fp8_check(200, 2048, 8, 6, scale_offset=1, num_sms=9)  # register kernel


@pytest.mark.parametrize("num_sms", [1, 9])
def test_combine_fp8_sm_budget(num_sms):
    _combine_fp8_check(300, 1024, 8, 7, num_sms=num_sms)


def test_combine_fp8_special_codes():
    # zero codes of both signs, the largest codes, subnormal codes
    T, k, H = 8, 2, 512
    n = T * k
    q = np.zeros((n, H), np.uint8)
    q[0] = 0x80
    q[1] = 0x7E
    q[2] = 0xFE
    q[3, :8] = np.arange(8, dtype=np.uint8)
    q[4, :8] = 0x80 | np.arange(8, dtype=np.uint8)
    s = np.full((n, H // 128), 2.0 ** -6, np.float32)
    s[1] = 3.0e38 / 448.0
    slot = np.arange(n, dtype=np.int32).reshape(T, k)
    w = np.full((T, k), 0.75, np.float32)
    out = ep.ep_combine_fp8(torch.from_numpy(q).cuda().view(torch.float8_e4m3fn),
                            torch.from_numpy(s).cuda(), torch.from_numpy(slot).cuda(),
                            torch.from_numpy(w).cuda())
    np.testing.assert_array_equal(tensor_bits16(out), oracle.combine_fp8(q, s, slot, w))


@pytest.mark.parametrize("num_sms", [0, 9])
def test_combine_fp8_subnormal_products(num_sms):
    # scales at and below the fp32 normal range, so that scaled values and
    # the fma chain run through fp32 subnormals: the packed f32x2 multiply
    # and fma must keep them exactly as the oracle's scalar fp32 does
    rng = np.random.default_rng(77)
    T, k, H = 64, 4, 1024
    n = T * k
    q = rng.integers(0, 256, size=(n, H), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x01  # no NaN codes
    choices = np.array([1.1754944e-38, 1e-38, 1e-40, 2.0 ** -140, 1.4e-45, 3e-42],
                       np.float32)
    s = rng.choice(choices, size=(n, H // 128)).astype(np.float32)
    slot = rng.permutation(n).astype(np.int32).reshape(T, k)
    w = rng.random((T, k)).astype(np.float32)
    w[:, 0] = 1.0
    out = ep.ep_combine_fp8(torch.from_numpy(q).cuda().view(torch.float8_e4m3fn),
                            torch.from_numpy(s).cuda(), torch.from_numpy(slot).cuda(),
                            torch.from_numpy(w).cuda(), num_sms=num_sms)
    want = oracle.combine_fp8(q, s, slot, w)
    assert (want & 0x7F80 == 0).any()  # some outputs are bf16 subnormals
    np.testing.assert_array_equal(tensor_bits16(out), want)


# -------------------------------------------------------------- replicas

def _replica_table(rng, E, hot, copies):
    """Logical experts `hot` get `copies` copies each, the rest one; the
    physical ids are a seeded permutation."""
    n_rep = np.ones(E, np.int64)
    n_rep[hot] = copies
    rep_off = np.concatenate([[0], np.cumsum(n_rep)]).astype(np.int32)
    rep_ids = rng.permutation(int(rep_off[-1])).astype(np.int32)
    return rep_off, rep_ids


@pytest.mark.parametrize("int32_ids", [False, True])
def test_replicas_on_the_skewed_workload(int32_ids):
    # the 16 hottest experts of the Zipf routing get 4 copies: 304 physical
    # experts in 8 ranks of 38; logical and physical layouts both bit-exact
    cfg, b = _batch("skewed", 0, H=8)
    E, R = cfg.E, cfg.R
    load = np.bincount(b.idx.numpy().reshape(-1), minlength=E)
    hot = np.argsort(-load, kind="stable")[:16]
    rng = np.random.default_rng(8)
    rep_off, rep_ids = _replica_table(rng, E, hot, 4)
    E_phys = int(rep_off[-1])
    idx = b.idx.to(torch.int32 if int32_ids else torch.int64).cuda()
    L = ep.ep_get_layout(idx, E, R)
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    phys = ep.ep_map_replicas(idx, L, torch.from_numpy(rep_off).cuda(),
                              torch.from_numpy(rep_ids).cuda(), d_err=d_err)
    want, st = oracle.map_replicas(b.idx, rep_off, rep_ids)
    np.testing.assert_array_equal(phys.cpu().numpy(), want)
    assert ep.ep_read_error(d_err) == st == ep.EP_OK
    P = ep.ep_get_layout(phys, E_phys, 8)
    ref = oracle.layout(torch.from_numpy(want.astype(np.int64)), E_phys, 8)
    for key in ("cnt_e", "off_e", "slot_pos", "recv_src", "in_rank", "cnt_r"):
        np.testing.assert_array_equal(getattr(P, key).cpu().numpy().reshape(-1),
                                      ref[key].reshape(-1), err_msg=key)
    assert ref["cnt_e"].max() < load.max()        # the hottest load went down


def test_replicas_drops_duplicates_bad_ids_and_missing_copies():
    cfg, b = _batch("decode", 9, T=500, H=8, drop_frac=0.1, dup_frac=0.2)
    E = cfg.E
    rng = np.random.default_rng(9)
    rep_off, rep_ids = _replica_table(rng, E, np.arange(0, E, 5), 3)
    rep_off = rep_off.copy()
    # expert 3 has no copy: its slots are reported and dropped
    n_rep = np.diff(rep_off)
    n_rep[3] = 0
    rep_off = np.concatenate([[0], np.cumsum(n_rep)]).astype(np.int32)
    rep_ids = rep_ids[:int(rep_off[-1])]
    idx = b.idx.clone()
    idx[7, 2] = 3
    idx[9, 0] = 4096                              # bad id
    L = ep.ep_get_layout(idx.cuda(), E, cfg.R)
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    phys = ep.ep_map_replicas(idx.cuda(), L, torch.from_numpy(rep_off).cuda(),
                              torch.from_numpy(rep_ids).cuda(), d_err=d_err)
    want, st = oracle.map_replicas(idx, rep_off, rep_ids)
    np.testing.assert_array_equal(phys.cpu().numpy(), want)
    assert st == ep.EP_ERR_INDEX and ep.ep_read_error(d_err) == ep.EP_ERR_INDEX
