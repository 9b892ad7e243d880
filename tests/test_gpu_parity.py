"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bar: layout (every array), bf16 dispatch, FP8 payload and FP8 scales
bit-exact; combine within 1 bf16 ulp per element (the kernels follow the
same fp32 fma chain, so it is expected to be exact).  Sizes: the five
workloads at full size (the large one checked on sampled tokens and by
properties that hold at any size), plus ragged and degenerate shapes.
All calls use the library's default launch configuration (all SMs), the
one the benchmark times, unless a test varies num_sms on purpose."""
import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads
from _parity import (assert_layout_equal, assert_scales_equal, bf16_ulp_dist, gpu_layout,
                     nan_inf_batch, tensor_bits16, tensor_bytes)

pytestmark = pytest.mark.gpu

CANARY16 = -23131   # 0xA5A5 as int16
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


# ------------------------------------------------------------------ layout

@pytest.mark.parametrize("name", list(workloads.CONFIGS))
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_layout_full_size(name, seed):
    cfg, b = _batch(name, seed, H=8)
    _, g = gpu_layout(b.idx, cfg.E, cfg.R)
    assert_layout_equal(g, oracle.layout(b.idx, cfg.E, cfg.R))


@pytest.mark.parametrize("T", [0, 1, 3, 31, 127, 512, 513, 2047, 4097, 8191, 8192, 9999,
                               32769, 65536, 65537, 70001])
@pytest.mark.parametrize("int32_ids", [False, True])
def test_layout_ragged_and_both_id_types(T, int32_ids):
    # k = 8: up to T = 256 one CTA, then a cluster of up to 16 CTAs (512 or
    # 1024 threads) up to 65535 slots (T = 8191); from T = 8192 (65536
    # slots) one CTA per SM with grid barriers; T*k = 2^19 (T = 65536) is
    # the largest such case, 65537 the first tiled one
    cfg, b = _batch("prefill", 3, T=T, H=8, drop_frac=0.1, dup_frac=0.1)
    _, g = gpu_layout(b.idx, cfg.E, cfg.R, int32_ids=int32_ids)
    assert_layout_equal(g, oracle.layout(b.idx, cfg.E, cfg.R))


@pytest.mark.parametrize("T,k,E,R", [(500, 1, 1, 1), (300, 32, 64, 64),
                                     (2500, 32, 1024, 64), (4000, 4, 1024, 1),
                                     (100000, 2, 16, 16), (300000, 2, 16, 16),
                                     (20000, 32, 1024, 64), (9000, 8, 1024, 64),
                                     (70000, 1, 2, 2)])
def test_layout_extreme_shapes(T, k, E, R):
    # (9000, 8, 1024, 64): a grid-path size whose count matrix would exceed
    # 256 KiB, so the cluster kernel runs; (70000, 1, 2, 2): the grid path
    # with a 4-column count matrix and a single slot per token
    rng = np.random.default_rng(T + k + E)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k] if E <= 64 else \
        np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    idx = torch.from_numpy(idx.astype(np.int64))
    _, g = gpu_layout(idx, E, R)
    assert_layout_equal(g, oracle.layout(idx, E, R))


def test_layout_skewed_hot_expert_and_all_dropped():
    T, k, E, R = 6000, 8, 256, 8
    idx = torch.full((T, k), -1, dtype=torch.int64)
    idx[:, 0] = 7                     # every token picks expert 7
    idx[::3, 1] = 200
    _, g = gpu_layout(idx, E, R)
    assert_layout_equal(g, oracle.layout(idx, E, R))
    idx = torch.full((T, k), -1, dtype=torch.int64)
    _, g = gpu_layout(idx, E, R)
    assert_layout_equal(g, oracle.layout(idx, E, R))


@pytest.mark.parametrize("T", [100, 5000])
def test_layout_bad_ids_reported_and_dropped(T):
    cfg, b = _batch("decode", 4, T=T, H=8)
    idx = b.idx.clone()
    idx[T // 2, 3] = 256              # == E: out of range
    idx[T - 1, 0] = -7
    _, g = gpu_layout(idx, cfg.E, cfg.R)
    ref = oracle.layout(idx, cfg.E, cfg.R)
    assert ref["status"] == ep.EP_ERR_INDEX
    assert_layout_equal(g, ref)


def test_layout_workspace_reused_across_calls():
    # tiled path: the ticket in the workspace resets itself, so one zeroed
    # buffer serves many calls in stream order
    cfg = workloads.CONFIGS["large"]
    T = 70000
    ws = torch.zeros(ep.ep_layout_workspace_bytes(T, cfg.k, cfg.E, cfg.R),
                     dtype=torch.uint8, device="cuda")
    assert ws.numel() > 0
    for seed in range(3):
        b = workloads.make_batch(cfg, seed, T=T, H=8)
        L = ep.ep_get_layout(b.idx.cuda(), cfg.E, cfg.R, ws=ws)
        ref = oracle.layout(b.idx, cfg.E, cfg.R)
        np.testing.assert_array_equal(L.slot_pos.cpu().numpy(), ref["slot_pos"])
        np.testing.assert_array_equal(L.off_e.cpu().numpy(), ref["off_e"])
    assert int(ws[:4].view(torch.int32).item()) == 0   # ticket back at 0


def test_layout_grid_workspace_reused_across_calls():
    # grid path (one CTA per SM, 65536 <= T*k <= 2^19): the barrier counters
    # in the workspace go back to zero, so one zeroed buffer serves many
    # calls in stream order
    cfg = workloads.CONFIGS["large"]
    ws = torch.zeros(ep.ep_layout_workspace_bytes(cfg.T, cfg.k, cfg.E, cfg.R),
                     dtype=torch.uint8, device="cuda")
    assert ws.numel() > 0
    for seed, T in ((0, cfg.T), (1, 9000), (2, 20000)):
        assert 65536 <= T * cfg.k <= 1 << 19
        b = workloads.make_batch(cfg, seed, T=T, H=8, drop_frac=0.05, dup_frac=0.05)
        d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
        L = ep.ep_get_layout(b.idx.cuda(), cfg.E, cfg.R, ws=ws, d_err=d_err)
        host = {key: getattr(L, key).cpu().numpy() for key in
                ("cnt_e", "cnt_r", "in_rank", "off_e", "off_r", "slot_pos", "recv_src")}
        host["status"] = ep.ep_read_error(d_err)
        assert_layout_equal(host, oracle.layout(b.idx, cfg.E, cfg.R))
        assert not ws[:12].view(torch.int32).any()    # counters back at 0


# ---------------------------------------------------------------- dispatch

def _dispatch_bf16_check(cfg, b, num_sms=0):
    T, H, k = b.T, b.H, cfg.k
    L, g = gpu_layout(b.idx, cfg.E, cfg.R)
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    assert_layout_equal(g, ref)
    recv = torch.full((T * k, H), CANARY16, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    ep.ep_dispatch(b.x.cuda(), L.slot_pos, recv=recv, num_sms=num_sms)
    want = oracle.dispatch_bf16(b.x, ref["slot_pos"], T * k,
                                np.full((T * k, H), 0xA5A5, np.uint16))
    np.testing.assert_array_equal(tensor_bits16(recv), want)


@pytest.mark.parametrize("name", ["tiny", "prefill"])
@pytest.mark.parametrize("seed", [0, 1])
def test_dispatch_bf16_full_size(name, seed):
    cfg, b = _batch(name, seed)
    _dispatch_bf16_check(cfg, b)


@pytest.mark.parametrize("H", [8, 136, 256, 504, 520, 7168, 7176])
def test_dispatch_bf16_ragged_hidden(H):
    cfg, b = _batch("prefill", 5, T=333, H=H, drop_frac=0.1, dup_frac=0.2)
    _dispatch_bf16_check(cfg, b)


@pytest.mark.parametrize("num_sms", [1, 7, 148])
def test_dispatch_bf16_sm_budget(num_sms):
    cfg, b = _batch("prefill", 6, T=700)
    _dispatch_bf16_check(cfg, b, num_sms=num_sms)


def test_dispatch_bf16_large_by_property():
    # full-size large workload: every filled row equals its source token's
    # row (recv_src from the bit-exact layout), unfilled rows untouched
    cfg, b = _batch("large", 0)
    T, H, k = b.T, b.H, cfg.k
    L, g = gpu_layout(b.idx, cfg.E, cfg.R)
    assert_layout_equal(g, oracle.layout(b.idx, cfg.E, cfg.R))
    x = b.x.cuda()
    recv = ep.ep_dispatch(x, L.slot_pos)
    n = int(L.off_e[-1].item())
    src = L.recv_src[:n].long()
    assert torch.equal(recv[:n].view(torch.int16), x[src].view(torch.int16))
    # and a sampled slice against the oracle itself (compact rows)
    sample = torch.from_numpy(np.random.default_rng(0).choice(T, 256, replace=False))
    sp = L.slot_pos[sample.cuda()].cpu().numpy()
    local = np.arange(sp.size, dtype=np.int32).reshape(sp.shape)
    local[sp < 0] = -1
    want = oracle.dispatch_bf16(b.x[sample], local, sp.size)
    keep = sp.reshape(-1) >= 0
    got = tensor_bits16(recv[torch.from_numpy(sp.reshape(-1)[keep]).long().cuda()])
    np.testing.assert_array_equal(got, want[keep])


def _dispatch_fp8_check(cfg, b, num_sms=0):
    T, H, k = b.T, b.H, cfg.k
    L, g = gpu_layout(b.idx, cfg.E, cfg.R)
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    assert_layout_equal(g, ref)
    q = torch.full((T * k, H), CANARY8, dtype=torch.uint8, device="cuda")
    s = torch.full((T * k, H // 128), -1.0, dtype=torch.float32, device="cuda")
    ep.ep_dispatch(b.x.cuda(), L.slot_pos, fp8=True, recv=q, recv_scale=s,
                   num_sms=num_sms)
    wq, ws_ = oracle.dispatch_fp8(b.x, ref["slot_pos"], T * k,
                                  np.full((T * k, H), CANARY8, np.uint8),
                                  np.full((T * k, H // 128), -1.0, np.float32))
    np.testing.assert_array_equal(tensor_bytes(q), wq)
    assert_scales_equal(s.cpu().numpy(), ws_)


@pytest.mark.parametrize("name", ["decode", "prefill", "skewed"])
def test_dispatch_fp8_full_size(name):
    cfg, b = _batch(name, 0)
    _dispatch_fp8_check(cfg, b)


@pytest.mark.parametrize("H", [128, 256, 384, 512, 640, 896, 1536, 4096, 7168, 7296, 16384])
def test_dispatch_fp8_ragged_hidden(H):
    # H % 512 == 0 (up to 16384) takes the shared-memory bulk-copy kernel,
    # other multiples of 128 the register kernel
    cfg, b = _batch("decode", 7, T=77, H=H, drop_frac=0.1)
    _dispatch_fp8_check(cfg, b)


def test_dispatch_fp8_misaligned_scales_use_register_path():
    # scale rows 4-byte (not 16-byte) aligned: bulk stores are not allowed
    cfg, b = _batch("decode", 13, T=50, H=1024)
    T, H, k = b.T, b.H, cfg.k
    L, g = gpu_layout(b.idx, cfg.E, cfg.R)
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    q = torch.full((T * k, H), CANARY8, dtype=torch.uint8, device="cuda")
    s_buf = torch.full((T * k * (H // 128) + 1,), -1.0, dtype=torch.float32, device="cuda")
    s = s_buf[1:].view(T * k, H // 128)             # offset by 4 bytes
    ep.ep_dispatch(b.x.cuda(), L.slot_pos, fp8=True, recv=q, recv_scale=s)
    wq, ws_ = oracle.dispatch_fp8(b.x, ref["slot_pos"], T * k)
    np.testing.assert_array_equal(tensor_bytes(q), wq)
    assert_scales_equal(s.cpu().numpy(), ws_)


def test_dispatch_fp8_special_values():
    # zero blocks (clamped scale), tiny blocks, huge values, negative zero,
    # values whose quotient lands on e4m3 ties
    cfg = workloads.CONFIGS["decode"]
    b = workloads.make_batch(cfg, 8, T=64, H=1024)
    x = b.x.float()
    x[0] = 0.0
    x[1, :128] = 1e-30
    x[2, 128:256] = 3.0e38
    x[3] = -0.0
    x[4, :128] = torch.arange(128) * (3.5 / 127)
    x[5, 256:384] = torch.tensor([17.0, 19.0, 9.5, -448.0] * 32) / 128.0
    b.x = x.to(torch.bfloat16)
    _dispatch_fp8_check(cfg, b)


@pytest.mark.parametrize("H", [1024, 896, 7168])
def test_dispatch_fp8_nan_and_inf(H):
    # H = 1024 and 7168 fill whole 512-channel groups (one 16-byte scale
    # store per group and row); H = 896 ends in a partial group
    cfg = workloads.CONFIGS["decode"]
    b = nan_inf_batch(cfg, 21, 16, H)
    _dispatch_fp8_check(cfg, b)


@pytest.mark.parametrize("num_sms", [1, 13])
def test_dispatch_fp8_sm_budget(num_sms):
    cfg, b = _batch("skewed", 9, T=500, H=1024)
    _dispatch_fp8_check(cfg, b, num_sms=num_sms)


# ----------------------------------------------------------------- combine

def _combine_check(cfg, b, sample=None, num_sms=0):
    T, H, k = b.T, b.H, cfg.k
    L, g = gpu_layout(b.idx, cfg.E, cfg.R)
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    assert_layout_equal(g, ref)
    y = workloads.expert_outputs(b.x, torch.from_numpy(ref["recv_src"]),
                                 torch.from_numpy(ref["off_e"]), cfg.expert)
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ep.ep_combine(y.cuda(), L.slot_pos, b.w.cuda(), num_sms=num_sms, d_err=d_err)
    assert ep.ep_read_error(d_err) == 0
    got = tensor_bits16(out)
    if sample is None:
        want = oracle.combine(y, ref["slot_pos"], b.w)
    else:
        # the oracle on the sampled tokens, over just the rows they use
        sp = ref["slot_pos"][sample]
        rows = np.unique(sp[sp >= 0])
        remap = np.full(T * k, -1, np.int32)
        remap[rows] = np.arange(rows.size, dtype=np.int32)
        sp_local = np.where(sp >= 0, remap[np.maximum(sp, 0)], -1).astype(np.int32)
        want = oracle.combine(y[torch.from_numpy(rows).long()], sp_local,
                              b.w[torch.from_numpy(sample)])
        got = got[sample]
    d = bf16_ulp_dist(got, want)
    assert d.max() <= 1, f"max ulp {d.max()}"
    return float((d == 0).mean())


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skewed"])
def test_combine_full_size(name):
    cfg, b = _batch(name, 0)
    exact = _combine_check(cfg, b)
    assert exact == 1.0          # same fp32 fma chain as the oracle


def test_combine_large_sampled():
    cfg, b = _batch("large", 1)
    sample = np.sort(np.random.default_rng(1).choice(b.T, 2048, replace=False))
    assert _combine_check(cfg, b, sample=sample) == 1.0


@pytest.mark.parametrize("H", [8, 136, 256, 264, 7176])
def test_combine_ragged_hidden_and_drops(H):
    cfg, b = _batch("large", 2, T=211, H=H, drop_frac=0.3, dup_frac=0.2)
    assert _combine_check(cfg, b) == 1.0


# under a budget the register kernel runs while its items fit one wave on
# the budgeted SMs (T = 16 on 29 SMs), the bulk-copy pipeline above that
@pytest.mark.parametrize("T,num_sms", [(300, 1), (300, 29), (16, 29)])
def test_combine_sm_budget(T, num_sms):
    cfg, b = _batch("prefill", 3, T=T)
    assert _combine_check(cfg, b, num_sms=num_sms) == 1.0


@pytest.mark.parametrize("num_sms", [0, 9])
def test_combine_subnormal_values(num_sms):
    # expert outputs that are bf16 subnormals and tiny normals, weights
    # below 1: the fp32 chain and the final bf16 rounding run through
    # subnormals and must match the oracle bit for bit
    rng = np.random.default_rng(78)
    T, k, H = 96, 8, 1024
    n = T * k
    mag = rng.integers(1, 0x0100, size=(n, H)).astype(np.uint16)   # exponent 0 or 1
    sign = (rng.random((n, H)) < 0.5).astype(np.uint16) << 15
    y = torch.from_numpy((mag | sign).view(np.int16)).view(torch.bfloat16)
    slot = rng.permutation(n).astype(np.int32).reshape(T, k)
    w = (rng.random((T, k)) * 0.9).astype(np.float32)
    out = ep.ep_combine(y.cuda(), torch.from_numpy(slot).cuda(), torch.from_numpy(w).cuda(),
                        num_sms=num_sms)
    want = oracle.combine(y, slot, torch.from_numpy(w))
    assert (want & 0x7F80 == 0).any()
    np.testing.assert_array_equal(tensor_bits16(out), want)


def test_combine_k32_and_k1():
    for k, E in ((32, 64), (1, 4)):
        cfg = workloads.Config("k", 200, 512, E, 4, k, "uniform", ("bf16",), "scale")
        b = workloads.make_batch(cfg, 11)
        assert _combine_check(cfg, b) == 1.0


def test_round_trip_identity_experts():
    # combine(dispatch(x)) with identity experts and weights summing to 1
    # returns x to within one bf16 ulp
    cfg, b = _batch("prefill", 12, T=1024)
    x = b.x.cuda()
    L = ep.ep_get_layout(b.idx.cuda(), cfg.E, cfg.R)
    recv = ep.ep_dispatch(x, L.slot_pos)
    out = ep.ep_combine(recv, L.slot_pos, b.w.cuda())
    d = bf16_ulp_dist(tensor_bits16(out), tensor_bits16(x))
    assert d.max() <= 1


def test_empty_batch_calls():
    cfg = workloads.CONFIGS["tiny"]
    idx = torch.empty((0, cfg.k), dtype=torch.int64, device="cuda")
    L = ep.ep_get_layout(idx, cfg.E, cfg.R)
    assert int(L.off_e[-1]) == 0 and int(L.cnt_e.sum()) == 0
    x = torch.empty((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    recv = ep.ep_dispatch(x, L.slot_pos)
    assert recv.shape == (0, cfg.H)
    out = ep.ep_combine(recv, L.slot_pos, torch.empty((0, cfg.k), device="cuda"))
    assert out.shape == (0, cfg.H)
    torch.cuda.synchronize()


def test_kernel_launch_counter_advances():
    before = ep.ep_kernel_launches()
    cfg, b = _batch("tiny", 0)
    L = ep.ep_get_layout(b.idx.cuda(), cfg.E, cfg.R)
    ep.ep_combine(ep.ep_dispatch(b.x.cuda(), L.slot_pos), L.slot_pos, b.w.cuda())
    torch.cuda.synchronize()
    assert ep.ep_kernel_launches() - before == 3
