"""The library's calls are stateless and stream-ordered: calls on two
streams at once, on different batches, give each batch's oracle result; a
CUDA graph of the whole path, replayed after new inputs are copied into its
buffers, gives the new inputs' oracle result (bit-exact)."""
import numpy as np
import pytest
import torch

import combine_ep_get_09_b200 as ep
import oracle
import workloads
from _parity import LAYOUT_KEYS, tensor_bits16, tensor_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ep.lib()
    yield
    torch.cuda.empty_cache()


def _expect(cfg, b):
    ref = oracle.layout(b.idx, cfg.E, cfg.R)
    n = b.T * cfg.k
    recv = oracle.dispatch_bf16(b.x, ref["slot_pos"], n)
    q, s = oracle.dispatch_fp8(b.x, ref["slot_pos"], n)
    out = oracle.combine(recv, ref["slot_pos"], b.w)
    return ref, recv, q, s, out


class Path:
    """Device buffers and the calls of one pass (layout, both dispatches,
    combine) on a given stream."""

    def __init__(self, cfg, T, H):
        dev = torch.device("cuda")
        k = cfg.k
        self.cfg = cfg
        self.idx = torch.zeros((T, k), dtype=torch.int64, device=dev)
        self.x = torch.zeros((T, H), dtype=torch.bfloat16, device=dev)
        self.w = torch.zeros((T, k), dtype=torch.float32, device=dev)
        self.L = ep.empty_layout(T, k, cfg.E, cfg.R, dev)
        nws = ep.ep_layout_workspace_bytes(T, k, cfg.E, cfg.R)
        self.ws = torch.zeros(max(nws, 16), dtype=torch.uint8, device=dev)
        self.recv = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
        self.q = torch.empty((T * k, H), dtype=torch.float8_e4m3fn, device=dev)
        self.s = torch.empty((T * k, H // 128), dtype=torch.float32, device=dev)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.d_err = torch.zeros(1, dtype=torch.int32, device=dev)

    def load(self, b, stream):
        with torch.cuda.stream(stream):
            self.idx.copy_(b.idx, non_blocking=True)
            self.x.copy_(b.x, non_blocking=True)
            self.w.copy_(b.w, non_blocking=True)
            # rows no slot points at are left untouched by dispatch; start
            # them at zero like the oracle's buffers
            self.recv.zero_()
            self.q.view(torch.uint8).zero_()
            self.s.zero_()

    def run(self, stream):
        c = self.cfg
        ep.ep_get_layout(self.idx, c.E, c.R, out=self.L, ws=self.ws, d_err=self.d_err,
                         stream=stream)
        ep.ep_dispatch(self.x, self.L.slot_pos, recv=self.recv, d_err=self.d_err, stream=stream)
        ep.ep_dispatch(self.x, self.L.slot_pos, fp8=True, recv=self.q, recv_scale=self.s,
                       d_err=self.d_err, stream=stream)
        ep.ep_combine(self.recv, self.L.slot_pos, self.w, out=self.out, d_err=self.d_err,
                      stream=stream)

    def check(self, expect):
        ref, recv, q, s, out = expect
        for key in LAYOUT_KEYS:
            np.testing.assert_array_equal(getattr(self.L, key).cpu().numpy().reshape(-1),
                                          ref[key].reshape(-1), err_msg=key)
        np.testing.assert_array_equal(tensor_bits16(self.recv), recv)
        np.testing.assert_array_equal(tensor_bytes(self.q), q)
        np.testing.assert_array_equal(self.s.cpu().numpy().view(np.uint32), s.view(np.uint32))
        np.testing.assert_array_equal(tensor_bits16(self.out), out)
        assert ep.ep_read_error(self.d_err) == ep.EP_OK


@pytest.mark.parametrize("T", [300, 5000])
def test_two_streams_at_once(T):
    cfg = workloads.CONFIGS["prefill"]
    b1 = workloads.make_batch(cfg, 31, T=T, H=1024)
    b2 = workloads.make_batch(cfg, 32, T=T, H=1024)
    p1, p2 = Path(cfg, T, 1024), Path(cfg, T, 1024)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    p1.load(b1, s1)
    p2.load(b2, s2)
    for _ in range(3):          # interleaved launches on both streams
        p1.run(s1)
        p2.run(s2)
    torch.cuda.synchronize()
    p1.check(_expect(cfg, b1))
    p2.check(_expect(cfg, b2))


def test_graph_replay_with_new_inputs():
    cfg = workloads.CONFIGS["decode"]
    T, H = cfg.T, 2048
    p = Path(cfg, T, H)
    st = torch.cuda.Stream()
    first = workloads.make_batch(cfg, 40, H=H)
    p.load(first, st)
    with torch.cuda.stream(st):
        p.run(st)               # warm-up outside the capture
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        p.run(st)
    for seed in (41, 42):
        b = workloads.make_batch(cfg, seed, H=H, drop_frac=0.05)
        p.load(b, st)
        with torch.cuda.stream(st):
            g.replay()
        st.synchronize()
        p.check(_expect(cfg, b))
    del g
