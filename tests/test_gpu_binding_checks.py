"""The Python binding refuses tensors the library would write through out
of bounds (wrong shape, dtype or device) before any call reaches it."""
import pytest
import torch

import combine_ep_get_09_b200 as ep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ep.lib()


def _inputs(T=16, k=4, H=512):
    dev = "cuda"
    idx = torch.randint(0, 16, (T, k), device=dev)
    x = torch.randn(T, H, device=dev).to(torch.bfloat16)
    return idx, x


def test_layout_output_sizes():
    idx, _ = _inputs()
    L = ep.empty_layout(16, 4, 16, 4, "cuda")
    bad = L._replace(slot_pos=torch.empty((16, 3), dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError, match="slot_pos"):
        ep.ep_get_layout(idx, 16, 4, out=bad)
    bad = L._replace(cnt_e=torch.empty(15, dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError, match="cnt_e"):
        ep.ep_layout_dispatch(idx, 16, 4, _inputs()[1], out=bad)


def test_dispatch_receive_buffers():
    idx, x = _inputs()
    L = ep.ep_get_layout(idx, 16, 4)
    with pytest.raises(ValueError, match="recv"):
        ep.ep_dispatch(x, L.slot_pos, recv=torch.empty((64, 256), dtype=torch.bfloat16,
                                                       device="cuda"))
    with pytest.raises(ValueError, match="recv"):
        ep.ep_dispatch(x, L.slot_pos, recv=torch.empty((64, 512), dtype=torch.float16,
                                                       device="cuda"))
    with pytest.raises(ValueError, match="recv_scale"):
        ep.ep_dispatch(x, L.slot_pos, fp8=True,
                       recv=torch.empty((64, 512), dtype=torch.float8_e4m3fn, device="cuda"),
                       recv_scale=torch.empty((63, 4), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError, match="recv"):
        ep.ep_layout_dispatch(idx, 16, 4, x, recv=torch.empty((63, 512), dtype=torch.bfloat16,
                                                             device="cuda"))
    with pytest.raises(ValueError, match="slot_pos"):
        ep.ep_dispatch(x, L.slot_pos[:8])


def test_combine_outputs_and_weights():
    idx, x = _inputs()
    L = ep.ep_get_layout(idx, 16, 4)
    y = ep.ep_dispatch(x, L.slot_pos)
    w = torch.rand(16, 4, device="cuda")
    with pytest.raises(ValueError, match="out"):
        ep.ep_combine(y, L.slot_pos, w, out=torch.empty((16, 256), dtype=torch.bfloat16,
                                                        device="cuda"))
    with pytest.raises(ValueError, match="w must"):
        ep.ep_combine(y, L.slot_pos, w[:, :3].contiguous())
    with pytest.raises(ValueError, match="d_err"):
        ep.ep_combine(y, L.slot_pos, w, d_err=torch.zeros(1, dtype=torch.int64, device="cuda"))
    with pytest.raises(ValueError, match="CUDA"):
        ep.ep_combine(y, L.slot_pos, w, out=torch.empty((16, 512), dtype=torch.bfloat16))
