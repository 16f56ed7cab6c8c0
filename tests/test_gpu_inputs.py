"""The seeded input recipe names the same tensors on every device: inputs and
cotangents drawn for the GPU equal, bit for bit, those drawn on the host with
the same seed (the draws and the rounding happen on the host; only the
rounded tensors move), so a host re-draw reproduces what a GPU run used."""
import pytest
import torch

from attention_forward_mode_b200.workloads import custom, make_cotangents, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("row_scale", [False, True])
def test_same_tensors_on_host_and_device(row_scale):
    w = custom(1, 3, 300, 257, 128, kv_row_scale=row_scale, q_std=2.0, t_std=0.1)
    dev = make_inputs(w, seed=11, device="cuda")
    host = make_inputs(w, seed=11, device="cpu")
    for n in host:
        assert dev[n].is_cuda and dev[n].dtype == torch.bfloat16
        assert torch.equal(dev[n].cpu(), host[n]), n
    dc, hc = make_cotangents(w, seed=12, device="cuda"), make_cotangents(w, seed=12, device="cpu")
    for n in hc:
        assert torch.equal(dc[n].cpu(), hc[n]), n
