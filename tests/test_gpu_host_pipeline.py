"""moe_layer_forward_host: batches in pinned host memory streamed through the layer with the copies
of neighbouring batches overlapping each batch's kernels.  Every output must equal, bit for bit,
the device-memory forward of the same batch (the pipeline only moves data; the layer's own parity
with the oracle is covered by the other GPU tests)."""
import numpy as np
import pytest

import moe_inputs
from moe_inputs import configs

from gpu_harness import abi_config

torch = pytest.importorskip("torch")
moe = pytest.importorskip("sparse_moe_layer_softmax_b200")
pytestmark = pytest.mark.gpu

CASES = [
    configs.small_muse(T=300, d=256, L=128, I=128, n=16, k=4, seed=61),   # latent Muse, bf16
    configs.small_shazeer(T=77, d=128, h=256, n=16, k=4, seed=62),        # Shazeer ReLU, bf16
    configs.TINY_SHAZEER_F32.replace(T=50, seed=63),                      # fp32 (4-byte rows)
]


def batch_inputs(cfg, n):
    """n distinct seeded inputs of the workload's shape (the weights stay those of cfg)."""
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    out = []
    for i in range(n):
        t = torch.empty((cfg.T, cfg.d_model), dtype=dt, device="cuda")
        moe_inputs.normal_device(t, cfg.seed + 1000 + i, configs.STREAM_X, 0, cfg.x_sigma)
        out.append(t)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: f"{c.name}-{c.dtype}")
@pytest.mark.parametrize("n_batches", [1, 2, 5])
def test_host_pipeline_equals_device_forward(cfg, n_batches):
    dev = moe_inputs.device_inputs(cfg)
    layer = moe.MoELayer(abi_config(cfg), dev)
    us = batch_inputs(cfg, n_batches)
    expected = [layer.forward(u, u) for u in us]
    torch.cuda.synchronize()
    u_hosts = [u.cpu().pin_memory() for u in us]
    out_hosts = [torch.full_like(h, float("nan")).pin_memory() for h in u_hosts]
    layer.forward_host(u_hosts, out_hosts)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    for i in range(n_batches):
        a = expected[i].cpu().view(torch.int16 if cfg.dtype == "bf16" else torch.int32).numpy()
        b = out_hosts[i].view(torch.int16 if cfg.dtype == "bf16" else torch.int32).numpy()
        np.testing.assert_array_equal(b, a, err_msg=f"batch {i}")


def test_host_pipeline_zero_batches_and_reuse():
    cfg = CASES[0]
    dev = moe_inputs.device_inputs(cfg)
    layer = moe.MoELayer(abi_config(cfg), dev)
    layer.forward_host([], [])
    torch.cuda.synchronize()
    # the same host buffers reused across calls and within one call (sequential outputs)
    us = batch_inputs(cfg, 3)
    expected = layer.forward(us[2], us[2]).cpu()
    u_hosts = [u.cpu().pin_memory() for u in us]
    out = torch.empty_like(u_hosts[0]).pin_memory()
    for _ in range(2):
        layer.forward_host(u_hosts, [out] * 3)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), expected.view(torch.int16))
