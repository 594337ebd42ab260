"""Host-side logic of bench.py: the multi-rank timing reduction (world size 2 over gloo, on CPU),
the clock-record parser, and the algorithmic work model."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from moe_inputs import configs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w = bench.init_dist("gloo")
    assert (r, w) == (rank, world)
    bench.barrier()
    out[rank] = bench.reduce_max(1.5 + rank)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_reduce_max_single_process_is_identity():
    assert bench.reduce_max(3.25) == 3.25


def test_clock_parser():
    text = ("0, 1965, 1965, 700.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
            "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
            "0, 1950, 1965, 980.2, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n")
    c = bench.ClockSampler.parse(text)
    assert c["sm_mhz"] == 1950 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    bad = text.replace("Not Active, Not Active, Not Active, Active", "Active, Not Active, Not Active, Active")
    assert "hw_slowdown" in bench.ClockSampler.parse(bad)["reasons"]


def test_work_model_matches_hand_count():
    cfg = configs.MUSE_PREFILL
    w = bench.work_model(cfg, 256)
    # 2 * (8192*256 + 8192*4096 + 8*3*4096^2 + 4096*8192) FLOP per token
    per_token = 2 * (8192 * 256 + 8192 * 4096 + 8 * 3 * 4096 ** 2 + 4096 * 8192)
    assert w["flops"] == per_token * cfg.T
    assert per_token == pytest.approx(943.7e6, rel=1e-4)
    assert w["gate_up"]["flops"] == 2 * cfg.T * 8 * 4096 * 8192
    # decode: weight bytes of the routed experts dominate
    d = bench.work_model(configs.MUSE_DECODE, 222)
    assert d["bytes"] == pytest.approx(222 * 100663296 + 2 * 67108864 + 4194304 + 2 * 64 * 8192 * 2)


def test_default_cpu_sample_is_bounded():
    for cfg in configs.CONFIGS.values():
        n = bench.default_cpu_sample(cfg)
        assert 1 <= n <= max(cfg.T, os.cpu_count() or 1)


def test_traffic_scales_the_capture_and_goes_null_for_another_kernel(monkeypatch):
    """The bench's measured-traffic field: the capture case's DRAM bytes scaled by the units a full
    launch processes (routed rows at prefill, routed experts at decode), and null as soon as the
    kernel source differs from the one that was captured."""
    caps = {"kernel_sha256_16": bench.kernel_fingerprint(),
            "muse_prefill": {"bytes": 1.0e9, "experts": 32, "rows": 2048 * 8},
            "muse_decode": {"bytes": 2.0e9, "experts": 29, "rows": 8 * 8}}
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURES", caps)
    pf = configs.MUSE_PREFILL
    assert bench.gate_up_traffic(pf, 256) == round(1.0e9 * pf.T * pf.top_k / (2048 * 8))
    assert bench.gate_up_traffic(configs.MUSE_DECODE, 228) == round(2.0e9 * 228 / 29)
    assert bench.gate_up_traffic(configs.SHAZEER_BF16, 256) is None  # no capture for it
    monkeypatch.setitem(caps, "kernel_sha256_16", "0" * 16)
    assert bench.gate_up_traffic(pf, 256) is None
