"""The seeded input generator: reproducibility, random access, distributions, recipes."""
import json
import math
import os

import numpy as np

import moe_inputs
from moe_inputs import configs


def test_random_access_and_reproducible():
    a = moe_inputs.normal_host(3, 5, 0, 100000, 0.5, "f32")
    b = moe_inputs.normal_host(3, 5, 777, 1000, 0.5, "f32")
    np.testing.assert_array_equal(a[777:1777], b)
    np.testing.assert_array_equal(a, moe_inputs.normal_host(3, 5, 0, 100000, 0.5, "f32"))
    assert not np.array_equal(a, moe_inputs.normal_host(3, 6, 0, 100000, 0.5, "f32"))
    assert not np.array_equal(a, moe_inputs.normal_host(4, 5, 0, 100000, 0.5, "f32"))


def test_thread_count_does_not_change_values():
    k = moe_inputs.key(9, 1)
    s = moe_inputs.lib().gen_normal_scale(1.0)
    outs = []
    for nt in (1, 3, 8):
        o = np.empty(300001, np.uint16)
        moe_inputs.lib().gen_normal_bf16_host(k, 11, o.size, s, o.ctypes.data, nt)
        outs.append(o)
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])


def test_normal_moments():
    x = moe_inputs.normal_host(1, 1, 0, 1 << 21, 2.0, "f32").astype(np.float64)
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 2.0) < 0.01
    # Irwin-Hall(8): bounded tails at ~4.9 sigma, excess kurtosis -6/(5*8) = -0.15
    assert np.abs(x).max() <= 2.0 * 524280 / (65536 * math.sqrt(8 / 3)) * (1 + 1e-6)
    kurt = np.mean((x / x.std()) ** 4) - 3
    assert abs(kurt + 0.15) < 0.02


def test_bf16_is_rne_of_f32():
    import torch
    f = moe_inputs.normal_host(2, 2, 0, 50000, 1.0, "f32")
    b = moe_inputs.normal_host(2, 2, 0, 50000, 1.0, "bf16")
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(b, ref)


def test_uniform_range():
    u = moe_inputs.uniform_host(0, 9, 0, 1 << 20)
    assert u.min() >= 0.0 and u.max() < 1.0 and abs(u.mean() - 0.5) < 0.002


def test_rows_and_expert_slices_match_whole_tensor():
    cfg = configs.small_muse(T=10)
    full = moe_inputs.host_inputs(cfg)
    rows = moe_inputs.host_rows(cfg, "u", rows=[3, 7])
    np.testing.assert_array_equal(rows, full["u"][[3, 7]])
    np.testing.assert_array_equal(moe_inputs.host_rows(cfg, "w_gu", lead=5), full["w_gu"][5])


def test_subsample_is_seeded_sorted_distinct():
    cfg = configs.MUSE_PREFILL
    s = moe_inputs.subsample_tokens(cfg)
    assert len(s) == 512 and len(set(s.tolist())) == 512 and np.all(np.diff(s) > 0)
    assert s.max() < cfg.T
    np.testing.assert_array_equal(s, moe_inputs.subsample_tokens(cfg))


def test_zipf_scale_matches_calibration_output():
    path = os.path.join(os.path.dirname(__file__), "golden", "zipf_bias_scale.json")
    with open(path) as f:
        assert json.load(f)["zipf_bias_scale"] == configs.ZIPF_BIAS_SCALE


def test_redrawn_rows_come_from_their_generation():
    cfg = configs.MUSE_DECODE
    assert cfg.u_redraw, "the decode workload has stored redraws"
    full = moe_inputs.host_rows(cfg, "u")
    first = moe_inputs.host_rows(cfg.replace(u_redraw=()), "u")
    red = dict(cfg.u_redraw)
    for t in range(cfg.T):
        g = red.get(t, 0)
        row = moe_inputs.normal_host(cfg.seed, configs.STREAM_X, (g * cfg.T + t) * cfg.d_model,
                                     cfg.d_model, cfg.x_sigma, "bf16")
        np.testing.assert_array_equal(full[t], row)
        assert np.array_equal(full[t], first[t]) == (g == 0)
    rows = sorted(red)[:2] + [0]
    np.testing.assert_array_equal(moe_inputs.host_rows(cfg, "u", rows=rows), full[rows])
    # deriving a workload drops the list (it belongs to one workload)
    assert cfg.replace(T=32).u_redraw == () and configs.small_muse().u_redraw == ()


def _separation():
    import importlib.util
    path = os.path.join(os.path.dirname(__file__), "golden", "separate_router_logits.py")
    spec = importlib.util.spec_from_file_location("separate_router_logits", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


SMALL_SEPARATED = ("tiny_shazeer_f32", "shazeer_bf16", "muse_decode", "muse_decode_sigmoid",
                   "muse_decode_block")


def test_stored_redraws_recomputed_for_small_workloads():
    sep = _separation()
    for name in SMALL_SEPARATED:
        cfg = configs.ALL_CONFIGS[name]
        red, _ = sep.redraws_for(cfg)
        assert red == cfg.u_redraw, name


def test_large_workloads_are_separated_on_redrawn_and_sampled_tokens():
    sep = _separation()
    for name in configs.SEPARATED_NAMES:
        if name in SMALL_SEPARATED:
            continue
        cfg = configs.ALL_CONFIGS[name]
        sample = moe_inputs.fisher_yates(cfg.seed + 77, configs.STREAM_SUBSAMPLE, cfg.T, 256)
        toks = np.union1d(np.array([t for t, _ in cfg.u_redraw], dtype=np.int64), sample)
        ratio = sep.check_separated(cfg, toks)
        assert ratio.min() >= 1.0, (name, float(ratio.min()))
        # and the first draw of those redrawn tokens was not separated
        red = np.array([t for t, _ in cfg.u_redraw][:64], dtype=np.int64)
        assert sep.check_separated(cfg.replace(u_redraw=()), red).max() < 1.0, name
