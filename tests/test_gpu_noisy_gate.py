"""Parity of moe_noisy_gate (Shazeer et al.'s noisy top-k gate with its importance and smooth-load
statistics) with the CPU oracle, on seeded inputs and seeded standard-normal draws.

The selection is compared bit for bit with the oracle's KeepTopK run on the GPU's noisy logits;
gate weights, noisy logits and load probabilities within tolerances derived from the fp32 logit
error; importance and load sums within the same tolerance plus one unit per token whose
selection is not unique (a near tie at the k-th or (k+1)-th place)."""
import ctypes

import numpy as np
import pytest

import moe_inputs
import oracle
from moe_inputs import configs

from gpu_harness import abi_config, logit_atol

torch = pytest.importorskip("torch")
moe = pytest.importorskip("sparse_moe_layer_softmax_b200")
pytestmark = pytest.mark.gpu


def oracle_noisy(cfg, inp):
    c = oracle.make_cfg(cfg.replace(gate_mode=configs.GATE_SOFTMAX))
    keep = oracle._Keep()
    x = oracle.make_tensors(cfg, inp, keep, experts={})
    xn = oracle.make_tensors(cfg, dict(inp, w_router=inp["w_noise"]), keep, experts={})
    T, n, k = cfg.T, cfg.n_experts, cfg.top_k
    l, m = np.zeros((T, n)), np.zeros((T, n))
    idx = np.zeros(k, dtype=np.int32)
    w = np.zeros(k)
    for t in range(T):
        oracle.lib().orc_router_token(ctypes.byref(c), ctypes.byref(x), t, l[t].ctypes.data,
                                      idx.ctypes.data, w.ctypes.data)
        oracle.lib().orc_router_token(ctypes.byref(c), ctypes.byref(xn), t, m[t].ctypes.data,
                                      idx.ctypes.data, w.ctypes.data)
    H, G, P, sel = oracle.noisy_gate(l, m, inp["noise_eps"].astype(np.float64), k)
    return {"l": l, "m": m, "H": H, "G": G, "P": P, "idx": sel}


CASES = [
    configs.small_shazeer(T=300, d=128, h=256, n=16, k=4, seed=41, noisy_gate=True),   # GEMM router
    configs.small_shazeer(T=40, d=256, h=256, n=64, k=2, seed=42, noisy_gate=True),    # few tokens
    configs.TINY_SHAZEER_F32.replace(T=70, seed=43, noisy_gate=True, router_gain=1.0),  # fp32
    configs.SHAZEER_BF16_NOISY,                                                          # full size
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: f"{c.name}-T{c.T}-{c.dtype}")
def test_noisy_gate(cfg):
    dev = moe_inputs.device_inputs(cfg)
    res = moe.noisy_gate(abi_config(cfg), dev["u"], dev["w_router"], dev["w_noise"],
                         dev["noise_eps"])
    assert moe.moe_get_device_status() == 0
    H = res["H"].cpu().numpy()
    idx = res["idx"].cpu().numpy()
    w = res["w"].cpu().numpy()
    P = res["P"].cpu().numpy()
    inp = moe_inputs.host_inputs(cfg)
    ref = oracle_noisy(cfg, inp)
    k, n = cfg.top_k, cfg.n_experts
    # selection: the oracle's KeepTopK on the GPU's fp32 noisy logits, bit for bit
    sel, wsel = oracle.softmax_topk(H.astype(np.float32), k)
    np.testing.assert_array_equal(idx, sel)
    np.testing.assert_allclose(w, wsel, rtol=2e-6, atol=1e-7)
    # noisy logits: |dH| <= |dl| + |eps| * |dm| (softplus is 1-Lipschitz)
    eps = inp["noise_eps"].astype(np.float64)
    atol_l = logit_atol(cfg, ref["l"]) + 1e-6 * np.abs(ref["l"]).max()
    atol_h = atol_l * (1.0 + np.abs(eps).max())
    np.testing.assert_allclose(H, ref["H"], rtol=0, atol=atol_h)
    # tokens whose k-th / (k+1)-th / (k+2)-th noisy logits nearly tie have no unique selection or
    # bar; compare the rest
    s = -np.sort(-ref["H"], axis=1)
    gaps = np.minimum(s[:, k - 1] - s[:, k], s[:, k] - s[:, k + 1] if k + 1 < n else np.inf)
    ties = gaps < 4 * atol_h
    assert ties.sum() <= max(2, cfg.T // 50)
    np.testing.assert_array_equal(idx[~ties], ref["idx"][~ties])
    # load probabilities: Phi moves by at most phi(0) * (|dl| + |d bar|) / softplus(m)
    sp = np.log1p(np.exp(ref["m"]))
    atol_p = 0.4 * (atol_l + atol_h) / sp + 1e-6
    bad = np.abs(P - ref["P"]) > atol_p
    assert not bad[~ties].any(), f"{bad[~ties].sum()} load probabilities off"
    # batch statistics: GPU sums over all tokens; near-tie tokens may add up to 1 each
    imp = res["importance"].cpu().numpy().astype(np.float64)
    load = res["load"].cpu().numpy().astype(np.float64)
    tol_sum = ties.sum() + 1e-4 * cfg.T
    np.testing.assert_allclose(imp, ref["G"].sum(0), rtol=0, atol=tol_sum)
    np.testing.assert_allclose(load, ref["P"].sum(0), rtol=0, atol=tol_sum + atol_p.sum(0).max())
    assert abs(imp.sum() - cfg.T) < 1e-3 * cfg.T  # each token's gate sums to 1
    cv2 = res["cv2"].cpu().numpy()
    assert cv2[0] == pytest.approx(oracle.cv_squared(imp), rel=1e-4, abs=1e-7)
    assert cv2[1] == pytest.approx(oracle.cv_squared(load), rel=1e-4, abs=1e-7)
    print(f"{cfg.name}: ties {int(ties.sum())}, CV^2 importance {cv2[0]:.4f} "
          f"(oracle {oracle.cv_squared(ref['G'].sum(0)):.4f}), load {cv2[1]:.4f} "
          f"(oracle {oracle.cv_squared(ref['P'].sum(0)):.4f})")
