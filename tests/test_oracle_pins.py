"""Pins of the CPU oracle to facts that do not come from the oracle itself.

* values the pages print for worked examples (tests/golden/*.json, each with its citation);
* closed forms and invariants (weights sum to 1, alpha^2 + beta^2 = 1, scale invariance of I_gamma);
* special cases that reduce to library routines (k = n is the dense softmax mixture, k = 1 is a
  single expert, Softmax(KeepTopK) written with -inf masking, a stable lexicographic sort for the
  permutation);
* brute force on tiny layers: every expert evaluated densely with numpy matmuls and torch's bf16
  conversion, then gathered, compared with the per-token oracle.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from moe_inputs import configs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ worked examples


def test_norm_worked_example():
    g = gold("norm_worked_example.json")
    x, gamma = np.array(g["x"]), np.array(g["gamma"])
    c = oracle.centered_rmsnorm(x, gamma, eps=g["eps"])
    i = oracle.input_scaled_rmsnorm(x, gamma, eps=g["eps"])
    np.testing.assert_allclose(c, g["centered"], rtol=1e-15)
    expect = np.array(g["input_scaled_numerator"]) / math.sqrt(g["input_scaled_divisor_squared"])
    np.testing.assert_allclose(i, expect, rtol=1e-15)
    # the vector I_gamma reduces is D_gamma x itself (the example's numerator)
    np.testing.assert_array_equal(oracle.input_scaled_vector(x, gamma, is_bf16=2),
                                  g["input_scaled_numerator"])
    # the two orders are collinear but not equal (same page)
    assert abs(c[0] * i[1] - c[1] * i[0]) < 1e-15 and not np.allclose(c, i)


def test_normalize_before_mix_counterexample():
    g = gold("normalize_before_mix.json")
    cfg = oracle.OrcCfg(is_bf16=2, top_k=2, d_model=2, d_latent=2, expert_norm=1)
    outs = [np.array(o) for o in g["expert_outputs"]]
    zero = np.zeros(2)
    ns = np.stack([oracle.input_scaled_rmsnorm(o, zero, eps=0.0) for o in outs])
    w = np.array(g["weights"])
    y = np.zeros(2)
    oracle.lib().orc_combine_token(oracle.ctypes.byref(cfg), ns.ctypes.data, w.ctypes.data,
                                   y.ctypes.data)
    np.testing.assert_allclose(y, g["normalize_then_mix"], rtol=1e-7)
    wrong = oracle.rms_normalize(w[0] * outs[0] + w[1] * outs[1])
    expect_wrong = np.array(g["mix_then_normalize_numerator"]) / math.sqrt(
        g["mix_then_normalize_divisor_squared"])
    np.testing.assert_allclose(wrong, expect_wrong, rtol=1e-15)
    assert np.max(np.abs(y - wrong)) > 0.5


def test_gate_worked_example():
    g = gold("gate_worked_example.json")
    idx, w = oracle.softmax_topk(np.array(g["logits"], dtype=np.float64), g["k"])
    assert list(idx) == g["selected_zero_based"]
    np.testing.assert_allclose(np.round(w, g["printed_decimals"]), g["gates_3dp"], atol=0)
    assert abs(w.sum() - 1.0) < 1e-15


def test_residual_gate_values():
    g = gold("residual_gate.json")
    a, b = oracle.resid_gate_coeffs(g["g_half"], g["tau"], g["delta"])
    assert b == pytest.approx(g["beta_half"], abs=1e-15)
    assert a == pytest.approx(g["alpha_half"], abs=1e-15)
    aligned = (a + b) ** 2        # |a r + b r|^2 for a unit vector r
    opposite = (a - b) ** 2       # |a r - b r|^2
    assert round(aligned, 3) == g["aligned_factor_3dp"]
    assert round(opposite, 3) == g["opposite_factor_3dp"]
    # orthogonal equal-norm vectors keep the squared norm (alpha^2 + beta^2 = 1)
    assert a * a + b * b == pytest.approx(1.0, abs=1e-15)


def test_residual_gate_floor():
    g = gold("residual_gate.json")
    tau, delta = g["tau"], g["delta"]
    # floor is active iff (1 - beta)(1 + beta) < delta, i.e. beta > sqrt(1 - delta)
    g_on = tau * math.log(math.sqrt(1 - delta) / (1 - math.sqrt(1 - delta))) + 1e-6
    for gv in np.linspace(-3, g_on - 1e-3, 57):
        a, b = oracle.resid_gate_coeffs(float(gv), tau, delta)
        assert a * a + b * b == pytest.approx(1.0, abs=1e-12)
        assert b == pytest.approx(1 / (1 + math.exp(-gv / tau)), rel=1e-14)
    for gv in (g_on + 1e-3, 3.0, 10.0, 100.0):
        a, _ = oracle.resid_gate_coeffs(gv, tau, delta)
        assert a == pytest.approx(g["alpha_floor"], rel=1e-14)


# ------------------------------------------------------------------ norms


def test_norm_invariants():
    rng = np.random.default_rng(0)
    for D in (2, 7, 64, 4096):
        x = rng.normal(size=D) * 3.0
        gamma = rng.normal(size=D) * 0.3
        r = oracle.rms_normalize(x, 0.0)
        assert math.sqrt(np.mean(r * r)) == pytest.approx(1.0, rel=1e-13)
        # gamma = 0 reduces both gains to R
        np.testing.assert_allclose(oracle.centered_rmsnorm(x, 0 * gamma, 0.0), r, rtol=1e-14)
        np.testing.assert_allclose(oracle.input_scaled_rmsnorm(x, 0 * gamma, 0.0), r, rtol=1e-14)
        # I_gamma is invariant to positive scaling of its input and has unit RMS at eps = 0
        i1 = oracle.input_scaled_rmsnorm(x, gamma, 0.0)
        i2 = oracle.input_scaled_rmsnorm(7.5 * x, gamma, 0.0)
        np.testing.assert_allclose(i1, i2, rtol=1e-13)
        assert math.sqrt(np.mean(i1 * i1)) == pytest.approx(1.0, rel=1e-13)
        # C_gamma's RMS is the RMS of (1+gamma)*R(x), not 1
        c = oracle.centered_rmsnorm(x, gamma, 0.0)
        np.testing.assert_allclose(c, (1 + gamma) * r, rtol=1e-14)
        # eps enters under the root, next to the mean
        e = oracle.rms_normalize(x, 0.25)
        np.testing.assert_allclose(e, x / np.sqrt(np.mean(x * x) + 0.25), rtol=1e-14)


def test_input_scaled_rounds_scaled_vector():
    # With bf16 storage, D_gamma x is rounded to bf16 before the reduction.
    x = np.array([1.0, 1.0, 1.0, 1.0])
    gamma = np.array([1.0 / 256 + 1e-9, 0.0, 0.0, 0.0])  # (1+gamma)*1 rounds back to 1 in bf16
    i_bf16 = oracle.input_scaled_rmsnorm(x, gamma, 0.0, is_bf16=1)
    i_f32 = oracle.input_scaled_rmsnorm(x, gamma, 0.0, is_bf16=2)
    np.testing.assert_allclose(i_bf16, np.ones(4), rtol=1e-15)
    assert i_f32[0] > 1.0 + 1e-3


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(size=2000) * 10 ** rng.uniform(-6, 6, 2000),
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, 65504.0]])
    mine = oracle.bf16_round(v)
    ref = torch.tensor(v, dtype=torch.float64).to(torch.float32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(mine, ref)
    assert mine[-5] == 1.0 and mine[-4] == 1.015625  # ties go to even


# ------------------------------------------------------------------ gate


def test_topk_equals_softmax_of_keeptopk():
    rng = np.random.default_rng(2)
    for n, k in ((4, 2), (8, 2), (16, 4), (256, 8), (256, 1), (8, 8)):
        l = rng.normal(size=(50, n)) * 2
        idx, w = oracle.softmax_topk(l, k)
        for r in range(50):
            top = np.argsort(-l[r], kind="stable")[:k]
            assert list(idx[r]) == list(top)
            masked = np.full(n, -np.inf)
            masked[top] = l[r, top]
            g = np.exp(masked - masked.max())
            g /= g.sum()
            np.testing.assert_allclose(w[r], g[top], rtol=1e-13)
            assert abs(w[r].sum() - 1.0) < 1e-14
            assert np.all(np.diff(w[r]) <= 0)


def test_topk_tie_break_lower_index():
    idx, w = oracle.softmax_topk(np.array([0.5, 1.0, 1.0, 0.25, 1.0]), 2)
    assert list(idx) == [1, 2]
    np.testing.assert_allclose(w, [0.5, 0.5])


def test_topk_f32_logits_path():
    rng = np.random.default_rng(3)
    l = rng.normal(size=(20, 64)).astype(np.float32)
    i32, w32 = oracle.softmax_topk(l, 8)
    i64, w64 = oracle.softmax_topk(l.astype(np.float64), 8)
    np.testing.assert_array_equal(i32, i64)
    np.testing.assert_array_equal(w32, w64)


# ------------------------------------------------------------------ permutation


def test_permutation_against_lexsort():
    rng = np.random.default_rng(4)
    for T, k, n in ((1, 1, 1), (5, 2, 3), (37, 4, 16), (300, 8, 64), (64, 8, 256)):
        idx = np.stack([rng.choice(n, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        off, perm, inv = oracle.permutation(T, k, n, idx)
        e_flat = idx.reshape(-1)
        t_flat = np.repeat(np.arange(T), k)
        order = np.lexsort((t_flat, e_flat))  # stable: expert, then token
        np.testing.assert_array_equal(perm, t_flat[order])
        expect_inv = np.empty(T * k, dtype=np.int64)
        expect_inv[order] = np.arange(T * k)
        np.testing.assert_array_equal(inv, expect_inv)
        np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(e_flat,
                                                                                      minlength=n))]))
        assert sorted(inv.tolist()) == list(range(T * k))


def test_permutation_rejects_bad_indices():
    with pytest.raises(ValueError):
        oracle.permutation(2, 2, 4, np.array([[0, 4], [1, 2]]))
    with pytest.raises(ValueError):
        oracle.permutation(2, 2, 4, np.array([[0, 0], [1, 2]]))


# ------------------------------------------------------------------ brute force layers


def _rnd(x, dtype):
    t = torch.tensor(x, dtype=torch.float64).to(torch.float32)
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.double().numpy()


def _val(a, dtype):
    if dtype == "bf16":
        return torch.from_numpy(a.astype(np.int16)).view(torch.bfloat16).double().numpy()
    return a.astype(np.float64)


def dense_bruteforce(cfg, inp):
    """Every expert evaluated on every token with numpy matmuls, then gathered by the gate."""
    dt = cfg.dtype
    u = _val(inp["u"], dt)
    h = u  # the residual stream
    if cfg.input_norm:
        gi = inp["gamma_in"].astype(np.float64)
        u = _rnd((1 + gi) * h / np.sqrt(np.mean(h * h, 1, keepdims=True) + cfg.eps_block), dt)
    wr = _val(inp["w_router"], "f32" if cfg.router_f32 else dt)
    logits = u @ wr.T
    if cfg.gate_mode == configs.GATE_SIGMOID:
        logits = logits * cfg.logit_mult
    if "logit_bias" in inp:
        logits = logits + inp["logit_bias"].astype(np.float64)
    if cfg.gate_mode == configs.GATE_SIGMOID:
        s = 1.0 / (1.0 + np.exp(-logits))
        key = s + inp["correction_bias"].astype(np.float64)
        top = np.argsort(-key, axis=1, kind="stable")[:, :cfg.top_k]
        w = np.take_along_axis(s, top, 1)
        w = w / (w.sum(1, keepdims=True) + 1e-15) * cfg.routed_scale
        logits = s  # the oracle reports the scores in this mode
    else:
        p = np.exp(logits - logits.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        top = np.argsort(-logits, axis=1, kind="stable")[:, :cfg.top_k]
        w = np.take_along_axis(p, top, 1)
        w = w / w.sum(1, keepdims=True) * cfg.routed_scale
    if cfg.latent:
        zr = _rnd(u @ _val(inp["p_down"], dt).T, dt)
        if cfg.pre_norm:
            g = inp["gamma_pre"].astype(np.float64)
            z = _rnd((1 + g) * zr / np.sqrt(np.mean(zr * zr, 1, keepdims=True) + cfg.eps), dt)
        else:
            z = zr
    else:
        z = u
    W1 = _val(inp["w_gu"], dt)
    W2 = _val(inp["w_down"], dt)
    I = cfg.d_ff
    allout, allpre = [], []
    for e in range(cfg.n_experts):
        a = z @ W1[e].T
        if cfg.act == configs.ACT_SWIGLU:
            g, v = a[:, :I], a[:, I:]
            hid = _rnd(g / (1 + np.exp(-g)) * v, dt)
        else:
            hid = _rnd(np.maximum(a, 0), dt)
        o = _rnd(hid @ W2[e].T, dt)
        s = o
        if cfg.expert_norm:
            s = _rnd(o * (1 + inp["gamma_expert"].astype(np.float64)), dt)
            o = _rnd(s / np.sqrt(np.mean(s * s, 1, keepdims=True) + cfg.eps), dt)
        allout.append(o)
        allpre.append(s)
    allout = np.stack(allout, 1)  # [T, n, E]
    sel = np.take_along_axis(allout, top[:, :, None], 1)
    dense_bruteforce.last = {"z": z,
                             "s": np.take_along_axis(np.stack(allpre, 1), top[:, :, None], 1)}
    y = _rnd(np.einsum("tk,tke->te", w, sel), dt)
    if cfg.latent:
        b = _rnd(y @ _val(inp["p_up"], dt).T, dt)
    else:
        b = y
    if cfg.post_norm:
        sp = _rnd(b * (1 + inp["gamma_post"].astype(np.float64)), dt)
        b = _rnd(sp / np.sqrt(np.mean(sp * sp, 1, keepdims=True) + cfg.eps_block), dt)
    if cfg.resid_mode == configs.RESID_MUSE_GATE:
        gg = inp["resid_g"].astype(np.float64)
        beta = 1 / (1 + np.exp(-gg / cfg.tau))
        alpha = np.sqrt(np.maximum((1 / (1 + np.exp(gg / cfg.tau))) * (1 + beta), cfg.resid_floor))
        out = _rnd(alpha * h + beta * b, dt)
    elif cfg.resid_mode == configs.RESID_LITERAL:
        out = _rnd(h + inp["resid_g"].astype(np.float64) * b, dt)
    else:
        out = b
    return out, logits, top, w, y


BRUTE_CASES = [
    configs.small_shazeer(T=23, d=40, h=56, n=6, k=2).replace(dtype="f32", x_sigma=1.0),
    configs.small_shazeer(T=17, d=32, h=24, n=5, k=3),
    configs.small_muse(T=13, d=48, L=32, I=24, n=6, k=3, gamma_sigma=0.3),
    configs.small_muse(T=9, d=40, L=24, I=16, n=5, k=2, gamma_sigma=0.3, dtype="f32"),
    configs.small_muse(T=11, d=32, L=16, I=24, n=4, k=2, resid_mode=configs.RESID_LITERAL,
                       gamma_sigma=0.3),
    configs.small_muse(T=7, d=32, L=16, I=16, n=4, k=2, pre_norm=0, resid_mode=configs.RESID_NONE),
    # Muse sigmoid gate with fp32 router weights, output_multiplier and routed_scaling_factor
    configs.small_muse(T=15, d=48, L=32, I=24, n=8, k=3, gamma_sigma=0.3,
                       gate_mode=configs.GATE_SIGMOID, router_f32=1, logit_mult=2.0,
                       corr_sigma=0.3, routed_scale=1.5),
    configs.small_muse(T=10, d=40, L=24, I=16, n=6, k=2, dtype="f32",
                       gate_mode=configs.GATE_SIGMOID, router_f32=1),
    # decoder wrap: residual-stream norm before the MoE, output norm before the residual gate
    configs.small_muse(T=12, d=48, L=32, I=24, n=6, k=3, gamma_sigma=0.3, input_norm=1,
                       post_norm=1),
    configs.small_muse(T=8, d=40, L=24, I=16, n=5, k=2, dtype="f32", gamma_sigma=0.3,
                       input_norm=1, post_norm=1, resid_mode=configs.RESID_LITERAL),
]


def test_noisy_gate_chart_values():
    g = gold("noisy_gate_chart.json")
    # expert 0 has noise pre-activation 0; the bar it must clear is max(H_1, H_2) = 1 (k = 1)
    sp = math.log(2.0)
    assert round(sp, 3) == g["softplus_3dp"]

    def p0(l0):
        l = np.array([[l0, 1.0, -5.0]])
        _, _, P, _ = oracle.noisy_gate(l, np.zeros((1, 3)), np.zeros((1, 3)), 1)
        return P[0, 0]

    assert round(100 * p0(0.0), 2) == g["p_one_unit_below_bar_pct_2dp"]   # one unit below
    h = 1e-5
    slope = (p0(1.0 + h) - p0(1.0 - h)) / (2 * h)
    assert round(slope, 3) == g["slope_at_bar_3dp"]
    assert p0(1.0) == pytest.approx(0.5, abs=1e-15)                    # at the bar


def test_noisy_gate_cv_example():
    g = gold("noisy_gate_chart.json")
    v = np.array(g["importance_example"], dtype=np.float64)
    cv2 = oracle.cv_squared(v)
    assert cv2 == pytest.approx(g["population_variance"] / g["mean"] ** 2, rel=1e-15)
    assert round(math.sqrt(cv2), 2) == g["cv_2dp"] and round(cv2, 2) == g["cv_squared_2dp"]
    assert round(g["w_importance"] * cv2, 3) == g["loss_3dp"]
    assert oracle.cv_squared(np.full(4, 25.0)) == 0.0


def test_noisy_gate_against_library_routines():
    from scipy.stats import norm
    rng = np.random.default_rng(8)
    rows, n, k = 30, 12, 3
    l, m, eps = rng.normal(size=(rows, n)), rng.normal(size=(rows, n)), rng.normal(size=(rows, n))
    H, G, P, idx = oracle.noisy_gate(l, m, eps, k)
    sp = np.log1p(np.exp(m))
    np.testing.assert_allclose(H, l + eps * sp, rtol=1e-14)
    for r in range(rows):
        top = np.argsort(-H[r], kind="stable")[:k]
        assert idx[r].tolist() == top.tolist()
        e = np.exp(H[r, top] - H[r, top].max())
        dense = np.zeros(n)
        dense[top] = e / e.sum()
        np.testing.assert_allclose(G[r], dense, rtol=1e-13, atol=1e-300)
        for i in range(n):
            kth = np.sort(np.delete(H[r], i))[::-1][k - 1]
            assert P[r, i] == pytest.approx(norm.cdf((l[r, i] - kth) / sp[r, i]), rel=1e-12, abs=1e-300)
    # without noise the gate is the plain softmax top-k, and P approaches the hard top-k
    _, G0, P0, idx0 = oracle.noisy_gate(l, np.full((rows, n), -60.0), np.zeros((rows, n)), k)
    sel, w = oracle.softmax_topk(l, k)
    np.testing.assert_array_equal(idx0, sel)
    np.testing.assert_allclose(np.take_along_axis(G0, sel.astype(np.int64), 1), w, rtol=1e-13)
    hard = np.zeros_like(P0)
    np.put_along_axis(hard, sel.astype(np.int64), 1.0, 1)
    np.testing.assert_allclose(P0, hard, atol=1e-12)


def test_post_norm_output_has_unit_rms():
    """With post_norm, no residual and gamma_post = 0, every output row is R(b): unit RMS."""
    cfg = configs.small_muse(T=9, d=48, L=32, I=24, n=6, k=2, dtype="f32", post_norm=1,
                             resid_mode=configs.RESID_NONE, gamma_sigma=0.0, eps_block=0.0,
                             eps=0.0)
    res = oracle.layer_forward(cfg, moe_inputs.host_inputs(cfg))
    np.testing.assert_allclose(np.sqrt(np.mean(res["out"] ** 2, 1)), 1.0, rtol=1e-5)


@pytest.mark.parametrize("cfg", BRUTE_CASES, ids=lambda c: f"{c.name}-{c.dtype}-r{c.resid_mode}")
def test_layer_bruteforce(cfg):
    inp = moe_inputs.host_inputs(cfg)
    res = oracle.layer_forward(cfg, inp)
    out, logits, top, w, y = dense_bruteforce(cfg, inp)
    np.testing.assert_array_equal(res["idx"], top)
    np.testing.assert_allclose(res["logits"], logits, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["w"], w, rtol=1e-12)
    np.testing.assert_allclose(res["y"], y, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(res["out"], out, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("cfg", [c for c in BRUTE_CASES if c.latent], ids=lambda c: c.name)
def test_staged_intermediates_bruteforce(cfg):
    """The staged driver's expert inputs z and per-slot pre-norm expert outputs s (the vector
    I_gamma reduces) against the dense brute force."""
    inp = moe_inputs.host_inputs(cfg)
    toks = np.arange(cfg.T)

    def get_inputs(tokens):
        d = {k: v for k, v in inp.items() if k not in ("w_gu", "w_down")}
        d["u"] = inp["u"][tokens]
        return d

    res = oracle.layer_forward_staged(cfg, toks, get_inputs,
                                      lambda e: (inp["w_gu"][e], inp["w_down"][e]), want_s=True)
    dense_bruteforce(cfg, inp)
    ref = dense_bruteforce.last
    np.testing.assert_allclose(res["z"], ref["z"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(res["s"], ref["s"], rtol=1e-9, atol=1e-12)


def test_k_equals_n_is_dense_softmax_mixture():
    cfg = configs.TINY_SHAZEER_F32.replace(top_k=8, T=32)
    inp = moe_inputs.host_inputs(cfg)
    res = oracle.layer_forward(cfg, inp)
    u = inp["u"].astype(np.float64)
    lg = u @ inp["w_router"].astype(np.float64).T
    p = torch.softmax(torch.from_numpy(lg), dim=1).numpy()
    ex = np.stack([np.maximum(u @ inp["w_gu"][e].astype(np.float64).T, 0)
                   @ inp["w_down"][e].astype(np.float64).T for e in range(8)], 1)
    dense = np.einsum("te,ted->td", p, ex)
    np.testing.assert_allclose(res["out"], dense, rtol=2e-6, atol=2e-6)


def test_k_equals_one_is_single_expert():
    cfg = configs.TINY_SHAZEER_F32.replace(top_k=1, T=40)
    inp = moe_inputs.host_inputs(cfg)
    res = oracle.layer_forward(cfg, inp)
    np.testing.assert_array_equal(res["w"], np.ones((40, 1)))
    u = inp["u"].astype(np.float64)
    for t in range(40):
        e = int(np.argmax(u[t] @ inp["w_router"].astype(np.float64).T))
        assert res["idx"][t, 0] == e
        o = np.maximum(u[t] @ inp["w_gu"][e].astype(np.float64).T, 0) @ inp["w_down"][e].astype(
            np.float64).T
        np.testing.assert_allclose(res["out"][t], o, rtol=2e-6, atol=2e-6)


def test_weights_sum_to_one_and_combine_rms_bound():
    cfg = configs.small_muse(T=29)
    inp = moe_inputs.host_inputs(cfg)
    res = oracle.layer_forward(cfg, inp)
    np.testing.assert_allclose(res["w"].sum(1), 1.0, rtol=1e-14)
    # y is a convex combination of unit-RMS vectors, so rms(y) <= 1 (+ bf16 rounding slack)
    rms = np.sqrt(np.mean(res["y"] ** 2, 1))
    assert np.all(rms <= 1.0 + 2e-2)
    # slots are ordered by descending weight
    assert np.all(np.diff(res["w"], axis=1) <= 0)


def test_staged_driver_equals_full_forward():
    cfg = configs.small_muse(T=21, n=8, k=3)
    inp = moe_inputs.host_inputs(cfg)
    toks = np.array([0, 3, 4, 11, 20])
    full = oracle.layer_forward(cfg, inp, tokens=toks)

    def get_inputs(tokens):
        d = {k: v for k, v in inp.items() if k not in ("w_gu", "w_down")}
        d["u"] = inp["u"][tokens]
        return d

    staged = oracle.layer_forward_staged(cfg, toks, get_inputs,
                                         lambda e: (inp["w_gu"][e], inp["w_down"][e]))
    for key in ("out", "logits", "idx", "w", "y"):
        np.testing.assert_array_equal(full[key], staged[key])


def test_zipf_bias_imbalance_recipe():
    cfg = configs.MUSE_IMBALANCED
    r = moe_inputs.zipf_ranks(cfg)
    assert sorted(r.tolist()) == list(range(1, cfg.n_experts + 1))
    b = moe_inputs.zipf_bias(cfg, scale=1.0)
    np.testing.assert_allclose(b, -1.2 * np.log(r), rtol=1e-6)
    assert b.max() == 0.0


# ------------------------------------------------------------------ Muse sigmoid gate
# sigmoid(ln 3) = 3/4 and sigmoid(-ln 3) = 1/4 exactly, so these weights have closed forms.


def test_sigmoid_gate_closed_form():
    l = np.array([[0.0, math.log(3.0), -math.log(3.0)]])
    idx, w, s = oracle.sigmoid_topk(l, 2)
    np.testing.assert_allclose(s[0], [0.5, 0.75, 0.25], rtol=1e-15)
    assert idx[0].tolist() == [1, 0]
    np.testing.assert_allclose(w[0], [0.75 / 1.25, 0.5 / 1.25], rtol=1e-14)
    # the correction bias changes the selection, not the weights' source (the original scores)
    idx, w, _ = oracle.sigmoid_topk(l, 2, correction_bias=np.array([0.0, 0.0, 1.0]))
    assert idx[0].tolist() == [2, 1]
    np.testing.assert_allclose(w[0], [0.25, 0.75], rtol=1e-14)
    # routed_scaling_factor multiplies the renormalised weights
    _, w2, _ = oracle.sigmoid_topk(l, 2, routed_scale=2.5)
    np.testing.assert_allclose(w2[0], 2.5 * np.array([0.6, 0.4]), rtol=1e-14)


def test_sigmoid_gate_invariants():
    rng = np.random.default_rng(5)
    l = rng.normal(size=(40, 16)) * 3
    cb = rng.normal(size=16).astype(np.float32) * 0.5
    # k = n: every expert kept, weights are the scores over their sum, whatever the bias
    idx, w, s = oracle.sigmoid_topk(l, 16, correction_bias=cb)
    for r in range(40):
        np.testing.assert_allclose(w[r], s[r, idx[r]] / s[r].sum(), rtol=1e-13)
    # selection follows score + bias, weights sum to routed_scale
    idx, w, s = oracle.sigmoid_topk(l, 4, correction_bias=cb)
    for r in range(40):
        key = s[r] + cb.astype(np.float64)
        assert idx[r].tolist() == np.argsort(-key, kind="stable")[:4].tolist()
        assert abs(w[r].sum() - 1.0) < 1e-13
    # the 1e-15 in the denominator only matters for vanishing scores
    idx, w, s = oracle.sigmoid_topk(np.full((1, 8), -100.0), 2)
    np.testing.assert_allclose(w[0], s[0, idx[0]] / (2 * s[0, 0] + 1e-15), rtol=1e-12)
    assert w[0].sum() < 1e-20
    # the fp32 selection on fp32 scores agrees when keys are distinct
    sf = s.astype(np.float32)
    i32, _ = oracle.sigmoid_topk_scores_f32(oracle.sigmoid_topk(l, 4, cb)[2].astype(np.float32),
                                            4, cb)
    np.testing.assert_array_equal(i32, oracle.sigmoid_topk(l, 4, cb)[0])
    del sf
