"""Helpers shared by the GPU parity tests, the smoke check and the benchmark.

Inputs come from the seeded generator only (device copies generated on the device, host copies
on the host, bit-identical).  Expected values come from the CPU oracle only.  The CUDA path is
called through the C ABI (the ctypes binding of libmoe.so).
"""
from __future__ import annotations

import numpy as np

import moe_inputs
import sparse_moe_layer_softmax_b200 as moe
from moe_inputs import configs

BF16_TOL = 2e-2   # max over tokens of |out - ref|_inf / |ref|_inf, bf16 storage
F32_TOL = 1e-4    # same for fp32 storage


def abi_config(cfg, T: int | None = None):
    return moe.make_config(
        T=cfg.T if T is None else T, d_model=cfg.d_model, n_experts=cfg.n_experts,
        top_k=cfg.top_k, d_ff=cfg.d_ff, d_latent=cfg.d_latent,
        dtype=moe.MOE_BF16 if cfg.dtype == "bf16" else moe.MOE_F32, expert_act=cfg.act,
        pre_norm=cfg.pre_norm, expert_norm=cfg.expert_norm, resid_mode=cfg.resid_mode,
        eps=cfg.eps, tau=cfg.tau, resid_floor=cfg.resid_floor, routed_scale=cfg.routed_scale,
        gate_mode=cfg.gate_mode, router_f32=cfg.router_f32, logit_mult=cfg.logit_mult,
        input_norm=cfg.input_norm, post_norm=cfg.post_norm, eps_block=cfg.eps_block)


def host_values(a: np.ndarray, dtype: str) -> np.ndarray:
    """float64 values of host tensors (bf16 codes or float32)."""
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def device_values(t) -> np.ndarray:
    """float64 values of a CUDA tensor (bf16 or fp32)."""
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def row_rel_err(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per-row |got - ref|_inf / |ref|_inf."""
    num = np.max(np.abs(got - ref), axis=-1)
    den = np.maximum(np.max(np.abs(ref), axis=-1), 1e-30)
    return num / den


def tolerance(cfg) -> float:
    return BF16_TOL if cfg.dtype == "bf16" else F32_TOL


def logit_atol(cfg, logits: np.ndarray) -> float:
    """Absolute tolerance of fp32-accumulated router logits against double: the products of two
    bf16 (or fp32-rounded) values are summed in fp32 over K = d_model terms; rounding errors of
    a K-term sum grow like sqrt(K) * 2^-24 * |partial sums|, so allow 16 sqrt(K) 2^-24 times the
    largest logit magnitude (at least 1).  fp32 router weights are summed as three bf16 parts
    (K = 3 d_model); the sigmoid gate's scores move by at most a quarter of the logit error times
    the output multiplier, so the same bound scaled by the multiplier covers them."""
    K = cfg.d_model * (3 if cfg.router_f32 and cfg.dtype == "bf16" else 1)
    mult = max(1.0, abs(cfg.logit_mult)) if cfg.gate_mode == configs.GATE_SIGMOID else 1.0
    tol = 16.0 * np.sqrt(K) * 2.0 ** -24 * mult * max(1.0, float(np.abs(logits).max()))
    if cfg.input_norm:
        # the router input is itself a bf16-rounded norm: fp32 (GPU) and double (oracle) may
        # round an element of u to neighbouring bf16 values; allow two such flips per row, each
        # moving the logit by at most |w|max * ulp(|u|max) with |u| < 6 (unit-RMS rows) and
        # |w| <= 4.9 sigma (the generator's Irwin-Hall bound)
        tol += mult * 2 * (6.0 * 2.0 ** -7) * 4.9 * cfg.sigma_router()
    return tol


def run_layer(cfg, dev: dict, want_logits: bool = True, want_taps: bool = False):
    """moe_layer_forward through the C ABI on device inputs; returns torch tensors.  With
    want_taps, moe_layer_forward_taps: the result also holds the intermediates z [T, E_in],
    s [T*k, E_in] (dispatch order), y [T, E_in] under "taps" and the dispatch rows under "inv"
    ([T, k])."""
    import torch
    c = abi_config(cfg)
    layer = moe.MoELayer(c, dev)
    u = dev["u"]
    out = torch.empty_like(u)
    logits = torch.empty((cfg.T, cfg.n_experts), dtype=torch.float32, device="cuda") \
        if want_logits else None
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device="cuda")
    taps = None
    if want_taps:
        E, TK = cfg.expert_in, cfg.T * cfg.top_k
        taps = {"z": torch.empty((cfg.T, E), dtype=u.dtype, device="cuda"),
                "s": torch.empty((TK, E), dtype=u.dtype, device="cuda"),
                "y": torch.empty((cfg.T, E), dtype=u.dtype, device="cuda"),
                "inv_perm": torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device="cuda")}
    layer.forward(u, u, out=out, logits_out=logits, topk_idx_out=idx, topk_w_out=w, taps=taps)
    status = moe.moe_get_device_status()
    assert status == 0, f"device status {moe.STATUS.get(status, status)}"
    res = {"out": out, "logits": logits, "idx": idx, "w": w, "layer": layer}
    if taps is not None:
        res["taps"] = taps
        res["inv"] = taps["inv_perm"]
    return res


def oracle_reference(cfg, tokens=None, want_s: bool = False):
    """Oracle layer outputs for the listed tokens (all by default).  Small workloads hold every
    tensor on the host; large ones evaluate one expert's weights at a time.  With want_s the
    staged evaluation is used at every size, and the result also holds the expert inputs z and
    each slot's pre-norm expert output s."""
    import oracle
    big = cfg.n_experts * cfg.gu_rows * cfg.expert_in > 64 * 1024 * 1024
    if not big and not want_s:
        inp = moe_inputs.host_inputs(cfg)
        return oracle.layer_forward(cfg, inp, tokens=tokens)
    tokens = np.arange(cfg.T) if tokens is None else np.asarray(tokens)

    def get_inputs(tk):
        d = {"u": moe_inputs.host_rows(cfg, "u", rows=tk)}
        for name in moe_inputs.tensor_specs(cfg):
            if name not in ("u", "w_gu", "w_down"):
                d[name] = moe_inputs.host_rows(cfg, name)
        if cfg.zipf_bias:
            d["logit_bias"] = moe_inputs.zipf_bias(cfg)
        return d

    def get_expert(e):
        return (moe_inputs.host_rows(cfg, "w_gu", lead=e), moe_inputs.host_rows(cfg, "w_down", lead=e))

    return oracle.layer_forward_staged(cfg, tokens, get_inputs, get_expert, want_s=want_s)


def correction_bias(cfg):
    """Host copy of the sigmoid gate's selection-only bias (None for the softmax gate)."""
    if cfg.gate_mode != configs.GATE_SIGMOID:
        return None
    return moe_inputs.host_rows(cfg, "correction_bias")


def selection_keys(cfg, logits: np.ndarray) -> np.ndarray:
    """What the top-k is taken on: the logits (softmax gate) or the scores + correction bias."""
    cb = correction_bias(cfg)
    return logits if cb is None else logits + cb.astype(np.float64)


def check_routing(cfg, logits_gpu: np.ndarray, idx_gpu: np.ndarray, w_gpu: np.ndarray):
    """Bit-exact routing on every token: the oracle's selection run on the GPU's fp32 logits (or
    sigmoid scores, with the selection key formed by one fp32 addition of the correction bias)
    must equal the GPU's indices; weights within 1e-6 relative."""
    import oracle
    if cfg.gate_mode == configs.GATE_SIGMOID:
        sel, wref = oracle.sigmoid_topk_scores_f32(logits_gpu.astype(np.float32), cfg.top_k,
                                                   correction_bias(cfg), cfg.routed_scale)
    else:
        sel, wref = oracle.softmax_topk(logits_gpu.astype(np.float32), cfg.top_k,
                                        cfg.routed_scale)
    np.testing.assert_array_equal(idx_gpu, sel)
    np.testing.assert_allclose(w_gpu, wref, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(w_gpu.sum(1), cfg.routed_scale, rtol=2e-6)


def order_tie_tokens(logits_ref: np.ndarray, k: int, rel: float = 1e-4) -> np.ndarray:
    """Tokens with two of their k selected oracle logits closer than rel * rms(logits): the set
    of selected experts is unique but their slot order is not (fp32 and double may differ)."""
    s = -np.sort(-logits_ref, axis=1)[:, :k]
    if k < 2:
        return np.zeros(len(logits_ref), dtype=bool)
    gaps = np.min(s[:, :-1] - s[:, 1:], axis=1)
    rms = np.sqrt(np.mean(logits_ref ** 2, axis=1))
    return gaps < rel * rms


def compare_selection(idx_gpu: np.ndarray, ref_logits: np.ndarray, ref_idx: np.ndarray, k: int):
    """GPU selection vs the oracle's (double-logit) selection, comparing what is unique: tokens
    with a near tie at the k-th place are skipped (their selected set is not unique), tokens with
    a near tie inside the selection are compared as sets.  Returns the boundary-tie mask."""
    ties = near_tie_tokens(ref_logits, k)
    ot = order_tie_tokens(ref_logits, k) & ~ties
    exact = ~ties & ~ot
    np.testing.assert_array_equal(idx_gpu[exact], ref_idx[exact])
    np.testing.assert_array_equal(np.sort(idx_gpu[ot], axis=1), np.sort(ref_idx[ot], axis=1))
    return ties


def separate(cfg):
    """`cfg` with its router inputs separated at the top-k boundary: a named workload keeps its
    stored redraw list; any other configuration gets one computed here with the oracle's router
    (tests/golden/separate_router_logits.py)."""
    if cfg.name in configs.SEPARATED_NAMES and cfg == configs.ALL_CONFIGS.get(cfg.name):
        return cfg
    import importlib.util
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "separate_router_logits.py")
    spec = importlib.util.spec_from_file_location("separate_router_logits", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    red, _ = mod.redraws_for(cfg)
    return cfg.replace(u_redraw=red)


def key_margins(keys: np.ndarray, k: int) -> np.ndarray:
    """k-th minus (k+1)-th largest key per row, over the rms of the row's keys (+inf if k = n)."""
    n = keys.shape[1]
    if k >= n:
        return np.full(len(keys), np.inf)
    s = -np.sort(-keys, axis=1)
    rms = np.sqrt(np.mean(keys.astype(np.float64) ** 2, axis=1))
    return (s[:, k - 1] - s[:, k]) / rms


def near_tie_tokens(logits_ref: np.ndarray, k: int, rel: float = 1e-4) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest oracle logits are closer than rel * rms(logits):
    fp32 and double accumulation may order them differently, so their selection is not unique."""
    n = logits_ref.shape[1]
    if k >= n:
        return np.zeros(len(logits_ref), dtype=bool)
    s = -np.sort(-logits_ref, axis=1)
    margin = s[:, k - 1] - s[:, k]
    rms = np.sqrt(np.mean(logits_ref ** 2, axis=1))
    return margin < rel * rms
