"""Python access to the CPU oracle of the MoE-layer forward (``moe_oracle.c``).

TEST INFRASTRUCTURE: imported only by tests/, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg.  The product library never loads it, and it never loads the product library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "moe_oracle.c")
    hdr = os.path.join(_HERE, "moe_oracle.h")
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(src), os.path.getmtime(hdr))):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-Wall", "-Wextra", "-o", tmp, src, "-lpthread", "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class OrcCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("T", "d_model", "d_latent", "d_ff", "n_experts",
                                            "top_k", "is_bf16", "act", "pre_norm",
                                            "expert_norm", "resid_mode")] + \
               [(n, ctypes.c_double) for n in ("eps", "tau", "resid_floor", "routed_scale")] + \
               [("gate_mode", ctypes.c_int), ("router_f32", ctypes.c_int),
                ("logit_mult", ctypes.c_double), ("input_norm", ctypes.c_int),
                ("post_norm", ctypes.c_int), ("eps_block", ctypes.c_double)]


class OrcTensors(ctypes.Structure):
    _fields_ = [("u", ctypes.c_void_p), ("h", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("logit_bias", ctypes.c_void_p), ("p_down", ctypes.c_void_p),
                ("p_up", ctypes.c_void_p), ("w_gu", ctypes.POINTER(ctypes.c_void_p)),
                ("w_down", ctypes.POINTER(ctypes.c_void_p)), ("gamma_pre", ctypes.c_void_p),
                ("gamma_expert", ctypes.c_void_p), ("resid_g", ctypes.c_void_p),
                ("correction_bias", ctypes.c_void_p), ("gamma_in", ctypes.c_void_p),
                ("gamma_post", ctypes.c_void_p)]


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        cp = ctypes.POINTER(OrcCfg)
        tp = ctypes.POINTER(OrcTensors)
        L.orc_round.restype = dbl
        L.orc_round.argtypes = [cp, dbl]
        L.orc_rms_normalize.argtypes = [vp, i32, dbl, vp]
        L.orc_centered_rmsnorm.argtypes = [vp, vp, i32, dbl, vp]
        L.orc_input_scaled_rmsnorm.argtypes = [cp, vp, vp, i32, dbl, vp]
        L.orc_softmax_topk.argtypes = [vp, i32, i32, dbl, vp, vp]
        L.orc_softmax_topk_f32.argtypes = [vp, i32, i32, dbl, vp, vp]
        L.orc_resid_gate_coeffs.argtypes = [dbl, dbl, dbl, vp, vp]
        L.orc_router_token.argtypes = [cp, tp, ctypes.c_int64, vp, vp, vp]
        L.orc_expert_input_token.argtypes = [cp, tp, ctypes.c_int64, vp]
        L.orc_expert_token.argtypes = [cp, vp, vp, vp, vp, vp]
        L.orc_combine_token.argtypes = [cp, vp, vp, vp]
        L.orc_output_token.argtypes = [cp, tp, ctypes.c_int64, vp, vp]
        L.orc_layer_forward.argtypes = [cp, tp, vp, i32, vp, vp, vp, vp, vp, i32]
        L.orc_expert_batch.argtypes = [cp, vp, vp, vp, vp, i32, vp, i32]
        L.orc_router_batch.argtypes = [cp, tp, vp, i32, vp, vp, vp, i32]
        L.orc_expert_batch_parts.argtypes = [cp, vp, vp, vp, vp, i32, vp, vp, i32]
        L.orc_expert_batch_parts.restype = None
        L.orc_expert_token_scaled.argtypes = [cp, vp, vp, vp, vp, vp]
        L.orc_input_scaled_vector.argtypes = [cp, vp, vp, i32, vp]
        L.orc_permutation.restype = i32
        L.orc_permutation.argtypes = [i32, i32, i32, vp, vp, vp, vp]
        L.orc_sigmoid_topk.argtypes = [vp, vp, i32, i32, dbl, vp, vp, vp]
        L.orc_sigmoid_topk.restype = None
        L.orc_sigmoid_topk_scores_f32.argtypes = [vp, vp, i32, i32, dbl, vp, vp]
        L.orc_sigmoid_topk_scores_f32.restype = None
        for f in ("orc_rms_normalize", "orc_centered_rmsnorm", "orc_input_scaled_rmsnorm",
                  "orc_softmax_topk", "orc_softmax_topk_f32", "orc_resid_gate_coeffs",
                  "orc_router_token", "orc_expert_input_token", "orc_expert_token",
                  "orc_combine_token", "orc_output_token", "orc_layer_forward",
                  "orc_expert_batch", "orc_router_batch", "orc_expert_token_scaled",
                  "orc_input_scaled_vector"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def threads() -> int:
    return max(1, os.cpu_count() or 1)


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


def make_cfg(cfg, T: int | None = None) -> OrcCfg:
    """Oracle settings of a workload (an ``moe_inputs.configs.MoEConfig``)."""
    return OrcCfg(T=cfg.T if T is None else T, d_model=cfg.d_model, d_latent=cfg.d_latent,
                  d_ff=cfg.d_ff, n_experts=cfg.n_experts, top_k=cfg.top_k,
                  is_bf16=1 if cfg.dtype == "bf16" else 0, act=cfg.act, pre_norm=cfg.pre_norm,
                  expert_norm=cfg.expert_norm, resid_mode=cfg.resid_mode, eps=cfg.eps,
                  tau=cfg.tau, resid_floor=cfg.resid_floor, routed_scale=cfg.routed_scale,
                  gate_mode=cfg.gate_mode, router_f32=cfg.router_f32, logit_mult=cfg.logit_mult,
                  input_norm=cfg.input_norm, post_norm=cfg.post_norm, eps_block=cfg.eps_block)


class _Keep:
    """Holds numpy arrays alive while C holds pointers into them."""

    def __init__(self):
        self.refs = []

    def ptr(self, a):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        self.refs.append(a)
        return a.ctypes.data


def make_tensors(cfg, inp: dict, keep: _Keep, experts: dict | None = None) -> OrcTensors:
    """``inp`` holds host arrays named as in ``moe_inputs.tensor_specs`` (u may be a row subset
    when tokens are given relative to it).  ``experts`` optionally maps expert -> (w_gu_e,
    w_down_e) instead of the full ``inp['w_gu']`` / ``inp['w_down']``."""
    n = cfg.n_experts
    gu = (ctypes.c_void_p * n)()
    dn = (ctypes.c_void_p * n)()
    if experts is None:
        wg = np.ascontiguousarray(inp["w_gu"])
        wd = np.ascontiguousarray(inp["w_down"])
        keep.refs += [wg, wd]
        for e in range(n):
            gu[e] = wg[e].ctypes.data
            dn[e] = wd[e].ctypes.data
    else:
        for e, (a, b) in experts.items():
            gu[e] = keep.ptr(a)
            dn[e] = keep.ptr(b)
    keep.refs += [gu, dn]
    u = keep.ptr(inp["u"])
    h = keep.ptr(inp["h"]) if "h" in inp else u
    return OrcTensors(u=u, h=h, w_router=keep.ptr(inp["w_router"]),
                      logit_bias=keep.ptr(inp.get("logit_bias")), p_down=keep.ptr(inp.get("p_down")),
                      p_up=keep.ptr(inp.get("p_up")), w_gu=gu, w_down=dn,
                      gamma_pre=keep.ptr(inp.get("gamma_pre")),
                      gamma_expert=keep.ptr(inp.get("gamma_expert")),
                      resid_g=keep.ptr(inp.get("resid_g")),
                      correction_bias=keep.ptr(inp.get("correction_bias")),
                      gamma_in=keep.ptr(inp.get("gamma_in")),
                      gamma_post=keep.ptr(inp.get("gamma_post")))


def layer_forward(cfg, inp: dict, tokens=None, nthreads: int | None = None) -> dict:
    """The whole layer on the listed tokens (all tokens by default) with every tensor resident.
    Returns out [ntok, d] (float64 holding dtype-representable values), logits [ntok, n],
    idx [ntok, k] int32, w [ntok, k], y [ntok, E_in]."""
    tokens = np.arange(cfg.T, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    keep = _Keep()
    c = make_cfg(cfg)
    x = make_tensors(cfg, inp, keep)
    nt = len(tokens)
    E = cfg.expert_in
    out = np.zeros((nt, cfg.d_model))
    logits = np.zeros((nt, cfg.n_experts))
    idx = np.zeros((nt, cfg.top_k), dtype=np.int32)
    w = np.zeros((nt, cfg.top_k))
    y = np.zeros((nt, E))
    tk = np.ascontiguousarray(tokens)
    lib().orc_layer_forward(ctypes.byref(c), ctypes.byref(x), _p(tk), nt, _p(out), _p(logits),
                            _p(idx), _p(w), _p(y), nthreads or threads())
    return {"out": out, "logits": logits, "idx": idx, "w": w, "y": y, "tokens": tokens}


def layer_forward_staged(cfg, tokens, get_inputs, get_expert, nthreads: int | None = None,
                         want_s: bool = False) -> dict:
    """The same per-token arithmetic as ``layer_forward`` with expert weights held one expert at a
    time: route and build expert inputs for every listed token, evaluate each expert on the rows
    routed to it, then combine and project.  ``get_inputs(tokens)`` returns the non-expert
    tensors with ``u`` restricted to those tokens' rows; ``get_expert(e)`` returns
    (w_gu_e, w_down_e).  Besides the outputs of ``layer_forward`` it returns the expert inputs
    z [ntok, E_in] and, with want_s, each slot's expert output before its norm s [ntok, k, E_in]
    (the vector I_gamma reduces)."""
    tokens = np.asarray(tokens, np.int64)
    nt = len(tokens)
    L = lib()
    c = make_cfg(cfg, T=nt)
    keep = _Keep()
    inp = get_inputs(tokens)
    x = make_tensors(cfg, inp, keep, experts={})
    n, k, E, d = cfg.n_experts, cfg.top_k, cfg.expert_in, cfg.d_model
    logits = np.zeros((nt, n))
    idx = np.zeros((nt, k), dtype=np.int32)
    w = np.zeros((nt, k))
    z = np.zeros((nt, E))
    for i in range(nt):  # rows of the restricted u are the listed tokens, in order
        L.orc_router_token(ctypes.byref(c), ctypes.byref(x), i, _p(logits[i]), _p(idx[i]), _p(w[i]))
        L.orc_expert_input_token(ctypes.byref(c), ctypes.byref(x), i, _p(z[i]))
    ns = np.zeros((nt, k, E))
    ss = np.zeros((nt, k, E)) if want_s else None
    gamma = keep.ptr(inp.get("gamma_expert"))
    for e in np.unique(idx):
        rows = np.argwhere(idx == e)
        zr = np.ascontiguousarray(z[rows[:, 0]])
        nr = np.zeros_like(zr)
        sr = np.zeros_like(zr) if want_s else None
        wg, wd = get_expert(int(e))
        wg = np.ascontiguousarray(wg)
        wd = np.ascontiguousarray(wd)
        L.orc_expert_batch_parts(ctypes.byref(c), _p(wg), _p(wd), gamma, _p(zr), len(rows),
                                 _p(sr) if want_s else None, _p(nr), nthreads or threads())
        ns[rows[:, 0], rows[:, 1]] = nr
        if want_s:
            ss[rows[:, 0], rows[:, 1]] = sr
    y = np.zeros((nt, E))
    out = np.zeros((nt, d))
    for i in range(nt):
        nsi = np.ascontiguousarray(ns[i])
        wi = np.ascontiguousarray(w[i])
        L.orc_combine_token(ctypes.byref(c), _p(nsi), _p(wi), _p(y[i]))
        L.orc_output_token(ctypes.byref(c), ctypes.byref(x), i, _p(y[i]), _p(out[i]))
    return {"out": out, "logits": logits, "idx": idx, "w": w, "y": y, "z": z, "s": ss,
            "tokens": tokens}


def router(cfg, inp: dict, rows=None, nthreads: int | None = None) -> dict:
    """The router step on rows of ``inp['u']`` (all rows by default), threads over rows: logits
    [rows, n] (the sigmoid scores in that mode), idx [rows, k], w [rows, k].  Only the router's
    tensors need be in ``inp`` (u, w_router and, as the mode needs, logit_bias, correction_bias,
    gamma_in)."""
    nrow = inp["u"].shape[0]
    rows = np.arange(nrow, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    keep = _Keep()
    c = make_cfg(cfg, T=nrow)
    x = make_tensors(cfg, inp, keep, experts={})
    nt = len(rows)
    logits = np.zeros((nt, cfg.n_experts))
    idx = np.zeros((nt, cfg.top_k), dtype=np.int32)
    w = np.zeros((nt, cfg.top_k))
    rk = np.ascontiguousarray(rows)
    lib().orc_router_batch(ctypes.byref(c), ctypes.byref(x), _p(rk), nt, _p(logits), _p(idx),
                           _p(w), nthreads or threads())
    return {"logits": logits, "idx": idx, "w": w}


def expert_scaled(cfg, w_gu_e, w_down_e, gamma_expert, z):
    """One expert's output rows before its norm (the vector I_gamma reduces, or o without
    expert_norm), for input rows z [rows, E_in] (float64)."""
    z = np.ascontiguousarray(np.atleast_2d(z), np.float64)
    out = np.zeros_like(z)
    keep = _Keep()
    c = make_cfg(cfg)
    wg, wd = keep.ptr(w_gu_e), keep.ptr(w_down_e)
    g = keep.ptr(None if gamma_expert is None else np.asarray(gamma_expert, np.float32))
    for i in range(z.shape[0]):
        lib().orc_expert_token_scaled(ctypes.byref(c), wg, wd, g, _p(z[i]), _p(out[i]))
    return out


def input_scaled_vector(x, gamma, is_bf16=1):
    """D_gamma x = (1 + gamma) * x rounded to the storage dtype (is_bf16 as in bf16_round)."""
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(gamma, np.float64)
    out = np.zeros_like(x)
    c = OrcCfg(is_bf16=is_bf16)
    lib().orc_input_scaled_vector(ctypes.byref(c), _p(x), _p(g), x.size, _p(out))
    return out


def permutation(T: int, k: int, n: int, idx: np.ndarray):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    offsets = np.zeros(n + 1, dtype=np.int32)
    perm = np.zeros(T * k, dtype=np.int32)
    inv = np.zeros(T * k, dtype=np.int32)
    rc = lib().orc_permutation(T, k, n, _p(idx), _p(offsets), _p(perm), _p(inv))
    if rc != 0:
        raise ValueError("routing indices out of range or repeated within a token")
    return offsets, perm, inv


def softmax_topk(logits: np.ndarray, k: int, routed_scale: float = 1.0):
    """Oracle selection on a logit vector (float64 or float32 input)."""
    n = logits.shape[-1]
    f32 = logits.dtype == np.float32
    rows = np.ascontiguousarray(logits.reshape(-1, n))
    idx = np.zeros((rows.shape[0], k), dtype=np.int32)
    w = np.zeros((rows.shape[0], k))
    fn = lib().orc_softmax_topk_f32 if f32 else lib().orc_softmax_topk
    for i in range(rows.shape[0]):
        fn(_p(rows[i]), n, k, routed_scale, _p(idx[i]), _p(w[i]))
    return idx.reshape(logits.shape[:-1] + (k,)), w.reshape(logits.shape[:-1] + (k,))


def sigmoid_topk(logits: np.ndarray, k: int, correction_bias=None, routed_scale: float = 1.0):
    """Muse sigmoid gate on double logits: (idx, w, scores) per row."""
    n = logits.shape[-1]
    rows = np.ascontiguousarray(logits.reshape(-1, n), dtype=np.float64)
    cb = None if correction_bias is None else np.ascontiguousarray(correction_bias, np.float32)
    idx = np.zeros((rows.shape[0], k), dtype=np.int32)
    w = np.zeros((rows.shape[0], k))
    s = np.zeros_like(rows)
    for i in range(rows.shape[0]):
        lib().orc_sigmoid_topk(_p(rows[i]), None if cb is None else _p(cb), n, k, routed_scale,
                               _p(idx[i]), _p(w[i]), _p(s[i]))
    return idx, w, s


def sigmoid_topk_scores_f32(scores: np.ndarray, k: int, correction_bias=None,
                            routed_scale: float = 1.0):
    """Selection of the sigmoid gate taken in fp32 on given fp32 scores: (idx, w) per row."""
    n = scores.shape[-1]
    rows = np.ascontiguousarray(scores.reshape(-1, n), dtype=np.float32)
    cb = None if correction_bias is None else np.ascontiguousarray(correction_bias, np.float32)
    idx = np.zeros((rows.shape[0], k), dtype=np.int32)
    w = np.zeros((rows.shape[0], k))
    for i in range(rows.shape[0]):
        lib().orc_sigmoid_topk_scores_f32(_p(rows[i]), None if cb is None else _p(cb), n, k,
                                          routed_scale, _p(idx[i]), _p(w[i]))
    return idx, w


def noisy_gate(l: np.ndarray, m: np.ndarray, eps: np.ndarray, k: int):
    """Noisy top-k gate per row of [rows, n] clean logits l, noise logits m and draws eps:
    returns H, G (dense), P (smooth load probabilities) and idx [rows, k]."""
    L = lib()
    if not hasattr(L, "_noisy_sig"):
        L.orc_noisy_gate_token.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 2 + \
            [ctypes.c_void_p] * 4
        L.orc_noisy_gate_token.restype = None
        L.orc_cv_squared.argtypes = [ctypes.c_void_p, ctypes.c_int]
        L.orc_cv_squared.restype = ctypes.c_double
        L._noisy_sig = True
    rows, n = l.shape
    l = np.ascontiguousarray(l, np.float64)
    m = np.ascontiguousarray(m, np.float64)
    eps = np.ascontiguousarray(eps, np.float64)
    H, G, P = np.zeros_like(l), np.zeros_like(l), np.zeros_like(l)
    idx = np.zeros((rows, k), dtype=np.int32)
    for r in range(rows):
        L.orc_noisy_gate_token(_p(l[r]), _p(m[r]), _p(eps[r]), n, k, _p(H[r]), _p(G[r]), _p(P[r]),
                               _p(idx[r]))
    return H, G, P, idx


def cv_squared(v) -> float:
    noisy_gate(np.zeros((1, 2)), np.zeros((1, 2)), np.zeros((1, 2)), 1)  # binds the signatures
    v = np.ascontiguousarray(v, np.float64)
    return float(lib().orc_cv_squared(_p(v), v.size))


def rms_normalize(x, eps=0.0):
    x = np.ascontiguousarray(x, np.float64)
    out = np.zeros_like(x)
    lib().orc_rms_normalize(_p(x), x.size, eps, _p(out))
    return out


def centered_rmsnorm(x, gamma, eps=0.0):
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(gamma, np.float64)
    out = np.zeros_like(x)
    lib().orc_centered_rmsnorm(_p(x), _p(g), x.size, eps, _p(out))
    return out


def input_scaled_rmsnorm(x, gamma, eps=0.0, is_bf16=2):
    """I_gamma on a float64 vector; is_bf16 = 1 rounds D_gamma x to bf16, 0 to fp32, 2 not at all."""
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(gamma, np.float64)
    out = np.zeros_like(x)
    c = OrcCfg(is_bf16=is_bf16)
    lib().orc_input_scaled_rmsnorm(ctypes.byref(c), _p(x), _p(g), x.size, eps, _p(out))
    return out


def resid_gate_coeffs(g: float, tau: float = 0.3, floor_: float = 1e-3):
    a = ctypes.c_double()
    b = ctypes.c_double()
    lib().orc_resid_gate_coeffs(g, tau, floor_, ctypes.byref(a), ctypes.byref(b))
    return a.value, b.value


def bf16_round(x, is_bf16=1):
    c = OrcCfg(is_bf16=is_bf16)
    f = lib().orc_round
    return np.array([f(ctypes.byref(c), float(v)) for v in np.ravel(x)]).reshape(np.shape(x))
