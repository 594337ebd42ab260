"""Seeded synthetic inputs for the MoE-layer forward (shared by the oracle tests, the GPU tests
and the benchmark).

The per-element formulas live in ``gen_core.h``; ``gen_host.c`` and ``gen_cuda.cu`` implement
them bit-identically on the CPU and on the GPU.  Nothing here computes any part of the layer.
"""
from __future__ import annotations

import ctypes
import functools
import math
import os
import subprocess

import numpy as np

from . import configs
from .configs import MoEConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoegen.so")
_SOURCES = ("gen_core.h", "gen_host.c", "gen_cuda.cu")
_lib = None


def build(force: bool = False) -> str:
    """Compile libmoegen.so (host C + CUDA sm_100a) in place."""
    srcs = [os.path.join(_HERE, s) for s in _SOURCES]
    if (not force and os.path.exists(_LIB_PATH)
            and all(os.path.getmtime(_LIB_PATH) >= os.path.getmtime(s) for s in srcs)):
        return _LIB_PATH
    bdir = os.path.join(_HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    host_o = os.path.join(bdir, "gen_host.o")
    cuda_o = os.path.join(bdir, "gen_cuda.o")
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-Wall", "-c", srcs[1], "-o", host_o])
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                           "-Xcompiler", "-fPIC", "-c", srcs[2], "-o", cuda_o])
    tmp = _LIB_PATH + ".tmp"
    subprocess.check_call(["nvcc", "-shared", "-o", tmp, host_o, cuda_o, "-lpthread"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, sz, f32, vp, i32 = (ctypes.c_uint64, ctypes.c_size_t, ctypes.c_float,
                                 ctypes.c_void_p, ctypes.c_int)
        L.gen_stream_key.restype = u64
        L.gen_stream_key.argtypes = [u64, u64]
        L.gen_normal_scale.restype = f32
        L.gen_normal_scale.argtypes = [ctypes.c_double]
        L.gen_draw_u64.restype = u64
        L.gen_draw_u64.argtypes = [u64, u64]
        for name in ("gen_normal_bf16_host", "gen_normal_f32_host"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [u64, u64, sz, f32, vp, i32]
        L.gen_uniform_f32_host.restype = None
        L.gen_uniform_f32_host.argtypes = [u64, u64, sz, vp, i32]
        for name in ("gen_normal_bf16_cuda", "gen_normal_f32_cuda"):
            getattr(L, name).restype = i32
            getattr(L, name).argtypes = [u64, u64, sz, f32, vp, vp]
        L.gen_uniform_f32_cuda.restype = i32
        L.gen_uniform_f32_cuda.argtypes = [u64, u64, sz, vp, vp]
        _lib = L
    return _lib


def host_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def key(seed: int, stream: int) -> int:
    return int(lib().gen_stream_key(seed, stream))


def draw_u64(k: int, i: int) -> int:
    return int(lib().gen_draw_u64(k, i))


def normal_host(seed: int, stream: int, first: int, count: int, sigma: float, dtype: str):
    """Elements [first, first+count) of a N(0, sigma^2) stream: uint16 bf16 codes or float32."""
    k = key(seed, stream)
    scale = lib().gen_normal_scale(sigma)
    if dtype == "bf16":
        out = np.empty(count, dtype=np.uint16)
        lib().gen_normal_bf16_host(k, first, count, scale, out.ctypes.data, host_threads())
    else:
        out = np.empty(count, dtype=np.float32)
        lib().gen_normal_f32_host(k, first, count, scale, out.ctypes.data, host_threads())
    return out


def uniform_host(seed: int, stream: int, first: int, count: int):
    out = np.empty(count, dtype=np.float32)
    lib().gen_uniform_f32_host(key(seed, stream), first, count, out.ctypes.data, host_threads())
    return out


def normal_device(t, seed: int, stream: int, first: int, sigma: float, stream_ptr: int = 0):
    """Fill a contiguous CUDA tensor (torch.uint16/bfloat16 or float32) from a normal stream."""
    k = key(seed, stream)
    scale = lib().gen_normal_scale(sigma)
    n = t.numel()
    if t.element_size() == 2:
        rc = lib().gen_normal_bf16_cuda(k, first, n, scale, t.data_ptr(), stream_ptr)
    else:
        rc = lib().gen_normal_f32_cuda(k, first, n, scale, t.data_ptr(), stream_ptr)
    if rc != 0:
        raise RuntimeError(f"input generator kernel failed with CUDA error {rc}")


def uniform_device(t, seed: int, stream: int, first: int, stream_ptr: int = 0):
    rc = lib().gen_uniform_f32_cuda(key(seed, stream), first, t.numel(), t.data_ptr(), stream_ptr)
    if rc != 0:
        raise RuntimeError(f"input generator kernel failed with CUDA error {rc}")


# ---------------------------------------------------------------------------------------------
# Derived integer recipes (permutations, sample choices, the Zipf router bias)
# ---------------------------------------------------------------------------------------------

def fisher_yates(seed: int, stream: int, n: int, m: int | None = None) -> np.ndarray:
    """First m entries of a Fisher-Yates shuffle of range(n) driven by the counter stream."""
    m = n if m is None else m
    k = key(seed, stream)
    a = np.arange(n, dtype=np.int64)
    for i in range(min(m, n - 1)):
        j = i + draw_u64(k, i) % (n - i)
        a[i], a[j] = a[j], a[i]
    return a[:m].copy()


def subsample_tokens(cfg: MoEConfig, count: int = 512) -> np.ndarray:
    """Seeded sample of distinct token indices (sorted) for oracle checks of large workloads."""
    if count >= cfg.T:
        return np.arange(cfg.T, dtype=np.int64)
    return np.sort(fisher_yates(cfg.seed, configs.STREAM_SUBSAMPLE, cfg.T, count))


def zipf_ranks(cfg: MoEConfig) -> np.ndarray:
    """rank_e in 1..n: a seeded random assignment of Zipf ranks to experts."""
    order = fisher_yates(cfg.seed, configs.STREAM_ZIPF, cfg.n_experts)
    ranks = np.empty(cfg.n_experts, dtype=np.int64)
    ranks[order] = np.arange(1, cfg.n_experts + 1)
    return ranks


def zipf_bias(cfg: MoEConfig, scale: float | None = None) -> np.ndarray:
    """Per-expert router logit bias  -c * s * ln(rank_e)  (float32)."""
    c = configs.ZIPF_BIAS_SCALE if scale is None else scale
    r = zipf_ranks(cfg).astype(np.float64)
    return (-c * configs.ZIPF_S * np.log(r)).astype(np.float32)


# ---------------------------------------------------------------------------------------------
# Whole tensors of a workload
# ---------------------------------------------------------------------------------------------

def tensor_specs(cfg: MoEConfig):
    """name -> (shape, stream, kind, sigma) with kind in {"act", "w", "f32n", "f32u"}."""
    n, d, L, I = cfg.n_experts, cfg.d_model, cfg.d_latent, cfg.d_ff
    specs = {
        "u": ((cfg.T, d), configs.STREAM_X, "act", cfg.x_sigma),
        "w_router": ((n, d), configs.STREAM_W_ROUTER, "f32n" if cfg.router_f32 else "w",
                     cfg.sigma_router()),
        "w_gu": ((n, cfg.gu_rows, cfg.expert_in), configs.STREAM_W_GU, "w", cfg.sigma_w_gu()),
        "w_down": ((n, cfg.expert_in, I), configs.STREAM_W_DOWN, "w", cfg.sigma_w_down()),
    }
    if cfg.latent:
        specs["p_down"] = ((L, d), configs.STREAM_P_DOWN, "w", cfg.sigma_p_down())
        specs["p_up"] = ((d, L), configs.STREAM_P_UP, "w", cfg.sigma_p_up())
    if cfg.pre_norm:
        specs["gamma_pre"] = ((L,), configs.STREAM_GAMMA_PRE, "f32n", cfg.gamma_sigma)
    if cfg.expert_norm:
        specs["gamma_expert"] = ((cfg.expert_in,), configs.STREAM_GAMMA_EXPERT, "f32n",
                                 cfg.gamma_sigma)
    if cfg.gate_mode == configs.GATE_SIGMOID:
        specs["correction_bias"] = ((n,), configs.STREAM_CORR_BIAS, "f32n", cfg.corr_sigma)
    if cfg.noisy_gate:
        specs["w_noise"] = ((n, d), configs.STREAM_W_NOISE, "f32n" if cfg.router_f32 else "w",
                            cfg.sigma_router())
        specs["noise_eps"] = ((cfg.T, n), configs.STREAM_NOISE_EPS, "f32n", 1.0)
    if cfg.input_norm:
        specs["gamma_in"] = ((d,), configs.STREAM_GAMMA_IN, "f32n", cfg.gamma_sigma)
    if cfg.post_norm:
        specs["gamma_post"] = ((d,), configs.STREAM_GAMMA_POST, "f32n", cfg.gamma_sigma)
    if cfg.resid_mode != configs.RESID_NONE:
        specs["resid_g"] = ((d,), configs.STREAM_RESID_G, "f32u", 0.0)
    return specs


@functools.lru_cache(maxsize=64)
def _redraw_map(redraws: tuple) -> dict:
    return dict(redraws)


def u_row_first(cfg: MoEConfig, row: int) -> int:
    """Counter index of the first element of row ``row`` of u (its latest redraw, if any)."""
    g = _redraw_map(cfg.u_redraw).get(int(row), 0)
    return (g * cfg.T + int(row)) * cfg.d_model


def host_rows(cfg: MoEConfig, name: str, rows=None, lead: int | None = None) -> np.ndarray:
    """A generated tensor on the host.  ``rows`` selects rows of a 2-D tensor (e.g. sampled
    tokens of u); ``lead`` selects one leading slice of a 3-D tensor (one expert's weights).
    Rows of u listed in the workload's redraw list come from their redraw."""
    shape, stream, kind, sigma = tensor_specs(cfg)[name]
    if name == "u":
        dt = cfg.dtype
        width = shape[-1]
        if rows is None:
            full = normal_host(cfg.seed, stream, 0, math.prod(shape), sigma, dt).reshape(shape)
            for t, _ in cfg.u_redraw:
                full[t] = normal_host(cfg.seed, stream, u_row_first(cfg, t), width, sigma, dt)
            return full
        out = [normal_host(cfg.seed, stream, u_row_first(cfg, r), width, sigma, dt) for r in rows]
        return np.stack(out) if out else np.empty((0, width), dtype=np.uint16 if dt == "bf16"
                                                   else np.float32)
    if kind == "f32n":
        return normal_host(cfg.seed, stream, 0, math.prod(shape), sigma, "f32").reshape(shape)
    if kind == "f32u":
        return uniform_host(cfg.seed, stream, 0, math.prod(shape)).reshape(shape)
    dt = cfg.dtype
    if lead is not None:
        per = shape[1] * shape[2]
        return normal_host(cfg.seed, stream, lead * per, per, sigma, dt).reshape(shape[1:])
    if rows is not None:
        width = shape[-1]
        out = [normal_host(cfg.seed, stream, int(r) * width, width, sigma, dt) for r in rows]
        return np.stack(out) if out else np.empty((0, width), dtype=np.uint16 if dt == "bf16"
                                                   else np.float32)
    return normal_host(cfg.seed, stream, 0, math.prod(shape), sigma, dt).reshape(shape)


def host_inputs(cfg: MoEConfig) -> dict:
    """Every input of a (small) workload as host arrays."""
    out = {name: host_rows(cfg, name) for name in tensor_specs(cfg)}
    if cfg.zipf_bias:
        out["logit_bias"] = zipf_bias(cfg)
    return out


def device_inputs(cfg: MoEConfig, device="cuda") -> dict:
    """Every input of a workload as CUDA tensors, generated on the device (bit-identical to
    ``host_inputs``).  bf16 tensors are torch.bfloat16; fp32 ones torch.float32."""
    import torch
    out = {}
    for name, (shape, stream, kind, sigma) in tensor_specs(cfg).items():
        if kind == "f32u":
            t = torch.empty(shape, dtype=torch.float32, device=device)
            uniform_device(t, cfg.seed, stream, 0)
        else:
            is_bf16 = kind in ("act", "w") and cfg.dtype == "bf16"
            t = torch.empty(shape, dtype=torch.bfloat16 if is_bf16 else torch.float32,
                            device=device)
            normal_device(t, cfg.seed, stream, 0, sigma)
            if name == "u":
                for row, _ in cfg.u_redraw:
                    normal_device(t[row], cfg.seed, stream, u_row_first(cfg, row), sigma)
        out[name] = t
    if cfg.zipf_bias:
        out["logit_bias"] = torch.from_numpy(zipf_bias(cfg)).to(device)
    torch.cuda.synchronize()
    return out
