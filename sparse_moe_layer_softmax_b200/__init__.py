"""Python binding of libmoe.so, the sm_100a forward pass of a top-k softmax-routed (latent)
mixture-of-experts layer.

The binding only marshals arguments: every step of the layer runs in the library's CUDA kernels.
PyTorch is used for device memory and streams.  There is no fallback: if libmoe.so is missing or
cannot be loaded, importing ``lib()`` raises.

C entry points (same names as in include/moe.h): moe_route, moe_permute, moe_expert_ffn,
moe_combine, moe_latent_down, moe_latent_up, moe_layer_forward, moe_workspace_size,
moe_get_device_status, moe_status_string.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
MOE_ACT_RELU, MOE_ACT_SWIGLU = 0, 1
MOE_RESID_NONE, MOE_RESID_MUSE_GATE, MOE_RESID_LITERAL = 0, 1, 2
MOE_GATE_SOFTMAX, MOE_GATE_SIGMOID = 0, 1
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_ALIGNMENT",
          4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_TIMEOUT",
          7: "MOE_ERR_DEVICE_CHECK"}
STATUS_CODES = {v: k for k, v in STATUS.items()}
EXPORTS = ("moe_status_string", "moe_workspace_size", "moe_route", "moe_permute",
           "moe_expert_ffn", "moe_combine", "moe_latent_down", "moe_latent_up",
           "moe_layer_forward", "moe_get_device_status", "moe_profile_begin", "moe_profile_end",
           "moe_launch_count", "moe_permute_static", "moe_selftest_wait_timeout",
           "moe_router_split_weights", "moe_residual_update", "moe_noisy_gate",
           "moe_noisy_gate_workspace_size", "moe_host_staging_size", "moe_layer_forward_host",
           "moe_row_sumsq_parts", "moe_gather_rows", "moe_layer_forward_taps",
           "moe_dispatch_rows")
PROFILE_STAGES = ("route", "latent_down", "dispatch", "expert_gate_up", "expert_down", "combine",
                  "latent_up_resgate")


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class Config(ctypes.Structure):
    """moe_config_t"""
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "d_model", "d_latent", "d_ff", "n_experts",
                                              "top_k", "dtype", "expert_act", "pre_norm",
                                              "expert_norm", "resid_mode")] + \
               [(n, ctypes.c_float) for n in ("eps", "tau", "resid_floor", "routed_scale")] + \
               [("gate_mode", ctypes.c_int32), ("router_f32", ctypes.c_int32),
                ("logit_mult", ctypes.c_float), ("input_norm", ctypes.c_int32),
                ("post_norm", ctypes.c_int32), ("eps_block", ctypes.c_float)]


class Taps(ctypes.Structure):
    """moe_layer_taps_t"""
    _fields_ = [(n, ctypes.c_void_p) for n in ("z", "s", "y", "inv_perm")]


class Weights(ctypes.Structure):
    """moe_weights_t"""
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_router", "p_down", "p_up", "w_gu", "w_down",
                                               "gamma_pre", "gamma_expert", "resid_g",
                                               "logit_bias", "correction_bias", "gamma_in",
                                               "gamma_post")]


_lib = None


def lib():
    """The loaded libmoe.so (built in place by ``build.build()``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so not built ({LIB_PATH}); run "
                              "python sparse_moe_layer_softmax_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        cp, wp = ctypes.POINTER(Config), ctypes.POINTER(Weights)
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [i32]
        sigs = {
            "moe_workspace_size": [cp, ctypes.POINTER(sz)],
            "moe_route": [cp, vp, vp, vp, vp, vp, vp, vp, vp],
            "moe_router_split_weights": [vp, ctypes.c_int32, ctypes.c_int32, vp, vp],
            "moe_residual_update": [cp, vp, vp, vp, vp, vp, vp],
            "moe_noisy_gate_workspace_size": [cp, ctypes.POINTER(sz)],
            "moe_noisy_gate": [cp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_permute": [cp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_expert_ffn": [cp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_combine": [cp, vp, vp, vp, vp, vp, vp],
            "moe_row_sumsq_parts": [cp, ctypes.POINTER(ctypes.c_int32)],
            "moe_gather_rows": [vp, ctypes.c_int64, vp, ctypes.c_int64, ctypes.c_int64, vp, vp],
            "moe_latent_down": [cp, vp, vp, vp, vp],
            "moe_latent_up": [cp, vp, vp, vp, vp, vp, vp],
            "moe_layer_forward": [cp, wp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_layer_forward_taps": [cp, wp, vp, vp, vp, vp, vp, vp,
                                       ctypes.POINTER(Taps), vp, sz, vp],
            "moe_host_staging_size": [cp, ctypes.POINTER(ctypes.c_size_t)],
            "moe_layer_forward_host": [cp, wp, ctypes.c_int32, ctypes.POINTER(vp),
                                       ctypes.POINTER(vp), vp, sz, vp, sz, vp],
            "moe_get_device_status": [vp],
            "moe_profile_begin": [ctypes.c_int32],
            "moe_profile_end": [vp, vp],
            "moe_permute_static": [cp, vp, vp, vp, vp, vp, vp, vp, vp],
            "moe_dispatch_rows": [cp, vp, vp, vp, vp, vp],
            "moe_selftest_wait_timeout": [ctypes.c_longlong, vp, vp],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.restype = i32
            f.argtypes = args
        L.moe_launch_count.restype = ctypes.c_ulonglong
        L.moe_launch_count.argtypes = []
        _lib = L
    return _lib


def make_config(T, d_model, n_experts, top_k, d_ff, d_latent=0, dtype=MOE_BF16,
                expert_act=MOE_ACT_SWIGLU, pre_norm=0, expert_norm=0, resid_mode=MOE_RESID_NONE,
                eps=1e-6, tau=0.3, resid_floor=1e-3, routed_scale=1.0, gate_mode=MOE_GATE_SOFTMAX,
                router_f32=0, logit_mult=1.0, input_norm=0, post_norm=0,
                eps_block=1e-5) -> Config:
    return Config(T=T, d_model=d_model, d_latent=d_latent, d_ff=d_ff, n_experts=n_experts,
                  top_k=top_k, dtype=dtype, expert_act=expert_act, pre_norm=pre_norm,
                  expert_norm=expert_norm, resid_mode=resid_mode, eps=eps, tau=tau,
                  resid_floor=resid_floor, routed_scale=routed_scale, gate_mode=gate_mode,
                  router_f32=router_f32, logit_mult=logit_mult, input_norm=input_norm,
                  post_norm=post_norm, eps_block=eps_block)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(name: str, code: int):
    if code != 0:
        raise MoeError(name, code)


def workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t()
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_route(cfg, u, w_router, logit_bias, logits_out, topk_idx, topk_w, stream=None,
              correction_bias=None):
    _check("moe_route", lib().moe_route(ctypes.byref(cfg), _ptr(u), _ptr(w_router),
                                        _ptr(logit_bias), _ptr(correction_bias), _ptr(logits_out),
                                        _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def moe_residual_update(cfg, b, r, gamma_post, resid_g, out, stream=None):
    _check("moe_residual_update", lib().moe_residual_update(
        ctypes.byref(cfg), _ptr(b), _ptr(r), _ptr(gamma_post), _ptr(resid_g), _ptr(out),
        _stream(stream)))


def noisy_gate(cfg, u, w_router, w_noise, noise_eps, stream=None, want_h=True, want_p=True):
    """moe_noisy_gate on CUDA tensors; returns a dict of CUDA tensors (H, idx, w, P,
    importance, load, cv2)."""
    import torch
    T, n, k = cfg.T, cfg.n_experts, cfg.top_k
    dev = u.device
    out = {"idx": torch.empty((T, k), dtype=torch.int32, device=dev),
           "w": torch.empty((T, k), dtype=torch.float32, device=dev),
           "importance": torch.empty(n, dtype=torch.float32, device=dev),
           "load": torch.empty(n, dtype=torch.float32, device=dev),
           "cv2": torch.empty(4, dtype=torch.float32, device=dev)}
    out["H"] = torch.empty((T, n), dtype=torch.float32, device=dev) if want_h else None
    out["P"] = torch.empty((T, n), dtype=torch.float32, device=dev) if want_p else None
    nbytes = ctypes.c_size_t()
    _check("moe_noisy_gate_workspace_size",
           lib().moe_noisy_gate_workspace_size(ctypes.byref(cfg), ctypes.byref(nbytes)))
    ws = torch.empty(nbytes.value, dtype=torch.uint8, device=dev)
    _check("moe_noisy_gate", lib().moe_noisy_gate(
        ctypes.byref(cfg), _ptr(u), _ptr(w_router), _ptr(w_noise), _ptr(noise_eps),
        _ptr(out["H"]), _ptr(out["idx"]), _ptr(out["w"]), _ptr(out["P"]), _ptr(out["importance"]),
        _ptr(out["load"]), _ptr(out["cv2"]), _ptr(ws), nbytes.value, _stream(stream)))
    out["workspace"] = ws
    return out


def moe_router_split_weights(w, w_split, stream=None):
    """fp32 router weights w [n, d] -> their exact bf16 hi/mid/lo split w_split [n, 3d]."""
    n, d = w.shape
    _check("moe_router_split_weights",
           lib().moe_router_split_weights(_ptr(w), n, d, _ptr(w_split), _stream(stream)))


def router_split(w, stream=None):
    import torch
    out = torch.empty((w.shape[0], 3 * w.shape[1]), dtype=torch.bfloat16, device=w.device)
    moe_router_split_weights(w, out, stream)
    return out


def moe_permute(cfg, topk_idx, expert_offsets, perm_token, inv_perm, x=None, gamma_pre=None,
                x_perm=None, workspace=None, workspace_bytes=0, stream=None):
    if workspace is not None and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("moe_permute", lib().moe_permute(ctypes.byref(cfg), _ptr(topk_idx), _ptr(expert_offsets),
                                            _ptr(perm_token), _ptr(inv_perm), _ptr(x),
                                            _ptr(gamma_pre), _ptr(x_perm), _ptr(workspace),
                                            workspace_bytes, _stream(stream)))


def moe_permute_static(cfg, topk_idx, expert_offsets, perm_token, inv_perm, x=None,
                       gamma_pre=None, x_perm=None, stream=None):
    """moe_permute for callers that cannot allocate: the scratch is a fixed 256 KB array inside
    the library (ceil(T/128) * n_experts <= 65536), shared by all calls, so calls must not
    overlap on the GPU."""
    _check("moe_permute_static", lib().moe_permute_static(
        ctypes.byref(cfg), _ptr(topk_idx), _ptr(expert_offsets), _ptr(perm_token),
        _ptr(inv_perm), _ptr(x), _ptr(gamma_pre), _ptr(x_perm), _stream(stream)))


def moe_dispatch_rows(cfg, inv_perm, x, gamma_pre, x_perm, stream=None):
    """The row half of moe_permute: x_perm[inv_perm[t*k+j]] = C_pre(x[t]) (or x[t])."""
    _check("moe_dispatch_rows", lib().moe_dispatch_rows(
        ctypes.byref(cfg), _ptr(inv_perm), _ptr(x), _ptr(gamma_pre), _ptr(x_perm),
        _stream(stream)))


def moe_expert_ffn(cfg, x_perm, expert_offsets, w_gu, w_down, gamma_expert, out_perm,
                   workspace=None, workspace_bytes=0, stream=None, row_sumsq=None):
    if workspace is not None and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("moe_expert_ffn", lib().moe_expert_ffn(ctypes.byref(cfg), _ptr(x_perm),
                                                  _ptr(expert_offsets), _ptr(w_gu), _ptr(w_down),
                                                  _ptr(gamma_expert), _ptr(out_perm),
                                                  _ptr(row_sumsq), _ptr(workspace),
                                                  workspace_bytes, _stream(stream)))


def row_sumsq_parts(cfg) -> int:
    """Partial sums of squares per expert-output row that moe_expert_ffn writes to row_sumsq."""
    n = ctypes.c_int32()
    _check("moe_row_sumsq_parts", lib().moe_row_sumsq_parts(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_combine(cfg, out_perm, inv_perm, topk_w, y, stream=None, row_sumsq=None):
    _check("moe_combine", lib().moe_combine(ctypes.byref(cfg), _ptr(out_perm), _ptr(row_sumsq),
                                            _ptr(inv_perm), _ptr(topk_w), _ptr(y),
                                            _stream(stream)))


def moe_latent_down(cfg, u, p_down, z_raw, stream=None):
    _check("moe_latent_down", lib().moe_latent_down(ctypes.byref(cfg), _ptr(u), _ptr(p_down),
                                                    _ptr(z_raw), _stream(stream)))


def moe_latent_up(cfg, y, p_up, r, resid_g, out, stream=None):
    _check("moe_latent_up", lib().moe_latent_up(ctypes.byref(cfg), _ptr(y), _ptr(p_up), _ptr(r),
                                                _ptr(resid_g), _ptr(out), _stream(stream)))


def moe_gather_rows(src, rows, dst, stream=None):
    """dst[i] = src[rows[i]] (rows of src's last dimension; rows[i] < 0 gives a zero row)."""
    import torch
    row_bytes = src.shape[-1] * src.element_size()
    if rows.dtype != torch.int32 or dst.shape[0] != rows.numel() or \
            dst.shape[-1] * dst.element_size() != row_bytes or not src.is_contiguous() or \
            not dst.is_contiguous() or not rows.is_contiguous():
        raise ValueError("moe_gather_rows: int32 rows, contiguous src/dst with equal row bytes "
                         "and one dst row per index")
    _check("moe_gather_rows", lib().moe_gather_rows(_ptr(src), src.shape[0], _ptr(rows),
                                                    rows.numel(), row_bytes, _ptr(dst),
                                                    _stream(stream)))
    return dst


def make_weights(w: dict) -> Weights:
    """moe_weights_t from a dict of CUDA tensors (missing entries are NULL)."""
    return Weights(**{k: _ptr(w.get(k)) for k, _ in Weights._fields_})


def moe_layer_forward(cfg, weights: Weights, u, r, out, logits_out=None, topk_idx_out=None,
                      topk_w_out=None, workspace=None, workspace_bytes=0, stream=None):
    if workspace is not None and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(cfg), ctypes.byref(weights), _ptr(u), _ptr(r), _ptr(out), _ptr(logits_out),
        _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace), workspace_bytes, _stream(stream)))


def moe_layer_forward_taps(cfg, weights: Weights, u, r, out, taps: dict, logits_out=None,
                           topk_idx_out=None, topk_w_out=None, workspace=None, workspace_bytes=0,
                           stream=None):
    """moe_layer_forward that also copies the intermediates named in ``taps`` (device tensors
    under the keys z, s, y, inv_perm; missing keys are skipped)."""
    if workspace is not None and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    t = Taps(**{k: _ptr(taps.get(k)) for k, _ in Taps._fields_})
    _check("moe_layer_forward_taps", lib().moe_layer_forward_taps(
        ctypes.byref(cfg), ctypes.byref(weights), _ptr(u), _ptr(r), _ptr(out), _ptr(logits_out),
        _ptr(topk_idx_out), _ptr(topk_w_out), ctypes.byref(t), _ptr(workspace), workspace_bytes,
        _stream(stream)))


def moe_get_device_status(stream=None) -> int:
    return lib().moe_get_device_status(_stream(stream))


def launch_count() -> int:
    """Kernels libmoe.so has launched in this process."""
    return int(lib().moe_launch_count())


def profile_begin(max_calls: int):
    """Start recording per-stage CUDA events in the next ``max_calls`` moe_layer_forward calls."""
    _check("moe_profile_begin", lib().moe_profile_begin(max_calls))


def profile_end() -> tuple[dict, int]:
    """Stop recording; returns ({stage: summed ms}, recorded calls)."""
    ms = (ctypes.c_float * len(PROFILE_STAGES))()
    calls = ctypes.c_int32()
    _check("moe_profile_end", lib().moe_profile_end(ms, ctypes.byref(calls)))
    return {k: float(v) for k, v in zip(PROFILE_STAGES, ms)}, calls.value


def host_staging_size(cfg: Config) -> int:
    n = ctypes.c_size_t()
    _check("moe_host_staging_size", lib().moe_host_staging_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


class MoELayer:
    """A layer instance holding its device weights and a workspace, with a forward() that takes
    device or pinned-host inputs.  Nothing here computes: forward() is one moe_layer_forward."""

    def __init__(self, cfg: Config, weights: dict):
        import torch
        self.cfg = cfg
        self.weights = weights
        if cfg.router_f32 and cfg.dtype == MOE_BF16 and weights["w_router"].dtype == torch.float32:
            # fp32 router weights go to the tensor cores as their exact bf16 split (once)
            weights = dict(weights, w_router=router_split(weights["w_router"]))
            self.weights = weights
        self._w = make_weights(weights)
        self.workspace = torch.empty(workspace_size(cfg), dtype=torch.uint8, device="cuda")

    def forward(self, u, r=None, out=None, logits_out=None, topk_idx_out=None, topk_w_out=None,
                stream=None, taps: dict | None = None):
        """One moe_layer_forward; with ``taps`` (a dict of device tensors under the keys z, s, y,
        inv_perm) one moe_layer_forward_taps that also copies those intermediates."""
        import torch
        if out is None:
            out = torch.empty_like(u)
        r = r if r is not None else u
        if taps is None:
            moe_layer_forward(self.cfg, self._w, u, r, out, logits_out, topk_idx_out, topk_w_out,
                              self.workspace, stream=stream)
        else:
            moe_layer_forward_taps(self.cfg, self._w, u, r, out, taps, logits_out, topk_idx_out,
                                   topk_w_out, self.workspace, stream=stream)
        return out

    def forward_host(self, u_hosts, out_hosts, stream=None):
        """Forwards of batches held in (pinned) host memory, one moe_layer_forward_host call:
        batch i's input u_hosts[i] (also its residual) goes to the device, through the layer and
        back to out_hosts[i]; the library overlaps the copies of neighbouring batches with each
        batch's kernels.  A single tensor stands for a one-batch list.  Synchronise `stream`
        (default: the current stream) before reading the outputs."""
        import torch
        if isinstance(u_hosts, torch.Tensor):
            u_hosts, out_hosts = [u_hosts], [out_hosts]
        if len(u_hosts) != len(out_hosts):
            raise ValueError("u_hosts and out_hosts differ in length")
        if getattr(self, "_staging", None) is None:
            self._staging = torch.empty(host_staging_size(self.cfg), dtype=torch.uint8,
                                        device="cuda")
        n = len(u_hosts)
        ins = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in u_hosts])
        outs = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in out_hosts])
        _check("moe_layer_forward_host",
               lib().moe_layer_forward_host(ctypes.byref(self.cfg), ctypes.byref(self._w), n, ins,
                                            outs, self._staging.data_ptr(),
                                            self._staging.numel(), self.workspace.data_ptr(),
                                            self.workspace.numel(), _stream(stream)))
        return out_hosts
