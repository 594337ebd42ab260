"""The five named workloads of the MoE-layer forward and their input recipes.

Shapes and value distributions follow the workloads this library is measured on:

* ``tiny_shazeer_f32``   - Shazeer-style MoE, fp32, T=128, d=64, n=8, k=2, experts 64->128 ReLU->64,
  router weights scaled x4 so logits are well separated (seed 0).
* ``shazeer_bf16``       - Shazeer-style MoE, bf16, T=8192, d=512, n=256, k=4, experts
  512->1024 ReLU->512, inputs and weights ~ N(0, 1/fan_in) (seed 1).
* ``muse_decode``        - Muse-shape latent MoE, T=64, hidden 8192, latent 4096, 256 SwiGLU
  experts (4096->4096->4096), top-8, per-expert input-scaled RMSNorm, residual gate (seed 2).
* ``muse_prefill``       - the same layer at T=16384 (seed 3).
* ``muse_imbalanced``    - the same layer at T=32768 with a Zipf(s=1.2) per-expert router bias
  scaled so the hottest expert receives about 20x the mean load (seed 4).

The Muse layer is the latent MoE block described in "Muse Spark Open: Norm-Preserving Gates Are
Not a Norm Guarantee" (flozi.net, sections "Latent experts: normalization happens before the
weighted sum" and "Residual gates"); the Shazeer layer is the one of "816 billion parameters, and
only 42 billion show up for each token" (bobbyburns.tech, sections "The math" and "The gate").

This module holds no layer arithmetic: only sizes, seeds and distributions.
"""
from __future__ import annotations

import dataclasses
import json
import math
import os

# Stream identifiers: one independent counter stream per tensor (any distinct integers work).
STREAM_X = 1
STREAM_W_ROUTER = 2
STREAM_P_DOWN = 3
STREAM_P_UP = 4
STREAM_W_GU = 5
STREAM_W_DOWN = 6
STREAM_GAMMA_PRE = 7
STREAM_GAMMA_EXPERT = 8
STREAM_RESID_G = 9
STREAM_RESID_H = 10
STREAM_ZIPF = 11
STREAM_SUBSAMPLE = 12

ACT_RELU = 0
ACT_SWIGLU = 1
RESID_NONE = 0
RESID_MUSE_GATE = 1
RESID_LITERAL = 2
GATE_SOFTMAX = 0
GATE_SIGMOID = 1
STREAM_CORR_BIAS = 13
STREAM_GAMMA_IN = 14
STREAM_GAMMA_POST = 15
STREAM_W_NOISE = 16
STREAM_NOISE_EPS = 17

# Scale c of the Zipf router bias  bias_e = -c * s * ln(rank_e)  (s = 1.2) for the imbalanced
# workload.  Calibrated by tests/golden/calibrate_zipf_bias.py, which bisects c with the CPU
# oracle's router on a seeded 2048-token calibration sample until the hottest expert's load is
# 20x the mean; the script's output is tests/golden/zipf_bias_scale.json and a CPU test keeps the
# two equal.
ZIPF_S = 1.2
ZIPF_BIAS_SCALE = 0.46277


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int                 # expert hidden width (ReLU hidden, or SwiGLU intermediate I)
    d_latent: int = 0         # 0: no latent projections (Shazeer layer)
    dtype: str = "bf16"       # "f32" or "bf16"
    act: int = ACT_SWIGLU
    pre_norm: int = 0         # centred RMSNorm after the latent down-projection
    expert_norm: int = 0      # per-expert input-scaled RMSNorm before the weighted sum
    resid_mode: int = RESID_NONE
    eps: float = 1e-6
    tau: float = 0.3
    resid_floor: float = 1e-3
    routed_scale: float = 1.0
    seed: int = 0
    x_sigma: float = 1.0      # std of the layer input u (and of the residual h = u)
    router_gain: float = 1.0  # extra factor on the router weights' std
    zipf_bias: bool = False
    gamma_sigma: float = 0.02
    gate_mode: int = GATE_SOFTMAX
    router_f32: int = 0         # router weights stored in fp32
    logit_mult: float = 1.0     # output_multiplier of the sigmoid gate
    corr_sigma: float = 0.05    # std of the sigmoid gate's selection-only correction bias
    input_norm: int = 0         # decoder wrap: u = C_in(h), centred RMSNorm of the residual stream
    post_norm: int = 0          # decoder wrap: input-scaled output norm I_post on b before the gate
    eps_block: float = 1e-5     # epsilon of the decoder-level norms (model sheet: 1e-5)
    noisy_gate: bool = False    # Shazeer's noisy gate: W_noise ~ N(0, router std^2), eps ~ N(0, 1)
    # Rows of u drawn again so that every token's router logits are separated at the top-k
    # boundary: ((token, generation), ...).  Row t of generation g is counter elements
    # [(g*T + t)*d, (g*T + t + 1)*d) of u's stream (generation 0 is the first draw).
    u_redraw: tuple = ()

    @property
    def latent(self) -> bool:
        return self.d_latent > 0

    @property
    def expert_in(self) -> int:
        """Width of an expert's input (latent width, or the model width without latent)."""
        return self.d_latent if self.latent else self.d_model

    @property
    def gu_rows(self) -> int:
        """Rows of one expert's first weight matrix: 2*I (gate rows, then up rows) or h."""
        return 2 * self.d_ff if self.act == ACT_SWIGLU else self.d_ff

    def replace(self, **kw) -> "MoEConfig":
        """A derived workload.  A redraw list belongs to the one workload it was computed for,
        so it is dropped unless given again."""
        kw.setdefault("u_redraw", ())
        return dataclasses.replace(self, **kw)

    # ---- std of each generated tensor (N(0, 1/fan_in) weights) ----
    def sigma_router(self) -> float:
        return self.router_gain / math.sqrt(self.d_model)

    def sigma_p_down(self) -> float:
        return 1.0 / math.sqrt(self.d_model)

    def sigma_p_up(self) -> float:
        return 1.0 / math.sqrt(self.d_latent)

    def sigma_w_gu(self) -> float:
        return 1.0 / math.sqrt(self.expert_in)

    def sigma_w_down(self) -> float:
        return 1.0 / math.sqrt(self.d_ff)


TINY_SHAZEER_F32 = MoEConfig(
    name="tiny_shazeer_f32", T=128, d_model=64, n_experts=8, top_k=2, d_ff=128, dtype="f32",
    act=ACT_RELU, seed=0, x_sigma=1.0, router_gain=4.0)

SHAZEER_BF16 = MoEConfig(
    name="shazeer_bf16", T=8192, d_model=512, n_experts=256, top_k=4, d_ff=1024, dtype="bf16",
    act=ACT_RELU, seed=1, x_sigma=1.0 / math.sqrt(512))

MUSE_DECODE = MoEConfig(
    name="muse_decode", T=64, d_model=8192, d_latent=4096, n_experts=256, top_k=8, d_ff=4096,
    dtype="bf16", act=ACT_SWIGLU, pre_norm=1, expert_norm=1, resid_mode=RESID_MUSE_GATE,
    eps=1e-6, seed=2, x_sigma=1.0)

MUSE_PREFILL = MUSE_DECODE.replace(name="muse_prefill", T=16384, seed=3)

MUSE_IMBALANCED = MUSE_DECODE.replace(name="muse_imbalanced", T=32768, seed=4, zipf_bias=True)

CONFIGS = {c.name: c for c in (TINY_SHAZEER_F32, SHAZEER_BF16, MUSE_DECODE, MUSE_PREFILL,
                               MUSE_IMBALANCED)}

# Profiler capture cases: the Muse layer with 32 experts instead of 256, so that a capture holds a
# few GB of weights, at the same rows per expert as the full workloads (prefill: 512 per expert;
# decode: 2 per expert), i.e. the same per-tile work in every kernel.
MUSE_PREFILL_N32 = MUSE_PREFILL.replace(name="muse_prefill_n32", T=2048, n_experts=32, seed=5)
MUSE_DECODE_N32 = MUSE_DECODE.replace(name="muse_decode_n32", T=8, n_experts=32, seed=6)
# The prefill layer with 128-wide experts: the router, dispatch and combine kernels run at exactly
# their prefill sizes (T=16384, d=8192, 256 experts, top-8, latent 4096) while the whole case
# holds about 2.5 GB, small enough for a profiler capture of those kernels.
MUSE_PREFILL_SMALLFFN = MUSE_PREFILL.replace(name="muse_prefill_smallffn", d_ff=128, seed=7)
PROFILE_CONFIGS = {c.name: c for c in (MUSE_PREFILL_N32, MUSE_DECODE_N32, MUSE_PREFILL_SMALLFFN)}

# The Muse router as the Muse audit describes it ("Latent experts"): fp32 router weights, sigmoid
# scores, a selection-only correction bias ~ N(0, 0.05^2) (values not given on the pages),
# output_multiplier 1 (value not given) and routed_scaling_factor 1 (model sheet).
MUSE_DECODE_SIGMOID = MUSE_DECODE.replace(name="muse_decode_sigmoid", gate_mode=GATE_SIGMOID,
                                          router_f32=1, seed=8)
MUSE_PREFILL_SIGMOID = MUSE_PREFILL.replace(name="muse_prefill_sigmoid", gate_mode=GATE_SIGMOID,
                                            router_f32=1, seed=9)
# The MoE sub-block of the decoder layer as the Muse audit describes it ("The complete layer has
# two separately normalized residual updates"): the residual stream h is normalised (block norm
# with a (1 + gamma) gain, eps 1e-5 per the model sheet), the latent MoE runs, its output goes
# through the FFN's input-scaled output norm, and the residual gate mixes it into h.
MUSE_DECODE_BLOCK = MUSE_DECODE.replace(name="muse_decode_block", input_norm=1, post_norm=1,
                                        seed=10)
MUSE_PREFILL_BLOCK = MUSE_PREFILL.replace(name="muse_prefill_block", input_norm=1, post_norm=1,
                                          seed=11)
VARIANT_CONFIGS = {c.name: c for c in (MUSE_DECODE_SIGMOID, MUSE_PREFILL_SIGMOID,
                                       MUSE_DECODE_BLOCK, MUSE_PREFILL_BLOCK)}

# Shazeer et al.'s noisy gate statistics on the Shazeer-shaped batch (training-time diagnostics
# computed forward: noisy logits, KeepTopK gate, importance and smooth load with their CV^2).
SHAZEER_BF16_NOISY = SHAZEER_BF16.replace(name="shazeer_bf16_noisy", noisy_gate=True, seed=12)
GATE_STAT_CONFIGS = {c.name: c for c in (SHAZEER_BF16_NOISY,)}
ALL_CONFIGS = {**CONFIGS, **PROFILE_CONFIGS, **VARIANT_CONFIGS}


def small_muse(T: int = 37, d: int = 256, L: int = 128, I: int = 128, n: int = 16, k: int = 4,
               seed: int = 7, **kw) -> MoEConfig:
    """A Muse-structured layer at sizes the oracle finishes in well under a second."""
    return MUSE_DECODE.replace(name=f"small_muse_T{T}", T=T, d_model=d, d_latent=L, d_ff=I,
                               n_experts=n, top_k=k, seed=seed, **kw)


def small_shazeer(T: int = 45, d: int = 128, h: int = 256, n: int = 16, k: int = 4,
                  seed: int = 5, **kw) -> MoEConfig:
    return SHAZEER_BF16.replace(name=f"small_shazeer_T{T}", T=T, d_model=d, d_ff=h, n_experts=n,
                                top_k=k, seed=seed, x_sigma=1.0 / math.sqrt(d), **kw)


# ---------------------------------------------------------------------------------------------
# Separated router logits.  The named workloads draw again every token of u whose k-th and
# (k+1)-th router selection keys (the logits, or the sigmoid scores plus the correction bias)
# are closer than SEPARATION * rms of that token's keys, so that the top-k selection is the same
# in any summation order.  The redraw lists are computed with the CPU oracle's router by
# tests/golden/separate_router_logits.py, which writes tests/golden/router_redraws.json; a CPU
# test recomputes them.
SEPARATION = 1e-3
REDRAWS_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests",
                            "golden", "router_redraws.json")


def _load_redraws() -> dict:
    if not os.path.exists(REDRAWS_PATH):
        return {}
    with open(REDRAWS_PATH) as f:
        data = json.load(f)
    return {name: tuple((int(t), int(g)) for t, g in w["redraws"])
            for name, w in data["workloads"].items()}


REDRAWS = _load_redraws()


def separated(cfg: MoEConfig) -> MoEConfig:
    """The named workload with its stored redraw list (unchanged if it has none)."""
    return dataclasses.replace(cfg, u_redraw=REDRAWS.get(cfg.name, ()))


TINY_SHAZEER_F32 = separated(TINY_SHAZEER_F32)
SHAZEER_BF16 = separated(SHAZEER_BF16)
MUSE_DECODE = separated(MUSE_DECODE)
MUSE_PREFILL = separated(MUSE_PREFILL)
MUSE_IMBALANCED = separated(MUSE_IMBALANCED)
MUSE_DECODE_SIGMOID = separated(MUSE_DECODE_SIGMOID)
MUSE_PREFILL_SIGMOID = separated(MUSE_PREFILL_SIGMOID)
MUSE_DECODE_BLOCK = separated(MUSE_DECODE_BLOCK)
MUSE_PREFILL_BLOCK = separated(MUSE_PREFILL_BLOCK)
SEPARATED_NAMES = tuple(c.name for c in (TINY_SHAZEER_F32, SHAZEER_BF16, MUSE_DECODE, MUSE_PREFILL,
                                         MUSE_IMBALANCED, MUSE_DECODE_SIGMOID,
                                         MUSE_PREFILL_SIGMOID, MUSE_DECODE_BLOCK,
                                         MUSE_PREFILL_BLOCK))
CONFIGS = {c.name: c for c in (TINY_SHAZEER_F32, SHAZEER_BF16, MUSE_DECODE, MUSE_PREFILL,
                               MUSE_IMBALANCED)}
VARIANT_CONFIGS = {c.name: c for c in (MUSE_DECODE_SIGMOID, MUSE_PREFILL_SIGMOID,
                                       MUSE_DECODE_BLOCK, MUSE_PREFILL_BLOCK)}
ALL_CONFIGS = {**CONFIGS, **PROFILE_CONFIGS, **VARIANT_CONFIGS}
