"""Separated router logits for the named workloads: which rows of u to draw again.

The gate keeps the k experts with the largest selection keys ("816 billion parameters, and only
42 billion show up for each token", section "The gate": KeepTopK), so a token whose k-th and
(k+1)-th keys are nearly equal has no selection that every summation order agrees on.  The
workloads therefore draw such a token's input row again, from a fresh stretch of the same counter
stream, until its margin is at least SEPARATION times the rms of its keys:

    keys   = router logits (softmax gate, Zipf bias included), or sigmoid scores + correction
             bias (Muse sigmoid gate), from the CPU oracle's router in double
    margin = key_(k) - key_(k+1)  (the k-th and (k+1)-th largest)
    redraw while margin < SEPARATION * sqrt(mean(keys^2))

A token drawn g times has row t of generation g: counter elements [(g*T + t)*d, (g*T + t + 1)*d)
of u's stream.  The script calls only the oracle and the input generator and writes
router_redraws.json beside it:

    python tests/golden/separate_router_logits.py
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import moe_inputs  # noqa: E402
import oracle  # noqa: E402
from moe_inputs import configs  # noqa: E402


def router_inputs(cfg) -> dict:
    """The router's tensors other than u."""
    specs = moe_inputs.tensor_specs(cfg)
    d = {name: moe_inputs.host_rows(cfg, name)
         for name in ("w_router", "correction_bias", "gamma_in") if name in specs}
    if cfg.zipf_bias:
        d["logit_bias"] = moe_inputs.zipf_bias(cfg)
    return d


def selection_keys(cfg, logits: np.ndarray, dense: dict) -> np.ndarray:
    """What the top-k is taken on: the oracle router's logits, or its sigmoid scores plus the
    selection-only correction bias."""
    if cfg.gate_mode == configs.GATE_SIGMOID:
        return logits + dense["correction_bias"].astype(np.float64)
    return logits


def margins(keys: np.ndarray, k: int):
    """(k-th minus (k+1)-th largest key, rms of the keys) per row; the margin is +inf when k = n."""
    rms = np.sqrt(np.mean(keys * keys, axis=1))
    if k >= keys.shape[1]:
        return np.full(keys.shape[0], np.inf), rms
    srt = -np.sort(-keys, axis=1)
    return srt[:, k - 1] - srt[:, k], rms


def redraws_for(cfg, rel: float = configs.SEPARATION, rows=None):
    """The redraw list of `cfg` (its own list ignored): ((token, generation), ...), and the
    number of oracle router passes.  `rows` limits the search to those tokens."""
    base = cfg.replace(u_redraw=())
    dense = router_inputs(base)
    gen: dict[int, int] = {}
    pending = np.arange(cfg.T) if rows is None else np.asarray(rows, dtype=np.int64)
    first = rows is None
    passes = 0
    while len(pending):
        cur = base.replace(u_redraw=tuple(sorted(gen.items())))
        u = moe_inputs.host_rows(cur, "u") if first else moe_inputs.host_rows(cur, "u",
                                                                              rows=pending)
        first = False
        res = oracle.router(cur, {**dense, "u": u})
        m, rms = margins(selection_keys(cfg, res["logits"], dense), cfg.top_k)
        passes += 1
        pending = pending[m < rel * rms]
        for t in pending.tolist():
            gen[t] = gen.get(t, 0) + 1
    return tuple(sorted(gen.items())), passes


def check_separated(cfg, tokens, rel: float = configs.SEPARATION) -> np.ndarray:
    """Margins / (rel * rms) of the listed tokens of `cfg` as generated (its redraw list
    applied); every entry must be >= 1."""
    dense = router_inputs(cfg)
    u = moe_inputs.host_rows(cfg, "u", rows=tokens)
    res = oracle.router(cfg, {**dense, "u": u})
    m, rms = margins(selection_keys(cfg, res["logits"], dense), cfg.top_k)
    return m / (rel * rms)


def main():
    out = {"separation": configs.SEPARATION,
           "recipe": "redraw row t of u (generation g: counter elements [(g*T+t)*d, (g*T+t+1)*d)) "
                     "while its k-th minus (k+1)-th router selection key is below separation * "
                     "rms(keys); keys from the CPU oracle's router",
           "workloads": {}}
    for name in configs.SEPARATED_NAMES:
        cfg = configs.ALL_CONFIGS[name]
        t0 = time.time()
        red, passes = redraws_for(cfg)
        out["workloads"][name] = {"T": cfg.T, "tokens_redrawn": len(red),
                                  "draws_beyond_first": int(sum(g for _, g in red)),
                                  "router_passes": passes, "redraws": [list(p) for p in red]}
        print(f"{name}: T={cfg.T} redrawn {len(red)} tokens in {passes} passes "
              f"({time.time() - t0:.1f} s)", flush=True)
    with open(configs.REDRAWS_PATH, "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
