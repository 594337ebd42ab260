"""Calibrate the scale c of the Zipf router bias of the load-imbalanced Muse workload.

The workload adds  bias_e = -c * 1.2 * ln(rank_e)  to expert e's router logit (ranks from a
seeded shuffle) and asks for a hottest expert carrying about 20x the mean load.  This script
routes a seeded 2048-token calibration sample with the CPU oracle's router, then bisects c (40
steps on [0, 16]) until max_e load_e / mean load = 20, and writes zipf_bias_scale.json beside it.
It calls only the oracle and the input generator.

    python tests/golden/calibrate_zipf_bias.py
"""
import ctypes
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs  # noqa: E402
import oracle  # noqa: E402
from moe_inputs import configs  # noqa: E402


def main():
    # the calibration sample is the first draw of u (the workload's separation redraws, which
    # depend on the bias, come after the scale is fixed)
    cfg = configs.MUSE_IMBALANCED.replace(u_redraw=())
    ncal = 2048
    toks = np.sort(moe_inputs.fisher_yates(cfg.seed, configs.STREAM_SUBSAMPLE, cfg.T, ncal))
    inp = {"u": moe_inputs.host_rows(cfg, "u", rows=toks),
           "w_router": moe_inputs.host_rows(cfg, "w_router")}
    keep = oracle._Keep()
    c = oracle.make_cfg(cfg, T=ncal)
    x = oracle.make_tensors(cfg, inp, keep, experts={})
    logits = np.zeros((ncal, cfg.n_experts))
    idx = np.zeros(cfg.top_k, dtype=np.int32)
    w = np.zeros(cfg.top_k)
    for i in range(ncal):  # unbiased logits; the bias is added per candidate c below
        oracle.lib().orc_router_token(ctypes.byref(c), ctypes.byref(x), i, logits[i].ctypes.data,
                                      idx.ctypes.data, w.ctypes.data)
    ranks = moe_inputs.zipf_ranks(cfg).astype(np.float64)
    mean_load = ncal * cfg.top_k / cfg.n_experts

    def ratio(scale):
        bias = (-scale * configs.ZIPF_S * np.log(ranks)).astype(np.float32).astype(np.float64)
        sel, _ = oracle.softmax_topk(logits + bias, cfg.top_k)
        return np.bincount(sel.reshape(-1), minlength=cfg.n_experts).max() / mean_load

    lo, hi = 0.0, 16.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if ratio(mid) < 20.0:
            lo = mid
        else:
            hi = mid
    scale = round(hi, 6)
    out = {"zipf_bias_scale": scale, "ratio_on_calibration_sample": ratio(scale),
           "calibration_tokens": ncal, "target_ratio": 20.0,
           "recipe": "bias_e = -c * 1.2 * ln(rank_e); c bisected with the oracle router"}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_bias_scale.json"),
              "w") as f:
        json.dump(out, f, indent=2)
    print(out)


if __name__ == "__main__":
    main()
