"""The five named workloads at full size, in the launch configuration the benchmark times
(moe_layer_forward on one stream).

Routing and the dispatch permutation are checked bit for bit on every token (the oracle's
selection on the GPU's fp32 logits, the oracle's canonical permutation of the GPU's indices).
The workloads' router inputs are separated at the top-k boundary (tokens with a k-th /
(k+1)-th margin below 1e-3 of the keys' rms are drawn again), so the oracle's own selection on
its double logits equals the GPU's on every checked token, none is skipped, and the GPU's keys
show no near tie on any token.  Values are checked against the oracle on every token for the
three smaller workloads and on the seeded 512-token subsample for the two large ones (tokens are
independent and nothing is dropped, so a token's output does not depend on which other tokens
are present).  On the same tokens the intermediates are checked too: the expert input z (after
C_pre), each slot's expert output s before its norm, and the combined latent y.
"""
import numpy as np
import pytest

import moe_inputs
import oracle
from moe_inputs import configs

from gpu_harness import (abi_config, check_routing, compare_selection, device_values, key_margins,
                         logit_atol, oracle_reference, row_rel_err, run_layer, selection_keys,
                         tolerance)

torch = pytest.importorskip("torch")
moe = pytest.importorskip("sparse_moe_layer_softmax_b200")
pytestmark = pytest.mark.gpu


def _permutation_bit_exact(cfg, idx_dev, idx):
    c = abi_config(cfg)
    n, TK = cfg.n_experts, cfg.T * cfg.top_k
    off = torch.empty(n + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(TK, dtype=torch.int32, device="cuda")
    inv = torch.empty(TK, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    moe.moe_permute(c, idx_dev, off, perm, inv, workspace=ws)
    assert moe.moe_get_device_status() == 0
    r_off, r_perm, r_inv = oracle.permutation(cfg.T, cfg.top_k, n, idx)
    np.testing.assert_array_equal(off.cpu().numpy(), r_off)
    np.testing.assert_array_equal(perm.cpu().numpy(), r_perm)
    np.testing.assert_array_equal(inv.cpu().numpy(), r_inv)
    return r_off


@pytest.mark.parametrize("name", list(configs.CONFIGS) + list(configs.VARIANT_CONFIGS))
def test_full_workload(name):
    cfg = configs.ALL_CONFIGS[name]
    dev = moe_inputs.device_inputs(cfg)
    res = run_layer(cfg, dev, want_taps=True)
    logits = res["logits"].cpu().numpy()
    idx = res["idx"].cpu().numpy()
    check_routing(cfg, logits, idx, res["w"].cpu().numpy())
    offsets = _permutation_bit_exact(cfg, res["idx"], idx)
    if cfg.zipf_bias:  # the hottest expert carries about 20x the mean load
        ratio = np.diff(offsets).max() / (cfg.T * cfg.top_k / cfg.n_experts)
        assert 15.0 <= ratio <= 25.0, ratio
    # separated inputs: no token's GPU selection keys are near a tie at the top-k boundary
    gm = key_margins(selection_keys(cfg, logits.astype(np.float64)), cfg.top_k)
    assert gm.min() >= 1e-4, f"GPU-key margin {gm.min():.2e} of rms"
    tokens = moe_inputs.subsample_tokens(cfg, cfg.T if cfg.T <= 8192 else 512)
    tk = torch.from_numpy(tokens).cuda()
    out = device_values(res["out"][tk])
    taps = res.get("taps")
    got = None
    if taps is not None:
        slots = res["inv"][tk].long()                       # [tokens, k] dispatch rows
        got = {"z": device_values(taps["z"][tk]), "y": device_values(taps["y"][tk]),
               "s": device_values(taps["s"][slots.flatten()]).reshape(len(tokens), cfg.top_k, -1)}
    del res, dev, taps
    torch.cuda.empty_cache()
    ref = oracle_reference(cfg, tokens, want_s=got is not None)
    ties = compare_selection(idx[tokens], selection_keys(cfg, ref["logits"]), ref["idx"], cfg.top_k)
    assert ties.sum() == 0, f"{int(ties.sum())} near ties in separated inputs"
    lg = logits[tokens]
    np.testing.assert_allclose(lg, ref["logits"], rtol=0, atol=logit_atol(cfg, lg))
    err = row_rel_err(out, ref["out"])
    print(f"{name}: tokens checked {len(tokens)}, redrawn inputs {len(cfg.u_redraw)}, "
          f"max row rel err {err.max():.3e}, mean {err.mean():.3e}, "
          f"p99 {np.percentile(err, 99):.3e}")
    assert err.max() <= tolerance(cfg)
    if got is not None:
        # slot j of a token is the GPU's j-th expert; the oracle's slots are in its own selection
        # order, which may swap two selected experts whose keys nearly tie: match slots by expert
        gi = idx[tokens]
        order = np.array([[list(ref["idx"][i]).index(e) for e in gi[i]] for i in range(len(gi))])
        ref["s"] = np.take_along_axis(ref["s"], order[:, :, None], axis=1)
        for key in ("z", "s", "y"):
            e = row_rel_err(got[key], ref[key])
            print(f"  {key}: max row rel err {e.max():.3e}")
            assert e.max() <= tolerance(cfg), key
