"""The five named workloads at full size, in the launch configuration the benchmark times
(moe_layer_forward on one stream).

Routing and the dispatch permutation are checked bit for bit on every token (the oracle's
selection on the GPU's fp32 logits, the oracle's canonical permutation of the GPU's indices).
Values are checked against the oracle on every token for the three smaller workloads and on the
seeded 512-token subsample for the two large ones (tokens are independent and nothing is
dropped, so a token's output does not depend on which other tokens are present).
"""
import numpy as np
import pytest

import moe_inputs
import oracle
from moe_inputs import configs

from gpu_harness import (abi_config, check_routing, compare_selection, device_values, logit_atol,
                         oracle_reference, row_rel_err, run_layer, selection_keys, tolerance)

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
    res = run_layer(cfg, dev)
    logits = res["logits"].cpu().numpy()
    idx = res["idx"].cpu().numpy()
    check_routing(cfg, logits, idx, res["w"].cpu().numpy())
    offsets = _permutation_bit_exact(cfg, res["idx"], idx)
    if cfg.zipf_bias:  # the hottest expert carries about 20x the mean load
        ratio = np.diff(offsets).max() / (cfg.T * cfg.top_k / cfg.n_experts)
        assert 15.0 <= ratio <= 25.0, ratio
    tokens = moe_inputs.subsample_tokens(cfg, cfg.T if cfg.T <= 8192 else 512)
    out = device_values(res["out"][torch.from_numpy(tokens).cuda()])
    del res, dev
    torch.cuda.empty_cache()
    ref = oracle_reference(cfg, tokens)
    ties = compare_selection(idx[tokens], selection_keys(cfg, ref["logits"]), ref["idx"], cfg.top_k)
    assert ties.sum() <= max(2, len(tokens) // 100)
    lg = logits[tokens]
    np.testing.assert_allclose(lg, ref["logits"], rtol=0, atol=logit_atol(cfg, lg))
    err = row_rel_err(out[~ties], ref["out"][~ties])
    print(f"{name}: tokens checked {int((~ties).sum())}, near ties {int(ties.sum())}, "
          f"max row rel err {err.max():.3e}, mean {err.mean():.3e}")
    assert err.max() <= tolerance(cfg)
