"""moe_permute_static: the dispatch permutation for callers that cannot allocate device memory
(a host that passes only input and output buffers and has no scratch pool to offer).  Its
scratch is a fixed array inside the library, so the test checks that two calls in a row, of
different sizes, give the same outputs as moe_permute with a caller workspace and the oracle's
canonical permutation, and that a size beyond the array is refused before anything runs.

Kept in its own file, collected last, so that a failure here cannot hide any other test.
"""
import numpy as np
import pytest

import moe_inputs
import oracle
from moe_inputs import configs

from gpu_harness import abi_config

torch = pytest.importorskip("torch")
moe = pytest.importorskip("sparse_moe_layer_softmax_b200")
pytestmark = pytest.mark.gpu


def _routing(T, n, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(n, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def _run(cfg, idx, use_static):
    c = abi_config(cfg)
    T, k, n, E = cfg.T, cfg.top_k, cfg.n_experts, cfg.d_latent
    x = torch.empty((T, E), dtype=torch.bfloat16, device="cuda")
    moe_inputs.normal_device(x, cfg.seed, 80, 0, 1.0)
    g = torch.empty(E, dtype=torch.float32, device="cuda")
    moe_inputs.normal_device(g, cfg.seed, 81, 0, 0.1)
    off = torch.full((n + 1,), -5, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -5, dtype=torch.int32, device="cuda")
    inv = torch.full((T * k,), -5, dtype=torch.int32, device="cuda")
    xp = torch.zeros((T * k, E), dtype=torch.bfloat16, device="cuda")
    d_idx = torch.from_numpy(idx).cuda()
    if use_static:
        moe.moe_permute_static(c, d_idx, off, perm, inv, x=x, gamma_pre=g, x_perm=xp)
    else:
        ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
        moe.moe_permute(c, d_idx, off, perm, inv, x=x, gamma_pre=g, x_perm=xp, workspace=ws)
    assert moe.moe_get_device_status() == 0
    return [t.cpu() for t in (off, perm, inv, xp)]


def test_permute_static_matches_workspace_version_twice():
    # two calls in a row; the second is smaller, so stale histograms from the first are present
    cases = [configs.small_muse(T=32768, d=256, L=256, n=256, k=8, seed=61),
             configs.small_muse(T=333, d=256, L=128, n=64, k=4, seed=62)]
    for cfg in cases:
        idx = _routing(cfg.T, cfg.n_experts, cfg.top_k, cfg.seed)
        ref = _run(cfg, idx, use_static=False)
        got = _run(cfg, idx, use_static=True)
        for a, b in zip(got[:3], ref[:3]):
            np.testing.assert_array_equal(a.numpy(), b.numpy())
        # and both equal the oracle's canonical permutation of the same routing
        for a, b in zip(got[:3], oracle.permutation(cfg.T, cfg.top_k, cfg.n_experts, idx)):
            np.testing.assert_array_equal(a.numpy(), b)
        # same kernels on the same inputs: the gathered, normalised rows agree exactly
        np.testing.assert_array_equal(got[3].float().numpy(), ref[3].float().numpy())


def test_permute_static_rejects_sizes_beyond_its_scratch():
    # real input and output buffers of the refused size (no stand-in addresses): the call is
    # refused on the host, so the outputs keep their fill
    cfg = configs.small_muse(T=32769, n=256, k=8)  # ceil(T/128) * 256 > 65536
    c = abi_config(cfg)
    T, k, n = cfg.T, cfg.top_k, cfg.n_experts
    idx = torch.from_numpy(_routing(T, n, k, 63)).cuda()
    off = torch.full((n + 1,), -5, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -5, dtype=torch.int32, device="cuda")
    inv = torch.full((T * k,), -5, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_static(c, idx, off, perm, inv)
    assert e.value.code == moe.STATUS_CODES["MOE_ERR_WORKSPACE"]
    torch.cuda.synchronize()
    for t in (off, perm, inv):  # nothing was launched: the outputs still hold their fill
        assert bool((t == -5).all())
