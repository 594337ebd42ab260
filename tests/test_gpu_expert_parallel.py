"""Expert parallelism on one GPU: every rank of an R-rank expert-parallel layer runs in one process
(the exchanges become slicing and concatenation; no rank waits on another), and the result is
compared with the single-device layer on the whole batch.

A token's output does not depend on which other tokens share its batch or its expert group (each
GEMM reduces every output element over k in the same order whatever tile holds it, and every
other stage works per token or per row), so with the same GEMM orientation on every owner the
expert-parallel layer gives the single-device staged layer's bits.  That holds while every rank
has more than 256 tokens: up to 256 the router's logits come from a CUDA-core kernel whose fp32
sums round differently from the tensor-core GEMM's, so decode-sized ranks are checked against
the oracle instead.
"""
import numpy as np
import pytest

import moe_inputs
from moe_inputs import configs

from gpu_harness import (abi_config, compare_selection, device_values, oracle_reference,
                         row_rel_err, run_layer, selection_keys, separate, tolerance)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_layer_softmax_b200")
from sparse_moe_layer_softmax_b200 import expert_parallel as ep  # noqa: E402


@pytest.fixture(autouse=True)
def _cuda_cleanup():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ row gather


@pytest.mark.parametrize("row_bytes", [16, 272, 8192])
def test_gather_rows_bit_exact(row_bytes):
    g = torch.Generator().manual_seed(row_bytes)
    src_rows, n_rows = 300, 1000
    src = torch.randint(-2**31, 2**31 - 1, (src_rows, row_bytes // 4), generator=g,
                        dtype=torch.int32)
    rows = torch.randint(-3, src_rows, (n_rows,), generator=g, dtype=torch.int32)
    dst = torch.full((n_rows, row_bytes // 4), 7, dtype=torch.int32, device="cuda")
    moe.moe_gather_rows(src.cuda(), rows.cuda(), dst)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    want = src[rows.clamp(min=0).long()]
    want[rows < 0] = 0                                   # a negative index is a zero row
    assert torch.equal(dst.cpu(), want)


def test_gather_rows_out_of_range_index_latches():
    src = torch.arange(4 * 8, dtype=torch.int32, device="cuda").reshape(4, 8)
    rows = torch.tensor([1, 4, 0], dtype=torch.int32, device="cuda")
    dst = torch.empty((3, 8), dtype=torch.int32, device="cuda")
    moe.moe_gather_rows(src, rows, dst)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.STATUS_CODES["MOE_ERR_DEVICE_CHECK"]
    assert torch.equal(dst[0], src[1]) and torch.equal(dst[2], src[0])
    assert int(dst[1].abs().sum()) == 0                  # read nothing out of bounds
    assert moe.moe_get_device_status() == 0              # the status was read and cleared


# ------------------------------------------------------------------ the single-device reference


def staged_layer(cfg, dev, u, logit_bias=None):
    """The layer composed from the staged entry points on the tokens u, with the combine reducing
    each expert-output row itself (no row partial sums): the composition each expert-parallel
    rank runs.  Returns (out, topk_idx)."""
    T, n, k = u.shape[0], cfg.n_experts, cfg.top_k
    c = abi_config(cfg, T=T)
    E = cfg.expert_in
    dt = u.dtype
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    logits = torch.empty((T, n), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(c, u, dev["w_router"], logit_bias, logits, idx, w)
    x = u
    if cfg.latent:
        x = torch.empty((T, E), dtype=dt, device="cuda")
        moe.moe_latent_down(c, u, dev["p_down"], x)
    offsets = torch.empty(n + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((T * k, E), dtype=dt, device="cuda")
    moe.moe_permute(c, idx, offsets, perm, inv, x, dev.get("gamma_pre") if cfg.pre_norm else None,
                    x_perm, ws)
    s = torch.empty_like(x_perm)
    moe.moe_expert_ffn(c, x_perm, offsets, dev["w_gu"], dev["w_down"],
                       dev.get("gamma_expert") if cfg.expert_norm else None, s, ws)
    y = torch.empty((T, E), dtype=dt, device="cuda")
    moe.moe_combine(c, s, inv, w, y)
    out = y
    if cfg.latent:
        out = torch.empty_like(u)
        moe.moe_latent_up(c, y, dev["p_up"], u, dev.get("resid_g"), out)
    return out, idx


def make_ranks(cfg, dev, world, logit_bias=None):
    """R expert-parallel ranks over the whole-batch inputs: rank r holds experts
    expert_ranges(n, R)[r] and tokens [r T/R, (r+1) T/R)."""
    Tr = cfg.T // world
    ranks, us = [], []
    for r, (lo, hi) in enumerate(ep.expert_ranges(cfg.n_experts, world)):
        weights = dict(dev)
        weights["w_gu"] = dev["w_gu"][lo:hi]
        weights["w_down"] = dev["w_down"][lo:hi]
        if logit_bias is not None:
            weights["logit_bias"] = logit_bias
        ranks.append(ep.ExpertParallelRank(abi_config(cfg, T=Tr), weights, r, world))
        us.append(dev["u"][r * Tr:(r + 1) * Tr])
    return ranks, us


def _tiling(mean_rows: float, E: int, H: int) -> tuple:
    """The expert tilings the library picks from the mean rows per expert: the swapped 1-SM tiles
    up to 48 rows; above that the down GEMM on the swapped CTA-pair tiles up to 256 rows (when its
    output width is a multiple of 256 and its reduction at most 1024 deep), the 128-row activation
    tiles otherwise."""
    if mean_rows <= 48.0:
        return ("swap", "swap")
    return ("normal", "pair" if (E % 256 == 0 and H <= 1024 and mean_rows <= 256.0) else "normal")


def owner_orients(cfg, idx, world):
    """Whether each owner's expert GEMMs take the same tilings as the whole-batch ones (both pick
    them from the mean rows per expert)."""
    counts = np.bincount(idx.reshape(-1), minlength=cfg.n_experts)
    E, H = cfg.d_latent or cfg.d_model, cfg.d_ff
    whole = _tiling(counts.sum() / cfg.n_experts, E, H)
    return [_tiling(counts[lo:hi].sum() / (hi - lo), E, H) == whole
            for lo, hi in ep.expert_ranges(cfg.n_experts, world)]


EP_CASES = [
    configs.small_muse(T=2048, d=256, L=128, I=128, n=16, k=4, seed=91),
    configs.small_muse(T=2048, d=256, L=256, I=256, n=8, k=2, seed=92),   # several chunks / expert
    configs.small_shazeer(T=2048, d=128, h=256, n=16, k=4, seed=93),      # ReLU, no latent
]


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("cfg", EP_CASES, ids=lambda c: f"{c.name}-n{c.n_experts}")
def test_emulated_expert_parallel_equals_single_device(cfg, world):
    dev = moe_inputs.device_inputs(cfg)
    ref, idx = staged_layer(cfg, dev, dev["u"])
    ranks, us = make_ranks(cfg, dev, world)
    outs = ep.emulated_forward(ranks, us)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    assert all(owner_orients(cfg, idx.cpu().numpy(), world))
    got = torch.cat(outs)
    np.testing.assert_array_equal(got.view(torch.int16).cpu().numpy(),
                                  ref.view(torch.int16).cpu().numpy())
    # and the fused single-device layer (which may reduce the expert norms from the down GEMM's
    # row partials) within the bf16 tolerance
    fused = run_layer(cfg, dev, want_logits=False)["out"]
    err = row_rel_err(got.float().cpu().numpy(), fused.float().cpu().numpy())
    assert err.max() <= tolerance(cfg)


@pytest.mark.parametrize("world", [2, 4])
def test_emulated_expert_parallel_skewed_and_idle_owner(world):
    """Skewed routing where the last owner's experts are never chosen: that owner receives no
    rows, runs no expert, and returns nothing; the others see large and small groups."""
    cfg = configs.small_muse(T=2048, d=256, L=128, I=128, n=16, k=4, seed=94)
    dev = moe_inputs.device_inputs(cfg)
    n = cfg.n_experts
    bias = np.linspace(2.0, -2.0, n).astype(np.float32)
    bias[n - n // world:] = -1.0e4                       # never selected
    logit_bias = torch.from_numpy(bias).cuda()
    ref, idx = staged_layer(cfg, dev, dev["u"], logit_bias)
    assert int((idx >= n - n // world).sum()) == 0
    ranks, us = make_ranks(cfg, dev, world, logit_bias)
    outs = ep.emulated_forward(ranks, us)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    got = torch.cat(outs)
    same = owner_orients(cfg, idx.cpu().numpy(), world)[:-1]
    if all(same):
        np.testing.assert_array_equal(got.view(torch.int16).cpu().numpy(),
                                      ref.view(torch.int16).cpu().numpy())
    err = row_rel_err(got.float().cpu().numpy(), ref.float().cpu().numpy())
    assert err.max() <= tolerance(cfg)


@pytest.mark.parametrize("world", [2, 4])
def test_emulated_expert_parallel_decode_sized_ranks_match_oracle(world):
    """Decode-sized ranks (64 tokens each; the router's CUDA-core path): the expert-parallel
    layer against the oracle, token by token, within the bf16 tolerance."""
    cfg = separate(configs.small_muse(T=64 * world, d=256, L=128, I=128, n=16, k=4, seed=97))
    dev = moe_inputs.device_inputs(cfg)
    ranks, us = make_ranks(cfg, dev, world)
    got = device_values(torch.cat(ep.emulated_forward(ranks, us)))
    Tr = cfg.T // world
    idx = []
    for u in us:                       # the ranks' own routing (the same kernel as dispatch)
        c = abi_config(cfg, T=Tr)
        lg = torch.empty((Tr, cfg.n_experts), dtype=torch.float32, device="cuda")
        i = torch.empty((Tr, cfg.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((Tr, cfg.top_k), dtype=torch.float32, device="cuda")
        moe.moe_route(c, u, dev["w_router"], None, lg, i, w)
        idx.append(i.cpu().numpy())
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    ref = oracle_reference(cfg)
    ties = compare_selection(np.concatenate(idx), selection_keys(cfg, ref["logits"]), ref["idx"],
                             cfg.top_k)
    assert ties.sum() == 0
    err = row_rel_err(got, ref["out"])
    assert err.max() <= tolerance(cfg), f"max row error {err.max():.3e}"


# ------------------------------------------------------------------ batch invariance


@pytest.mark.parametrize("cfg", [configs.small_muse(T=2048, d=256, L=128, I=128, n=16, k=4,
                                                    seed=95),
                                 configs.small_shazeer(T=1024, d=128, h=256, n=16, k=4, seed=96)],
                         ids=lambda c: c.name)
def test_forward_is_batch_invariant(cfg):
    """moe_layer_forward on two halves of a batch gives the whole batch's bits (same GEMM
    orientation and router path at both sizes)."""
    dev = moe_inputs.device_inputs(cfg)
    whole = run_layer(cfg, dev, want_logits=False)["out"]
    h = cfg.T // 2
    halves = []
    for part in (slice(0, h), slice(h, cfg.T)):
        d = dict(dev)
        d["u"] = dev["u"][part]
        halves.append(run_layer(cfg.replace(T=h), d, want_logits=False)["out"])
    np.testing.assert_array_equal(torch.cat(halves).view(torch.int16).cpu().numpy(),
                                  whole.view(torch.int16).cpu().numpy())
