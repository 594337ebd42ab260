"""Parity of the CUDA path (called through the C ABI) with the CPU oracle on seeded inputs.

Routing indices and the dispatch permutation are compared bit for bit; values within the
tolerance of the storage dtype (max over tokens of |out - ref|_inf / |ref|_inf <= 2e-2 for bf16,
1e-4 for fp32, against the double-accumulating oracle).
"""
import numpy as np
import pytest

import moe_inputs
import oracle
from moe_inputs import configs

from gpu_harness import (abi_config, check_routing, compare_selection, device_values, host_values,
                         logit_atol, oracle_reference, row_rel_err, run_layer, selection_keys,
                         separate, tolerance)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_layer_softmax_b200")


@pytest.fixture(autouse=True)
def _cuda_cleanup():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ input generator


def test_generator_device_matches_host():
    for seed, stream, first, count, sigma in ((0, 1, 0, 100003, 1.0), (3, 5, 12345, 4099, 0.02),
                                              (4, 6, 1 << 33, 777, 0.5)):
        t = torch.empty(count, dtype=torch.bfloat16, device="cuda")
        moe_inputs.normal_device(t, seed, stream, first, sigma)
        h = moe_inputs.normal_host(seed, stream, first, count, sigma, "bf16")
        np.testing.assert_array_equal(t.view(torch.int16).cpu().numpy().view(np.uint16), h)
        f = torch.empty(count, dtype=torch.float32, device="cuda")
        moe_inputs.normal_device(f, seed, stream, first, sigma)
        np.testing.assert_array_equal(f.cpu().numpy(), moe_inputs.normal_host(seed, stream, first,
                                                                             count, sigma, "f32"))
        moe_inputs.uniform_device(f, seed, stream, first)
        np.testing.assert_array_equal(f.cpu().numpy(), moe_inputs.uniform_host(seed, stream, first,
                                                                              count))
    # a workload with redrawn input rows (separated router logits): the same rows on both sides
    cfg = configs.MUSE_DECODE
    assert cfg.u_redraw
    u = moe_inputs.device_inputs(cfg)["u"]
    np.testing.assert_array_equal(u.view(torch.int16).cpu().numpy().view(np.uint16),
                                  moe_inputs.host_rows(cfg, "u"))


# ------------------------------------------------------------------ whole layer, small shapes

SMALL = [
    # normal orientation, ragged T, several M tiles, Muse structure
    configs.small_muse(T=300, d=512, L=256, I=256, n=16, k=4, seed=11),
    # CTA-pair tiles (>= 192 rows per expert; dense projections with T >= 256), ragged groups
    configs.small_muse(T=517, d=512, L=256, I=256, n=4, k=2, seed=22),
    configs.small_muse(T=1100, d=256, L=256, I=512, n=8, k=2, seed=23,
                       resid_mode=configs.RESID_LITERAL),
    # swap orientation (few rows per expert), max experts and top-k
    configs.small_muse(T=40, d=256, L=128, I=128, n=256, k=8, seed=12),
    configs.small_muse(T=77, d=256, L=256, I=128, n=64, k=8, seed=13),
    # residual variants and no pre-norm
    configs.small_muse(T=130, d=256, L=128, I=192, n=8, k=2, seed=14,
                       resid_mode=configs.RESID_LITERAL),
    configs.small_muse(T=65, d=192, L=128, I=128, n=8, k=3, seed=15, pre_norm=0,
                       resid_mode=configs.RESID_NONE),
    # k = 1 (one-hot gate) and k = n (dense softmax mixture)
    configs.small_muse(T=129, d=256, L=128, I=128, n=8, k=1, seed=16),
    configs.small_muse(T=50, d=256, L=128, I=128, n=8, k=8, seed=17),
    # Shazeer structure in bf16 (ReLU experts, no latent, no norm)
    configs.small_shazeer(T=257, d=128, h=256, n=16, k=4, seed=18),
    configs.small_shazeer(T=33, d=256, h=512, n=64, k=2, seed=19),
    # 49-256 rows per expert with a 256-wide expert output: the down GEMM on the CTA-pair tiles
    configs.small_shazeer(T=600, d=256, h=512, n=16, k=4, seed=31),
    # fp32 CUDA-core path
    configs.TINY_SHAZEER_F32.replace(T=45, seed=20),
    configs.TINY_SHAZEER_F32.replace(T=64, top_k=8, seed=21),
    # Muse sigmoid gate: fp32 router weights (exact bf16 split) on the GEMM router (T > 256)
    # and on the few-token router, bf16 router weights, and the fp32 layer
    configs.small_muse(T=300, d=512, L=256, I=256, n=16, k=4, seed=25, gate_mode=configs.GATE_SIGMOID,
                       router_f32=1, logit_mult=2.0, corr_sigma=0.3, routed_scale=1.5),
    configs.small_muse(T=40, d=256, L=128, I=128, n=64, k=8, seed=26,
                       gate_mode=configs.GATE_SIGMOID, router_f32=1),
    configs.small_muse(T=96, d=256, L=128, I=128, n=32, k=4, seed=27,
                       gate_mode=configs.GATE_SIGMOID, corr_sigma=0.2),
    configs.TINY_SHAZEER_F32.replace(T=50, seed=24, gate_mode=configs.GATE_SIGMOID,
                                     logit_mult=0.5, router_gain=1.0),
    # decoder wrap: residual-stream norm in, FFN output norm before the residual gate
    configs.small_muse(T=300, d=512, L=256, I=256, n=16, k=4, seed=28, input_norm=1, post_norm=1,
                       gamma_sigma=0.2),
    configs.small_muse(T=40, d=256, L=128, I=128, n=64, k=8, seed=29, input_norm=1, post_norm=1,
                       resid_mode=configs.RESID_LITERAL),
    configs.small_muse(T=70, d=8192, L=128, I=128, n=8, k=2, seed=30, input_norm=1, post_norm=0),
]


PAIR_CASES = [c for c in SMALL if c.T in (517, 1100)]
# layers whose expert groups are prefill-sized (more than 48 rows per expert on average)
PREFILL_GROUP_CASES = [c for c in SMALL if c.T * c.top_k / c.n_experts > 48]


@pytest.mark.parametrize("cfg", PREFILL_GROUP_CASES, ids=lambda c: c.name)
def test_layer_small_swap_pair_expert_tiles(cfg, monkeypatch):
    """The same layers with the prefill expert GEMMs on the swapped CTA-pair tiles
    (MOE_EXPERT_TILES=swap_pair) instead of the 1-SM 128-row activation tiles."""
    monkeypatch.setenv("MOE_EXPERT_TILES", "swap_pair")
    _check_layer(cfg)


@pytest.mark.parametrize("cfg", PREFILL_GROUP_CASES, ids=lambda c: c.name)
def test_layer_small_normal_expert_tiles(cfg, monkeypatch):
    """The same layers with both expert GEMMs on the 1-SM 128-row activation tiles
    (MOE_EXPERT_TILES=normal), whatever the rows per expert."""
    monkeypatch.setenv("MOE_EXPERT_TILES", "normal")
    _check_layer(cfg)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"{c.name}-n{c.n_experts}k{c.top_k}-{c.dtype}"
                         f"-r{c.resid_mode}p{c.pre_norm}")
def test_layer_small(cfg):
    _check_layer(cfg)


# batch sizes at the layer's switch points: one token; the split latent projections (T <= 64);
# the few-token router (T <= 256); the one-launch dispatch (T * k <= 2048 slots)
EDGE_CASES = [configs.small_muse(T=T, d=512, L=256, I=256, n=16, k=4, seed=200 + T)
              for T in (1, 2, 63, 64, 65)] + \
             [configs.small_muse(T=T, d=256, L=128, I=128, n=64, k=8, seed=300 + T)
              for T in (255, 256, 257)]


@pytest.mark.parametrize("cfg", EDGE_CASES, ids=lambda c: f"T{c.T}-n{c.n_experts}k{c.top_k}")
def test_layer_at_switch_points(cfg):
    _check_layer(cfg)


def test_dense_pair_tiles_at_prefill_size(monkeypatch):
    """From 2048 rows the latent projections run on CTA-pair 256-row tiles by default: the layer
    matches the oracle, and gives the same bits as with every GEMM on the 1-SM tiles
    (MOE_GEMM_PAIR=0)."""
    import torch
    raw = configs.small_muse(T=2304, d=512, L=256, I=128, n=16, k=4, seed=310)
    _check_layer(raw)
    cfg = separate(raw)
    dev = moe_inputs.device_inputs(cfg)
    a = run_layer(cfg, dev, want_logits=False)["out"]
    monkeypatch.setenv("MOE_GEMM_PAIR", "0")
    b = run_layer(cfg, dev, want_logits=False)["out"]
    torch.cuda.synchronize()
    np.testing.assert_array_equal(a.view(torch.int16).cpu().numpy(), b.view(torch.int16).cpu().numpy())


def test_layer_empty_batch():
    """T = 0: the forward launches nothing that touches the (empty) buffers and reports success."""
    import torch
    cfg = configs.small_muse(T=0, d=256, L=128, I=128, n=16, k=4, seed=399)
    c = abi_config(cfg)
    dev = moe_inputs.device_inputs(cfg.replace(T=1))
    layer = moe.MoELayer(c, dev)
    u = torch.empty((0, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(u)
    layer.forward(u, u, out=out)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0


@pytest.mark.parametrize("cfg", PAIR_CASES, ids=lambda c: c.name)
def test_layer_small_pair_tiles(cfg, monkeypatch):
    """The same layers with the CTA-pair 256-row GEMM tiles selected (MOE_GEMM_PAIR=1)."""
    monkeypatch.setenv("MOE_GEMM_PAIR", "1")
    _check_layer(cfg)


def _check_layer(cfg):
    cfg = separate(cfg)  # router inputs separated at the top-k boundary: no token is skipped
    dev = moe_inputs.device_inputs(cfg)
    res = run_layer(cfg, dev)
    ref = oracle_reference(cfg)
    logits = res["logits"].cpu().numpy()
    idx = res["idx"].cpu().numpy()
    check_routing(cfg, logits, idx, res["w"].cpu().numpy())
    ties = compare_selection(idx, selection_keys(cfg, ref["logits"]), ref["idx"], cfg.top_k)
    assert ties.sum() == 0
    np.testing.assert_allclose(logits, ref["logits"], rtol=0, atol=logit_atol(cfg, logits))
    err = row_rel_err(device_values(res["out"]), ref["out"])
    assert err.max() <= tolerance(cfg), f"max row error {err.max():.3e}"


# ------------------------------------------------------------------ individual entry points


def test_router_split_is_exact():
    """hi + mid + lo reconstructs every fp32 router weight exactly."""
    w = torch.empty((64, 512), dtype=torch.float32, device="cuda")
    moe_inputs.normal_device(w, 3, 90, 0, 0.7)
    w[0, :8] = torch.tensor([0.0, -0.0, 1.0, -3.0e-5, 1.0e4, 1.0 / 3.0, 2.0 ** -100, 65504.0])
    parts = moe.router_split(w).view(64, 3, 512).double()
    np.testing.assert_array_equal(parts.sum(1).cpu().numpy(), w.double().cpu().numpy())


def _rand_routing(T, n, k, seed, hot=None):
    rng = np.random.default_rng(seed)
    p = None
    if hot is not None:
        p = np.full(n, (1 - hot) / (n - 1))
        p[0] = hot
    return np.stack([rng.choice(n, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,n,k,hot", [(1, 4, 2, None), (129, 16, 4, None), (1000, 256, 8, None),
                                       (513, 64, 3, 0.9), (300, 256, 1, None), (64, 8, 8, None)])
def test_permute_bit_exact(T, n, k, hot):
    cfg = configs.small_muse(T=T, n=n, k=k)
    c = abi_config(cfg)
    idx = _rand_routing(T, n, k, seed=T + n, hot=hot)
    d_idx = torch.from_numpy(idx).cuda()
    off = torch.full((n + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    moe.moe_permute(c, d_idx, off, perm, inv, workspace=ws)
    assert moe.moe_get_device_status() == 0
    r_off, r_perm, r_inv = oracle.permutation(T, k, n, idx)
    np.testing.assert_array_equal(off.cpu().numpy(), r_off)
    np.testing.assert_array_equal(perm.cpu().numpy(), r_perm)
    np.testing.assert_array_equal(inv.cpu().numpy(), r_inv)


def test_permute_empty_and_bad_index():
    cfg = configs.small_muse(T=0, n=16, k=4)
    c = abi_config(cfg)
    off = torch.full((17,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    moe.moe_permute(c, None, off, None, None, workspace=ws)
    assert moe.moe_get_device_status() == 0
    assert (off.cpu().numpy() == 0).all()
    # an out-of-range expert index is latched as a device check error and the slot dropped
    cfg = configs.small_muse(T=3, n=4, k=2)
    c = abi_config(cfg)
    idx = torch.tensor([[0, 1], [2, 9], [3, 0]], dtype=torch.int32, device="cuda")
    off = torch.zeros(5, dtype=torch.int32, device="cuda")
    perm = torch.zeros(6, dtype=torch.int32, device="cuda")
    inv = torch.zeros(6, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    moe.moe_permute(c, idx, off, perm, inv, workspace=ws)
    assert moe.moe_get_device_status() == moe.STATUS_CODES["MOE_ERR_DEVICE_CHECK"]
    assert moe.moe_get_device_status() == 0  # cleared by the read
    assert off.cpu().numpy().tolist() == [0, 2, 3, 4, 5]
    assert inv.cpu().numpy()[3] == -1


@pytest.mark.parametrize("T,k,n", [(500, 8, 16), (3000, 4, 256)])
def test_permute_chunked_bad_index(T, k, n):
    """The chunked permutation (more than 2048 slots: counts, scan and rank over several chunks)
    with an expert index out of range: the error is latched, that slot is dropped, and the other
    slots keep the canonical order (offsets from the valid counts; rows by expert, then token)."""
    idx_h = _rand_routing(T, n, k, seed=T + n)
    idx_h[T // 2, 1] = n + 3
    cfg = configs.small_muse(T=T, n=n, k=k)
    c = abi_config(cfg)
    off = torch.zeros(n + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    inv = torch.zeros(T * k, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    moe.moe_permute(c, torch.from_numpy(idx_h).cuda(), off, perm, inv, workspace=ws)
    assert moe.moe_get_device_status() == moe.STATUS_CODES["MOE_ERR_DEVICE_CHECK"]
    flat = idx_h.reshape(-1)
    valid = flat < n
    counts = np.bincount(flat[valid], minlength=n)
    np.testing.assert_array_equal(off.cpu().numpy(), np.concatenate([[0], np.cumsum(counts)]))
    slots = np.nonzero(valid)[0]
    order = slots[np.lexsort((slots // k, flat[slots]))]  # expert ascending, then token
    want_inv = np.full(T * k, -1)
    want_inv[order] = np.arange(len(order))
    np.testing.assert_array_equal(inv.cpu().numpy(), want_inv)
    np.testing.assert_array_equal(perm.cpu().numpy()[:len(order)], order // k)


@pytest.mark.parametrize("E,gamma", [(256, True), (4096, True), (512, False), (8192, True)])
def test_scatter_rows_with_centred_norm(E, gamma):
    T, n, k = 37, 8, 3
    cfg = configs.small_muse(T=T, d=E, L=E, I=128, n=n, k=k)
    c = abi_config(cfg)
    x_h = moe_inputs.normal_host(5, 40, 0, T * E, 1.7, "bf16").reshape(T, E)
    g_h = moe_inputs.normal_host(5, 41, 0, E, 0.3, "f32")
    idx = _rand_routing(T, n, k, seed=E)
    x = torch.from_numpy(x_h.view(np.int16)).view(torch.bfloat16).cuda()
    g = torch.from_numpy(g_h).cuda()
    off = torch.empty(n + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    xp = torch.empty((T * k, E), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    moe.moe_permute(c, torch.from_numpy(idx).cuda(), off, perm, inv, x=x,
                    gamma_pre=g if gamma else None, x_perm=xp, workspace=ws)
    assert moe.moe_get_device_status() == 0
    xv = host_values(x_h, "bf16")
    _, _, r_inv = oracle.permutation(T, k, n, idx)
    got = device_values(xp)
    for t in range(T):
        ref = oracle.centered_rmsnorm(xv[t], g_h.astype(np.float64), cfg.eps) if gamma else xv[t]
        ref = oracle.bf16_round(ref)
        for j in range(k):
            row = got[r_inv[t * k + j]]
            if gamma:
                assert row_rel_err(row, ref) <= 1e-2
            else:
                np.testing.assert_array_equal(row, ref)


@pytest.mark.parametrize("cfg", [
    configs.small_muse(T=200, d=256, L=256, I=384, n=8, k=2, seed=31),    # normal orientation
    configs.small_muse(T=24, d=256, L=256, I=256, n=64, k=8, seed=32),    # swap orientation
    configs.small_muse(T=700, d=256, L=256, I=256, n=4, k=2, seed=35),    # CTA-pair tiles
    configs.small_shazeer(T=900, d=256, h=512, n=4, k=2, seed=36),        # pair tiles, ReLU
    configs.small_shazeer(T=300, d=128, h=256, n=8, k=2, seed=33),
    configs.small_shazeer(T=20, d=128, h=256, n=64, k=4, seed=34),
], ids=lambda c: f"{c.name}-n{c.n_experts}k{c.top_k}-act{c.act}")
def test_expert_ffn(cfg, monkeypatch):
    """Experts on dispatched rows (inputs from the generator, routing synthetic); the large-group
    cases run with the CTA-pair tiles selected."""
    if cfg.T in (700, 900):
        monkeypatch.setenv("MOE_GEMM_PAIR", "1")
    c = abi_config(cfg)
    T, k, n, E, H = cfg.T, cfg.top_k, cfg.n_experts, cfg.expert_in, cfg.d_ff
    idx = _rand_routing(T, n, k, seed=cfg.seed)
    off, perm, inv = oracle.permutation(T, k, n, idx)
    xh = moe_inputs.normal_host(cfg.seed, 50, 0, T * k * E, 1.0, "bf16").reshape(T * k, E)
    gam = moe_inputs.host_rows(cfg, "gamma_expert") if cfg.expert_norm else None
    w_gu = moe_inputs.host_rows(cfg, "w_gu")
    w_dn = moe_inputs.host_rows(cfg, "w_down")
    dev = moe_inputs.device_inputs(cfg)
    x = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).cuda()
    out = torch.empty((T * k, E), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    parts = moe.row_sumsq_parts(c)
    ss = torch.full((T * k, parts), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn(c, x, torch.from_numpy(off).cuda(), dev["w_gu"], dev["w_down"],
                       dev.get("gamma_expert"), out, workspace=ws,
                       row_sumsq=ss if cfg.expert_norm else None)
    assert moe.moe_get_device_status() == 0
    got = device_values(out)
    if cfg.expert_norm:
        # the partials partition each row: their sum is the row's sum of squares of the stored
        # bf16 values (fp32 sums of up to 256 terms each)
        tot = ss.double().sum(1).cpu().numpy()
        np.testing.assert_allclose(tot, (got * got).sum(1), rtol=2e-5, atol=1e-30)
    errs = _expert_rows_vs_oracle(cfg, off, host_values(xh, "bf16"), got, w_gu, w_dn, gam)
    assert errs.max() <= 2e-2


def _expert_rows_vs_oracle(cfg, off, xv, got, w_gu, w_dn, gam):
    """Row errors of expert outputs (dispatch order) against the oracle's pre-norm expert output
    s (the vector I_gamma reduces with expert_norm, else o) on the same input rows."""
    oc = oracle.make_cfg(cfg)
    E = cfg.expert_in
    gp = None if gam is None else np.ascontiguousarray(gam, dtype=np.float32)
    errs = []
    for e in range(cfg.n_experts):
        rows = np.arange(off[e], off[e + 1])
        if len(rows) == 0:
            continue
        ref = np.zeros((len(rows), E))
        nrm = np.zeros((len(rows), E))
        wg = np.ascontiguousarray(w_gu[e])
        wd = np.ascontiguousarray(w_dn[e])
        zr = np.ascontiguousarray(xv[rows])
        oracle.lib().orc_expert_batch_parts(oracle.ctypes.byref(oc), wg.ctypes.data,
                                            wd.ctypes.data, None if gp is None else gp.ctypes.data,
                                            zr.ctypes.data, len(rows), ref.ctypes.data,
                                            nrm.ctypes.data, 4)
        errs.append(row_rel_err(got[rows], ref))
    return np.concatenate(errs)


# group sizes around the swapped pair tiles' 16-row and 256-row steps, an empty group and a hot
# group of many chunks
PAIR_GROUPS = [0, 1, 15, 16, 17, 255, 256, 257, 511, 513, 1000, 40, 3000]


@pytest.mark.parametrize("tiles", ["swap_pair", "normal"])
@pytest.mark.parametrize("cfg", [
    configs.small_muse(T=sum(PAIR_GROUPS), d=256, L=256, I=256, n=len(PAIR_GROUPS), k=1, seed=37),
    configs.small_muse(T=sum(PAIR_GROUPS), d=256, L=128, I=384, n=len(PAIR_GROUPS), k=1, seed=38),
    configs.small_shazeer(T=sum(PAIR_GROUPS), d=256, h=512, n=len(PAIR_GROUPS), k=1, seed=39),
], ids=lambda c: f"{c.name}-L{c.expert_in}-I{c.d_ff}-act{c.act}")
def test_expert_ffn_prefill_tiles(cfg, tiles, monkeypatch):
    """Prefill-sized expert groups of chosen sizes on the swapped CTA-pair tiles (tokens on the
    MMA's N side, chunks cut to 16 rows) and on the 1-SM 128-row tiles: each against the oracle,
    and the row partial sums of squares against the stored rows.  (A 128-wide latent is not a
    multiple of the pair's 256 down-projection features: that down GEMM keeps the 1-SM tiles.)"""
    monkeypatch.setenv("MOE_EXPERT_TILES", tiles)
    c = abi_config(cfg)
    n, E = cfg.n_experts, cfg.expert_in
    counts = np.array(PAIR_GROUPS)
    idx = np.repeat(np.arange(n, dtype=np.int32), counts).reshape(-1, 1)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    TK = int(off[-1])
    xh = moe_inputs.normal_host(cfg.seed, 50, 0, TK * E, 1.0, "bf16").reshape(TK, E)
    gam = moe_inputs.host_rows(cfg, "gamma_expert") if cfg.expert_norm else None
    dev = moe_inputs.device_inputs(cfg)
    x = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).cuda()
    out = torch.empty((TK, E), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    parts = moe.row_sumsq_parts(c)
    ss = torch.full((TK, parts), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn(c, x, torch.from_numpy(off).cuda(), dev["w_gu"], dev["w_down"],
                       dev.get("gamma_expert"), out, workspace=ws,
                       row_sumsq=ss if cfg.expert_norm else None)
    assert moe.moe_get_device_status() == 0
    got = device_values(out)
    if cfg.expert_norm:
        tot = ss.double().sum(1).cpu().numpy()
        np.testing.assert_allclose(tot, (got * got).sum(1), rtol=2e-5, atol=1e-30)
    errs = _expert_rows_vs_oracle(cfg, off, host_values(xh, "bf16"),
                                  got, moe_inputs.host_rows(cfg, "w_gu"),
                                  moe_inputs.host_rows(cfg, "w_down"), gam)
    print(f"{tiles}: parts {parts}, max row rel err {errs.max():.3e}")
    assert errs.max() <= 2e-2
    del idx


@pytest.mark.parametrize("with_ss", [False, True], ids=["reduce", "row_sumsq"])
@pytest.mark.parametrize("E,k,norm", [(128, 4, 1), (4096, 8, 1), (512, 4, 0), (1024, 1, 1)])
def test_combine(E, k, norm, with_ss):
    """Normalise + combine, with the row norms reduced in the kernel or taken from partial sums
    of squares (here the host's: the whole row's sum in part 0, zeros in the others)."""
    T, n = 45, 16
    cfg = configs.small_muse(T=T, d=E, L=E, I=128, n=n, k=k, expert_norm=norm)
    c = abi_config(cfg)
    idx = _rand_routing(T, n, k, seed=E + k)
    _, _, inv = oracle.permutation(T, k, n, idx)
    sh = moe_inputs.normal_host(9, 60, 0, T * k * E, 0.8, "bf16").reshape(T * k, E)
    wr = moe_inputs.uniform_host(9, 61, 0, T * k).reshape(T, k).astype(np.float64) + 0.05
    wr = (wr / wr.sum(1, keepdims=True)).astype(np.float32)
    y = torch.empty((T, E), dtype=torch.bfloat16, device="cuda")
    ss = None
    if with_ss:
        sv64 = host_values(sh, "bf16")
        parts = np.zeros((T * k, moe.row_sumsq_parts(c)), dtype=np.float32)
        parts[:, 0] = (sv64 * sv64).sum(1)
        ss = torch.from_numpy(parts).cuda()
    moe.moe_combine(c, torch.from_numpy(sh.view(np.int16)).view(torch.bfloat16).cuda(),
                    torch.from_numpy(inv).cuda(), torch.from_numpy(wr).cuda(), y, row_sumsq=ss)
    assert moe.moe_get_device_status() == 0
    sv = host_values(sh, "bf16")
    oc = oracle.make_cfg(cfg)
    got = device_values(y)
    zero = np.zeros(E)
    for t in range(T):
        ns = np.zeros((k, E))
        for j in range(k):
            s = sv[inv[t * k + j]]
            ns[j] = oracle.bf16_round(oracle.input_scaled_rmsnorm(s, zero, cfg.eps, 1)) if norm else s
        ref = np.zeros(E)
        wj = wr[t].astype(np.float64)
        oracle.lib().orc_combine_token(oracle.ctypes.byref(oc), np.ascontiguousarray(ns).ctypes.data,
                                       wj.ctypes.data, ref.ctypes.data)
        assert row_rel_err(got[t], ref) <= 1e-2


@pytest.mark.parametrize("E,k,norm", [(4096, 8, 1), (4096, 4, 0), (8192, 2, 1)])
def test_combine_bulk_matches_per_token(E, k, norm):
    """The prefill combine (persistent CTAs, expert rows by bulk copies; from 1024 tokens whose k
    expert rows hold at least 32 KB) against
    the per-token combine on the same rows, bit for bit (two calls of fewer tokens each), and
    against the oracle on sampled tokens; a few slots are dropped (negative dispatch row)."""
    T, n = 1500, 16
    cfg = configs.small_muse(T=T, d=E, L=E, I=128, n=n, k=k, expert_norm=norm)
    idx = _rand_routing(T, n, k, seed=E + 3 * k)
    _, _, inv = oracle.permutation(T, k, n, idx)
    inv = inv.copy()
    inv[[5, 777 * k + k - 1, (T - 1) * k]] = -1
    sh = moe_inputs.normal_host(10, 60, 0, T * k * E, 0.8, "bf16").reshape(T * k, E)
    wr = moe_inputs.uniform_host(10, 61, 0, T * k).reshape(T, k).astype(np.float64) + 0.05
    wr = (wr / wr.sum(1, keepdims=True)).astype(np.float32)
    sv = host_values(sh, "bf16")
    s_d = torch.from_numpy(sh.view(np.int16)).view(torch.bfloat16).cuda()
    inv_d = torch.from_numpy(inv).cuda()
    w_d = torch.from_numpy(wr).cuda()
    c = abi_config(cfg)
    ss = None
    if norm:
        parts = np.zeros((T * k, moe.row_sumsq_parts(c)), dtype=np.float32)
        parts[:, 0] = (sv * sv).sum(1)
        parts[:, -1] = 0.0
        ss = torch.from_numpy(parts).cuda()
    y = torch.empty((T, E), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(c, s_d, inv_d, w_d, y, row_sumsq=ss)
    h = T // 2  # below the bulk path's threshold: the per-token kernel
    y2 = torch.empty_like(y)
    for part in (slice(0, h), slice(h, T)):
        ch = abi_config(cfg.replace(T=part.stop - part.start))
        moe.moe_combine(ch, s_d, inv_d[part.start * k:part.stop * k], w_d[part], y2[part],
                        row_sumsq=ss)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy(),
                                  y2.view(torch.int16).cpu().numpy())
    got = device_values(y)
    oc = oracle.make_cfg(cfg)
    zero = np.zeros(E)
    for t in list(range(0, T, 97)) + [777, T - 1]:
        ns = np.zeros((k, E))
        for j in range(k):
            r = inv[t * k + j]
            if r < 0:
                continue
            ns[j] = oracle.bf16_round(oracle.input_scaled_rmsnorm(sv[r], zero, cfg.eps, 1)) \
                if norm else sv[r]
        ref = np.zeros(E)
        wj = wr[t].astype(np.float64) * (inv[t * k:(t + 1) * k] >= 0)
        oracle.lib().orc_combine_token(oracle.ctypes.byref(oc), np.ascontiguousarray(ns).ctypes.data,
                                       wj.ctypes.data, ref.ctypes.data)
        assert row_rel_err(got[t], ref) <= 1e-2


@pytest.mark.parametrize("T", [150, 64, 17, 1])
def test_latent_down_and_up(T):
    """The standalone latent projections against the oracle: over 64 rows one GEMM; up to 64 rows
    the reduction split over clusters of 8 (down) and 4 (up) CTAs that add their partial tiles in
    distributed shared memory."""
    cfg = configs.small_muse(T=T, d=512, L=256, I=128, n=8, k=2, seed=41)
    c = abi_config(cfg)
    dev = moe_inputs.device_inputs(cfg)
    inp = moe_inputs.host_inputs(cfg)
    z = torch.empty((cfg.T, cfg.d_latent), dtype=torch.bfloat16, device="cuda")
    moe.moe_latent_down(c, dev["u"], dev["p_down"], z)
    yh = moe_inputs.normal_host(41, 70, 0, cfg.T * cfg.d_latent, 0.7, "bf16").reshape(cfg.T, -1)
    out = torch.empty_like(dev["u"])
    moe.moe_latent_up(c, torch.from_numpy(yh.view(np.int16)).view(torch.bfloat16).cuda(),
                      dev["p_up"], dev["u"], dev["resid_g"], out)
    assert moe.moe_get_device_status() == 0
    oc = oracle.make_cfg(cfg.replace(pre_norm=0))
    keep = oracle._Keep()
    x = oracle.make_tensors(cfg, inp, keep)
    zg, og = device_values(z), device_values(out)
    yv = host_values(yh, "bf16")
    for t in range(cfg.T):
        zr = np.zeros(cfg.d_latent)
        oracle.lib().orc_expert_input_token(oracle.ctypes.byref(oc), oracle.ctypes.byref(x), t,
                                            zr.ctypes.data)
        assert row_rel_err(zg[t], zr) <= 1e-2
        o = np.zeros(cfg.d_model)
        yt = np.ascontiguousarray(yv[t])
        oracle.lib().orc_output_token(oracle.ctypes.byref(oc), oracle.ctypes.byref(x), t,
                                      yt.ctypes.data, o.ctypes.data)
        assert row_rel_err(og[t], o) <= 1e-2


# ------------------------------------------------------------------ failure detection


def test_bounded_wait_runs_out_and_reports():
    """A wait on a barrier nothing arrives at gives up after its budget, latches MOE_ERR_TIMEOUT
    in the status word, and the context stays usable."""
    gave_up = torch.zeros(4, dtype=torch.int32, device="cuda")
    rc = moe.lib().moe_selftest_wait_timeout(2_000_000, gave_up.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    assert moe.moe_get_device_status() == moe.STATUS_CODES["MOE_ERR_TIMEOUT"]
    assert gave_up[0].item() == 1
    assert moe.moe_get_device_status() == 0
    # the device still runs work correctly afterwards
    cfg = configs.small_muse(T=40, d=256, L=128, I=128, n=16, k=4, seed=77)
    _check_layer(cfg)


ROUTE_CASES = [
    configs.small_shazeer(T=300, d=256, h=256, n=64, k=4, seed=71),
    configs.small_muse(T=513, d=256, L=128, I=128, n=256, k=8, seed=72),
    configs.small_muse(T=400, d=256, L=128, I=128, n=48, k=6, seed=73, gate_mode=configs.GATE_SIGMOID,
                       logit_mult=1.5),
    configs.MUSE_IMBALANCED.replace(T=700, seed=74),   # Zipf logit bias on the large-T path
]


@pytest.mark.parametrize("cfg", ROUTE_CASES, ids=lambda c: f"{c.name}-n{c.n_experts}-k{c.top_k}")
def test_route_without_logits_buffer_matches(cfg):
    """moe_route beyond the small-batch path: with a logits buffer the GEMM stores logits and a
    warp per token selects; without one the GEMM epilogue selects from its accumulators.  Both
    must give the same experts and the same weights, bit for bit, and the selection must be the
    oracle's on the GPU's logits."""
    import torch
    dev = moe_inputs.device_inputs(cfg)
    c = abi_config(cfg)
    T, n, k = cfg.T, cfg.n_experts, cfg.top_k
    bias = dev.get("logit_bias")
    corr = dev.get("correction_bias")
    logits = torch.empty((T, n), dtype=torch.float32, device="cuda")
    idx1 = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w1 = torch.empty((T, k), dtype=torch.float32, device="cuda")
    idx2, w2 = torch.empty_like(idx1), torch.empty_like(w1)
    moe.moe_route(c, dev["u"], dev["w_router"], bias, logits, idx1, w1, correction_bias=corr)
    moe.moe_route(c, dev["u"], dev["w_router"], bias, None, idx2, w2, correction_bias=corr)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    np.testing.assert_array_equal(idx2.cpu().numpy(), idx1.cpu().numpy())
    np.testing.assert_array_equal(w2.cpu().numpy().view(np.int32), w1.cpu().numpy().view(np.int32))
    lg = logits.cpu().numpy()
    if cfg.gate_mode == configs.GATE_SIGMOID:
        sel, wsel = oracle.sigmoid_topk_scores_f32(lg, k, corr.cpu().numpy(), cfg.routed_scale)
    else:
        sel, wsel = oracle.softmax_topk(lg, k)
    np.testing.assert_array_equal(idx1.cpu().numpy(), sel)
    np.testing.assert_allclose(w1.cpu().numpy(), wsel, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T", [40, 300])
def test_route_with_masked_experts(T):
    """A logit bias of -inf on n-k+1 experts leaves fewer than k finite logits: the selection
    takes the k-1 finite ones, then the lowest-index masked expert with weight 0 (the oracle's
    order on the same logits), every index distinct, on the few-token router, the warp-per-token
    top-k after the GEMM router, and the GEMM epilogue's own selection."""
    import torch
    cfg = configs.small_muse(T=T, d=256, L=128, I=128, n=32, k=4, seed=75)
    dev = moe_inputs.device_inputs(cfg)
    c = abi_config(cfg)
    n, k = cfg.n_experts, cfg.top_k
    rng = np.random.default_rng(76)
    masked = rng.choice(n, size=n - k + 1, replace=False)
    bias_h = np.zeros(n, dtype=np.float32)
    bias_h[masked] = -np.inf
    bias = torch.from_numpy(bias_h).cuda()
    logits = torch.empty((T, n), dtype=torch.float32, device="cuda")
    outs = []
    for lg in (logits, None):
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        moe.moe_route(c, dev["u"], dev["w_router"], bias, lg, idx, w)
        outs.append((idx, w))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    lgh = logits.cpu().numpy()
    sel, wsel = oracle.softmax_topk(lgh, k)
    first_masked = np.sort(masked)[0]
    for idx, w in outs:
        ih, wh = idx.cpu().numpy(), w.cpu().numpy()
        np.testing.assert_array_equal(ih, sel)
        assert all(len(set(r)) == k for r in ih.tolist())
        assert (ih[:, -1] == first_masked).all()
        assert (wh[:, -1] == 0.0).all()
        np.testing.assert_allclose(wh, wsel, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T", [40, 300])
def test_route_exact_ties_take_lower_index(T):
    """Router weight rows copied between experts give bit-equal logits for every token: the
    selection must take the lower expert index first wherever such a pair meets at or inside the
    top k, as the oracle's order on the same logits does, on the few-token router, the
    warp-per-token top-k after the GEMM router and the GEMM epilogue's own selection."""
    import torch
    cfg = configs.small_muse(T=T, d=256, L=128, I=128, n=64, k=8, seed=77)
    dev = moe_inputs.device_inputs(cfg)
    c = abi_config(cfg)
    n, k = cfg.n_experts, cfg.top_k
    w = dev["w_router"].clone()
    pairs = [(3, 17), (40, 5), (22, 63), (9, 10), (31, 0), (50, 51), (12, 48), (60, 33)]
    for a, b in pairs:
        w[b] = w[a]
    logits = torch.empty((T, n), dtype=torch.float32, device="cuda")
    outs = []
    for lg in (logits, None):
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
        moe.moe_route(c, dev["u"], w, None, lg, idx, wt)
        outs.append((idx, wt))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    lgh = logits.cpu().numpy()
    for a, b in pairs:
        np.testing.assert_array_equal(lgh[:, a].view(np.int32), lgh[:, b].view(np.int32))
    sel, wsel = oracle.softmax_topk(lgh, k)
    # the copies meet inside the top k, or at its boundary, on many tokens
    hit = sum(int(np.isin([a, b], sel[t]).all()) for t in range(T) for a, b in pairs)
    assert hit >= T // 8
    for idx, wt in outs:
        np.testing.assert_array_equal(idx.cpu().numpy(), sel)
        np.testing.assert_allclose(wt.cpu().numpy(), wsel, rtol=2e-6, atol=1e-7)


STAGED_CASES = [
    configs.small_muse(T=300, d=256, L=128, I=128, n=16, k=4, seed=81),
    configs.small_muse(T=1000, d=256, L=256, I=256, n=8, k=2, seed=82),     # several chunks / expert
    configs.small_shazeer(T=250, d=128, h=256, n=16, k=4, seed=83),         # ReLU, no latent
    configs.MUSE_IMBALANCED.replace(T=700, seed=84),                        # Zipf-skewed groups
]


@pytest.mark.parametrize("cfg", STAGED_CASES, ids=lambda c: f"{c.name}-n{c.n_experts}")
def test_layer_equals_staged_entry_points(cfg):
    """moe_layer_forward against the same layer composed from the staged entry points (route,
    latent down, permute with the row scatter, expert FFN with its row partial sums of squares,
    combine from those partials, latent up): the same output bits (the fused call shares the
    workspace between stages; nothing else may differ)."""
    import torch
    dev = moe_inputs.device_inputs(cfg)
    c = abi_config(cfg)
    fused = run_layer(cfg, dev)["out"]
    T, n, k = cfg.T, cfg.n_experts, cfg.top_k
    E = cfg.expert_in
    dt = fused.dtype
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    logits = torch.empty((T, n), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(c, dev["u"], dev["w_router"], dev.get("logit_bias"), logits, idx, w)
    x = dev["u"]
    if cfg.latent:
        x = torch.empty((T, E), dtype=dt, device="cuda")
        moe.moe_latent_down(c, dev["u"], dev["p_down"], x)
    offsets = torch.empty(n + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((T * k, E), dtype=dt, device="cuda")
    moe.moe_permute(c, idx, offsets, perm, inv, x, dev.get("gamma_pre") if cfg.pre_norm else None,
                    x_perm, ws)
    s = torch.empty_like(x_perm)
    # the fused call takes the row partials when the down GEMM writes at most 32 per row (its
    # normal-orientation tiles); otherwise the combine reduces the rows itself
    parts = moe.row_sumsq_parts(c)
    ss = torch.empty((T * k, parts), dtype=torch.float32, device="cuda") \
        if cfg.expert_norm and parts <= 32 else None
    moe.moe_expert_ffn(c, x_perm, offsets, dev["w_gu"], dev["w_down"],
                       dev.get("gamma_expert") if cfg.expert_norm else None, s, ws, row_sumsq=ss)
    y = torch.empty((T, E), dtype=dt, device="cuda")
    moe.moe_combine(c, s, inv, w, y, row_sumsq=ss)
    staged = y
    if cfg.latent:
        staged = torch.empty_like(fused)
        moe.moe_latent_up(c, y, dev["p_up"], dev["u"], dev.get("resid_g"), staged)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    a = fused.view(torch.int16).cpu().numpy()
    b = staged.view(torch.int16).cpu().numpy()
    np.testing.assert_array_equal(a, b)
