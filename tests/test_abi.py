"""The C-ABI library without a GPU: it builds, loads, exports every declared symbol, and rejects
bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import sparse_moe_layer_softmax_b200 as moe
from sparse_moe_layer_softmax_b200 import build as moe_build
from moe_inputs import configs

from gpu_harness import abi_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 10
    assert set(moe.EXPORTS) == set(syms)
    for s in syms:
        assert hasattr(lib, s), s


def test_status_strings(lib):
    for code, name in moe.STATUS.items():
        assert lib.moe_status_string(code).decode().startswith(name)


def test_workspace_size_is_host_arithmetic(lib):
    for cfg in configs.CONFIGS.values():
        n = moe.workspace_size(abi_config(cfg))
        TK = cfg.T * cfg.top_k
        # at least the dispatched rows and the expert activation
        assert n >= TK * cfg.expert_in * 2 + TK * cfg.d_ff * (2 if cfg.dtype == "bf16" else 4)
    assert moe.workspace_size(abi_config(configs.MUSE_PREFILL)) < 4 << 30


@pytest.mark.parametrize("field,value,code", [
    ("n_experts", 0, "MOE_ERR_INVALID_ARG"), ("top_k", 9, "MOE_ERR_UNSUPPORTED"),
    ("top_k", 300, "MOE_ERR_INVALID_ARG"), ("n_experts", 300, "MOE_ERR_UNSUPPORTED"),
    ("d_model", 100, "MOE_ERR_UNSUPPORTED"), ("dtype", 7, "MOE_ERR_UNSUPPORTED"),
    ("T", -1, "MOE_ERR_INVALID_ARG"), ("tau", 0.0, "MOE_ERR_INVALID_ARG"),
])
def test_bad_config_rejected(lib, field, value, code):
    c = abi_config(configs.MUSE_DECODE)
    setattr(c, field, value)
    n = ctypes.c_size_t()
    assert lib.moe_workspace_size(ctypes.byref(c), ctypes.byref(n)) == moe.STATUS_CODES[code]


def test_null_and_misaligned_pointers_rejected(lib):
    c = abi_config(configs.MUSE_DECODE)
    rc = lib.moe_route(ctypes.byref(c), None, None, None, None, None, None, None, None)
    assert rc == moe.STATUS_CODES["MOE_ERR_INVALID_ARG"]
    rc = lib.moe_route(ctypes.byref(c), 0x1001, 0x2000, None, None, None, 0x3000, 0x4000, None)
    assert rc == moe.STATUS_CODES["MOE_ERR_ALIGNMENT"]
    # a misaligned correction bias is caught too
    rc = lib.moe_route(ctypes.byref(c), 0x1000, 0x2000, None, 0x3004, None, 0x3000, 0x4000, None)
    assert rc == moe.STATUS_CODES["MOE_ERR_ALIGNMENT"]
    # the split entry point checks its sizes and pointers on the host
    assert lib.moe_router_split_weights(None, 4, 64, 0x1000, None) == \
        moe.STATUS_CODES["MOE_ERR_INVALID_ARG"]
    assert lib.moe_router_split_weights(0x1000, 4, 100, 0x2000, None) == \
        moe.STATUS_CODES["MOE_ERR_UNSUPPORTED"]
    rc = lib.moe_route(ctypes.byref(c), 0x1001, 0x2000, None, None, None, 0x3000, 0x4000, None)
    assert rc == moe.STATUS_CODES["MOE_ERR_ALIGNMENT"]
    rc = lib.moe_layer_forward(ctypes.byref(c), None, 0x1000, 0x1000, 0x2000, None, None, None,
                               None, 0, None)
    assert rc == moe.STATUS_CODES["MOE_ERR_INVALID_ARG"]
    w = moe.Weights(w_router=0x1000, p_down=0x1000, p_up=0x1000, w_gu=0x1000, w_down=0x1000,
                    gamma_pre=0x1000, gamma_expert=0x1000, resid_g=0x1000)
    rc = lib.moe_layer_forward(ctypes.byref(c), ctypes.byref(w), 0x1000, 0x1000, 0x2000, None,
                               None, None, 0x4000, 16, None)
    assert rc == moe.STATUS_CODES["MOE_ERR_WORKSPACE"]
    # fp32 with a latent projection is outside the supported set
    c2 = abi_config(configs.MUSE_DECODE.replace(dtype="f32"))
    assert lib.moe_latent_down(ctypes.byref(c2), 0x1000, 0x1000, 0x1000, None) == \
        moe.STATUS_CODES["MOE_ERR_UNSUPPORTED"]
    # permute: workspace smaller than the per-chunk histograms
    c3 = abi_config(configs.MUSE_PREFILL)
    rc = lib.moe_permute(ctypes.byref(c3), 0x1000, 0x1000, 0x1000, 0x1000, None, None, None,
                         0x1000, 16, None)
    assert rc == moe.STATUS_CODES["MOE_ERR_WORKSPACE"]


def test_no_cpu_fallback_in_product_package():
    """The product package never imports the oracle and has no host compute path."""
    pkg = os.path.join(ROOT, "sparse_moe_layer_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, fn)) as f:
                    src = f.read()
                assert "oracle" not in src.replace("oracle_", ""), fn
                assert "moe_inputs" not in src, fn


def test_host_pipeline_checks_on_host(lib):
    c = abi_config(configs.MUSE_PREFILL)
    n = moe.host_staging_size(c)
    assert n == 4 * ((c.T * c.d_model * 2 + 255) // 256 * 256)
    w = moe.Weights(w_router=0x1000, p_down=0x1000, p_up=0x1000, w_gu=0x1000, w_down=0x1000,
                    gamma_pre=0x1000, gamma_expert=0x1000, resid_g=0x1000)
    ptrs = (ctypes.c_void_p * 1)(0x1000)
    code = moe.STATUS_CODES
    f = lib.moe_layer_forward_host
    assert f(ctypes.byref(c), ctypes.byref(w), -1, ptrs, ptrs, 0x1000, n, 0x1000, 1 << 34,
             None) == code["MOE_ERR_INVALID_ARG"]
    assert f(ctypes.byref(c), ctypes.byref(w), 1, None, ptrs, 0x1000, n, 0x1000, 1 << 34,
             None) == code["MOE_ERR_INVALID_ARG"]
    nulls = (ctypes.c_void_p * 1)(None)
    assert f(ctypes.byref(c), ctypes.byref(w), 1, nulls, ptrs, 0x1000, n, 0x1000, 1 << 34,
             None) == code["MOE_ERR_INVALID_ARG"]
    assert f(ctypes.byref(c), ctypes.byref(w), 1, ptrs, ptrs, 0x1000, n - 1, 0x1000, 1 << 34,
             None) == code["MOE_ERR_WORKSPACE"]
    assert f(ctypes.byref(c), ctypes.byref(w), 1, ptrs, ptrs, 0x1008, n, 0x1000, 1 << 34,
             None) == code["MOE_ERR_ALIGNMENT"]
    # the layer's own checks run before anything is queued: a short workspace
    assert f(ctypes.byref(c), ctypes.byref(w), 1, ptrs, ptrs, 0x1000, n, 0x1000, 16,
             None) == code["MOE_ERR_WORKSPACE"]


def test_row_sumsq_parts_is_host_arithmetic(lib):
    # prefill: normal-orientation down GEMM, one partial per 256-column tile of the 4096-wide row
    # (one per CTA's 128 features with the swapped CTA-pair tiles); decode: swapped orientation,
    # one per 32-feature warp slice of each 128-feature tile
    assert moe.row_sumsq_parts(abi_config(configs.MUSE_PREFILL)) == 4096 // 256
    assert moe.row_sumsq_parts(abi_config(configs.MUSE_DECODE)) == 4096 // 128 * 4
    n = ctypes.c_int32()
    c = abi_config(configs.MUSE_DECODE)
    c.top_k = 0
    assert lib.moe_row_sumsq_parts(ctypes.byref(c), ctypes.byref(n)) == \
        moe.STATUS_CODES["MOE_ERR_INVALID_ARG"]
    assert lib.moe_row_sumsq_parts(ctypes.byref(abi_config(configs.MUSE_DECODE)), None) == \
        moe.STATUS_CODES["MOE_ERR_INVALID_ARG"]


def test_gather_rows_checks_on_host(lib):
    code = moe.STATUS_CODES
    f = lib.moe_gather_rows
    assert f(0x1000, 4, 0x1000, -1, 64, 0x1000, None) == code["MOE_ERR_INVALID_ARG"]
    assert f(0x1000, 4, 0x1000, 2, 24, 0x1000, None) == code["MOE_ERR_UNSUPPORTED"]
    assert f(0x1000, 4, 0x1000, 2, 0, 0x1000, None) == code["MOE_ERR_UNSUPPORTED"]
    assert f(None, 4, 0x1000, 2, 64, 0x1000, None) == code["MOE_ERR_INVALID_ARG"]
    assert f(0x1000, 4, 0x1000, 2, 64, 0x1004, None) == code["MOE_ERR_ALIGNMENT"]
    # nothing to gather: no launch, no pointer needed
    assert f(None, 0, None, 0, 64, None, None) == code["MOE_OK"]
