"""The C ABI library loads and exports every entry point include/w8a8.h declares (CPU only:
no kernel is launched here)."""
import ctypes
import os
import re

import pytest

from w8a8_int8_quantized_act_b200 import binding as B
from w8a8_int8_quantized_act_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w8a8.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(w8a8_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    try:
        build_mod.build()
    except RuntimeError as e:  # pragma: no cover
        pytest.skip(f"cannot build: {e}")
    return B.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(B.SIGNATURES), "binding and header disagree"


def test_version_and_status_strings(lib):
    assert lib.w8a8_version() == 220
    for st in range(-5, 1):
        assert B.status_string(st) not in ("", "unknown status")


def test_workspace_queries_are_host_only(lib):
    assert B.w8a8_moe_workspace_size(64, 2048, 128, 8, 768) > 64 * 8 * 2048
    L = B.w8a8_moe_workspace_layout(64, 2048, 128, 8, 768)
    offs = [L[k] for k in ("topk_ids", "topk_w", "tile_counts", "offsets", "perm", "sx", "sx_sorted", "xq",
                           "h", "s_h", "hq", "o", "logits", "sync")]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs) and L["total"] > offs[-1]
    assert L["o"] + 64 * 8 * 2048 * 2 <= L["logits"] and L["logits"] + 64 * 128 * 4 <= L["total"]
    # rejected shapes report size 0
    assert B.w8a8_moe_workspace_size(64, 2000, 128, 8, 768) == 0  # H % 128
    assert B.w8a8_moe_workspace_size(64, 2048, 300, 8, 768) == 0  # E > 256
    assert B.w8a8_moe_workspace_size(64, 2048, 128, 17, 768) == 0  # k > 16
    assert B.w8a8_moe_workspace_size(64, 2048, 4, 8, 768) == 0  # k > E
    assert B.w8a8_linear_workspace_size(2048, 2048, 6144, 1, 64) == 0  # group != 128
    assert B.w8a8_linear_workspace_size(2048, 2048, 6144, 1, 128) > 0
    assert B.w8a8_mxfp8_linear_workspace_size(2048, 2048, 6144) >= 2048 * 2048 + 2048 * 64
    assert B.w8a8_mxfp8_linear_workspace_size(2048, 2112, 6144) == 0  # K % 128
    assert B.w8a8_mxfp8_linear_workspace_size(2048, 2048, 6100) == 0  # N % 128


def test_argument_checks_reject_before_any_launch(lib):
    c = ctypes.c_void_p
    # negative sizes, null pointers, unsupported shapes: all rejected on the host
    assert lib.w8a8_quant_act_per_token(None, -1, 128, None, None, None) == B.W8A8_ERR_ARG
    assert lib.w8a8_quant_act_per_token(c(16), 4, 7, c(16), c(16), None) == B.W8A8_ERR_UNSUPPORTED
    assert lib.w8a8_quant_act_per_token(None, 4, 128, None, None, None) == B.W8A8_ERR_ARG
    assert lib.w8a8_quant_act_per_token(None, 0, 128, None, None, None) == B.W8A8_OK  # empty
    assert lib.w8a8_moe_forward(None, None, None, None, None, None, None, 8, 2048, 128, 8, 768, 1, None, 0, None,
                                None) == B.W8A8_ERR_ARG
    assert lib.w8a8_moe_forward(None, None, None, None, None, None, None, 0, 2048, 128, 8, 768, 1, None, 0, None,
                                None) == B.W8A8_OK  # T = 0 is a no-op
    assert lib.w8a8_moe_forward(c(256), c(256), None, c(256), c(256), c(256), c(256), 8, 2048, 128, 8, 768, 1,
                                c(256), 10, c(256), None) == B.W8A8_ERR_WORKSPACE
    assert lib.w8a8_moe_route(None, None, None, 4, 2048, 128, 9, 1, None, None, None, None) == B.W8A8_ERR_ARG
    assert lib.w8a8_quantize_weight_int4_per_group(None, 4, 256, 64, None, None, None) == B.W8A8_ERR_UNSUPPORTED
    assert lib.w8a8_gemm_s8s8s32(None, None, None, 4, 100, 128, None) == B.W8A8_ERR_UNSUPPORTED
    assert lib.w8a8_mxfp8_quantize(c(16), 4, 48, c(16), c(16), None) == B.W8A8_ERR_UNSUPPORTED  # K % 32
    assert lib.w8a8_mxfp8_quantize(None, 4, 64, None, None, None) == B.W8A8_ERR_ARG
    assert lib.w8a8_mxfp8_quantize(None, 0, 64, None, None, None) == B.W8A8_OK  # empty
    assert lib.w8a8_mxfp8_linear(c(256), c(256), c(256), 8, 128, 256, c(256), 10, c(256), None) == \
        B.W8A8_ERR_WORKSPACE
    assert lib.w8a8_mxfp8_linear(c(256), c(256), c(256), 8, 192, 256, c(256), 1 << 20, c(256), None) == \
        B.W8A8_ERR_UNSUPPORTED  # K % 128
    assert lib.w8a8_mxfp4_quantize(c(16), 4, 48, c(16), c(16), None) == B.W8A8_ERR_UNSUPPORTED  # K % 32
    assert lib.w8a8_mxfp4_quantize(None, 4, 64, None, None, None) == B.W8A8_ERR_ARG
    assert lib.w8a8_mxfp4_quantize(None, 0, 64, None, None, None) == B.W8A8_OK  # empty
    assert lib.w8a8_mxfp4_quantize(c(16), 4, 64, c(18), c(16), None) == B.W8A8_ERR_UNSUPPORTED  # packed alignment
    assert lib.w8a8_mxfp_a8w4_linear(c(256), c(256), c(256), 8, 128, 256, c(256), 10, c(256), None) == \
        B.W8A8_ERR_WORKSPACE
    assert lib.w8a8_mxfp_a8w4_linear(c(256), c(256), c(256), 8, 192, 256, c(256), 1 << 20, c(256), None) == \
        B.W8A8_ERR_UNSUPPORTED  # K % 128
    assert lib.w8a8_mxfp_a8w4_linear(c(256), c(272), c(256), 8, 128, 256, c(256), 1 << 20, c(256), None) == \
        B.W8A8_ERR_UNSUPPORTED  # packed weights not 32-byte aligned (the 4-bit TMA type needs it)
    assert lib.w8a8_mxfp_a8w4_linear_prequant(c(256), c(256), c(256), c(256), 8, 128, 200, c(256), None) == \
        B.W8A8_ERR_UNSUPPORTED  # N % 128
    # expert-parallel entries: shapes, offsets and pointers are checked on the host
    assert lib.w8a8_moe_route_group(None, None, None, 8, 200, 8, 2, 1, None, 0, None) == B.W8A8_ERR_UNSUPPORTED
    assert lib.w8a8_moe_route_group(None, None, None, 0, 256, 8, 2, 1, None, 0, None) == B.W8A8_OK  # empty
    assert lib.w8a8_moe_route_group(c(256), c(256), None, 8, 256, 8, 2, 1, c(256), 10, None) == B.W8A8_ERR_WORKSPACE
    assert B.w8a8_moe_experts_workspace_size(100, 256, 128, 8) > 0
    assert B.w8a8_moe_experts_workspace_size(100, 200, 128, 8) == 0  # H % 128
    assert B.w8a8_moe_experts_workspace_size(100, 256, 128, 1025) == 0  # more than 1024 groups
    offs = (ctypes.c_int * 3)(0, 4, 3)
    assert lib.w8a8_moe_experts(c(256), c(256), offs, 2, 2, 3, 256, 128, 2, c(256), c(256), c(256), c(256),
                                c(256), 1 << 20, c(256), None) == B.W8A8_ERR_ARG  # decreasing offsets
    offs = (ctypes.c_int * 3)(0, 4, 9)
    assert lib.w8a8_moe_experts(c(256), c(256), offs, 2, 3, 9, 256, 128, 2, c(256), c(256), c(256), c(256),
                                c(256), 1 << 20, c(256), None) == B.W8A8_ERR_ARG  # weight_groups > Ew
    assert lib.w8a8_moe_experts(c(256), c(256), offs, 2, 2, 9, 256, 128, 2, c(256), c(256), c(256), c(256),
                                c(256), 10, c(256), None) == B.W8A8_ERR_WORKSPACE
    assert lib.w8a8_moe_combine_sorted(c(256), c(256), c(256), 4, 200, 2, c(256), c(256), None) == \
        B.W8A8_ERR_UNSUPPORTED  # H % 128
    assert lib.w8a8_moe_combine_sorted(None, None, None, 4, 256, 2, None, None, None) == B.W8A8_ERR_ARG
    assert lib.w8a8_debug_wait_timeout(0, None) == B.W8A8_ERR_ARG
    assert lib.w8a8_debug_rcp_approx_ulp(0, 10, c(16), None) == B.W8A8_ERR_ARG  # not a normal input
    assert lib.w8a8_debug_rcp_approx_ulp(0x7E7FFFFF, 2, c(16), None) == B.W8A8_ERR_ARG  # reciprocal subnormal
    assert lib.w8a8_debug_ex2_approx_ulp(0x7FFFFFFF, 2, c(16), None) == B.W8A8_ERR_ARG  # crosses the sign
    assert lib.w8a8_debug_ex2_approx_ulp(0x43000000, 4, c(16), None) == B.W8A8_ERR_ARG  # 2^128 overflows


def test_package_has_no_oracle_dependency():
    pkg = os.path.join(ROOT, "w8a8_int8_quantized_act_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", src, re.M), f
