"""The C-ABI library loads and exports every entry point the header
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from moe_gemm_absmax_b200 import build, w8a8

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "w8a8.h")).read()
    return sorted(set(re.findall(r"^W8A8_API\s+[\w\s\*]+?\b((?:w8a8|fwht128|group128)_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return w8a8.lib()


def test_header_declares_the_four_named_entry_points():
    names = _declared()
    for n in ("w8a8_quant_act", "w8a8_linear", "w8a8_moe_forward", "fwht128_quant"):
        assert n in names
    assert set(names) == set(w8a8.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    for n in _declared():
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    assert w8a8.status_str(0) == "ok"
    assert w8a8.status_str(-2) == "workspace too small"
    assert "sm_100a" in w8a8.version()


def test_workspace_queries(L):
    assert L.w8a8_linear_workspace_size(8, 5120, 17408) >= 8 * 17408 + 32
    assert L.w8a8_linear_workspace_size(0, 5, 5) == 0
    assert L.w8a8_moe_workspace_size(4096, 256, 2048, 512, 8) > 4096 * 8 * 2048
    assert L.w8a8_gemm_workspace_size(4096, 5120, 17408, w8a8.PATH_TCGEN05) == 0


def test_moe_combine_mode(L):
    auto = L.w8a8_moe_workspace_size(4096, 256, 2048, 512, 8)
    assert w8a8.moe_set_combine(w8a8.MOE_COMBINE_EXACT) == w8a8.MOE_COMBINE_AUTO
    try:
        exact = L.w8a8_moe_workspace_size(4096, 256, 2048, 512, 8)
        # the [T * topk, H] fp32 contributions instead of the [T, H] atomic buffer
        assert exact - auto >= (4096 * 8 - 4096) * 2048 * 4
        assert L.w8a8_moe_set_combine(7) == w8a8.ERR_INVALID_ARG
    finally:
        assert w8a8.moe_set_combine(w8a8.MOE_COMBINE_AUTO) == w8a8.MOE_COMBINE_EXACT
    assert L.w8a8_moe_workspace_size(4096, 256, 2048, 512, 8) == auto
    # small T: the slot-order combine either way
    assert L.w8a8_moe_workspace_size(8, 256, 2048, 512, 8) > 8 * 8 * 2048 * 4


def test_argument_checks_without_gpu(L):
    vp = ctypes.c_void_p
    fake = vp(0x10000)
    # null pointers, bad sizes, misalignment: rejected before anything is enqueued
    assert L.w8a8_quant_act(None, 4, 64, 64, fake, fake, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_quant_act(fake, 4, 60, 64, fake, fake, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_quant_act(vp(0x10001), 4, 64, 64, fake, fake, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_linear(fake, fake, fake, fake, 4, 12, 64, fake, 1 << 20, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_linear(fake, fake, fake, fake, 4, 16, 64, fake, 16, None) == w8a8.ERR_WORKSPACE
    assert L.fwht128_quant(fake, 2, 192, fake, fake, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_moe_forward(fake, fake, fake, fake, fake, fake, fake, 4, 8, 256, 64, 9, fake, 1 << 30,
                              None, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_moe_forward(fake, fake, fake, fake, fake, fake, fake, 4, 8, 256, 64, 2, fake, 64,
                              None, None) == w8a8.ERR_WORKSPACE
    assert L.w8a8_gemm_q(fake, fake, fake, fake, fake, 4, 16, 64, 7, None, 0, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_debug_wait_timeout(10, None) == w8a8.ERR_INVALID_ARG


def test_rotated_grid_workspace_queries(L):
    # the FWHT128-grid MoE keeps the slot contributions [T*k, H] fp32 for the exact combine
    assert L.w8a8_moe_g128_workspace_size(4096, 256, 2048, 512, 8) >= 4096 * 8 * 2048 * 4
    assert L.w8a8_moe_g128_workspace_size(0, 256, 2048, 512, 8) == 0
    assert L.w8a8_shared_expert_workspace_size(8, 2048, 512) >= 8 * 2048 * 4 + 8 * 512 * 4
    assert L.w8a8_shared_expert_workspace_size(8, 128, 512) == 0


def test_rotated_grid_argument_checks_without_gpu(L):
    vp = ctypes.c_void_p
    fake = vp(0x10000)
    # K not a multiple of 128 (group grid), or of 256 (trunk format)
    assert L.group128_quant(fake, 2, 192, fake, fake, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_linear_group128(fake, fake, fake, fake, fake, 2, 16, 192, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_trunk_weight_quant(fake, 4, 384, fake, fake, fake, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_trunk_weight_quant(fake, 4, 16384, fake, fake, fake, None) == w8a8.ERR_UNSUPPORTED
    assert L.w8a8_linear_trunk(fake, fake, fake, fake, fake, fake, 2, 16, 384, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_linear_trunk(fake, fake, fake, None, fake, fake, 2, 16, 512, None) == w8a8.ERR_INVALID_ARG
    # routed experts on the grid: H or I off the 128 grid, topk > E, too small a workspace
    assert L.w8a8_moe_g128_forward(fake, fake, fake, fake, fake, fake, fake, 4, 8, 192, 128, 2, fake, 1 << 30,
                                   None, None) == w8a8.ERR_UNSUPPORTED
    assert L.w8a8_moe_g128_forward(fake, fake, fake, fake, fake, fake, fake, 4, 8, 256, 128, 9, fake, 1 << 30,
                                   None, None) == w8a8.ERR_INVALID_ARG
    assert L.w8a8_moe_g128_forward(fake, fake, fake, fake, fake, fake, fake, 4, 8, 256, 128, 2, fake, 64,
                                   None, None) == w8a8.ERR_WORKSPACE
    assert L.w8a8_shared_expert_forward(fake, fake, fake, fake, fake, fake, fake, 4, 384, 128, fake, 1 << 30,
                                        None, None) == w8a8.ERR_UNSUPPORTED
    assert L.w8a8_shared_expert_forward(fake, fake, fake, fake, fake, fake, fake, 4, 256, 128, fake, 64,
                                        None, None) == w8a8.ERR_WORKSPACE
