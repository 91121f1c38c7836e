"""The C-ABI library on the host (no GPU compute): it loads, exports every
symbol ``include/ssa.h`` declares, sizes workspaces, and rejects bad
arguments with status codes before touching CUDA."""
import ctypes
import os
import re

import pytest

from gist_token_chunk_b200 import ssa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "ssa.h")).read()
    return sorted(set(re.findall(r"SSA_API\s+[\w\s\*]+?\b(ssa_\w+)\s*\(", txt)))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(ssa.lib, n), f"libssa.so does not export {n}"


def test_status_strings_and_version():
    for code in range(7):
        assert ssa.lib.ssa_status_string(code)
    assert ssa.lib.ssa_version() >= 1


def shape(**kw):
    base = dict(B=4, Hq=32, Hkv=8, d=64, n_max=131072, dtype=ssa.SSA_BF16)
    base.update(kw)
    return ssa.make_shape(**base)


def test_workspace_size_scales_with_problem():
    small = ssa.ssa_workspace_size(shape(n_max=8192), 128, 8, 32)
    big = ssa.ssa_workspace_size(shape(), 128, 8, 32)
    assert 0 < small < big
    h2 = ssa.ssa_workspace_size_h2(shape(B=8, n_max=131072), 64, 8, 16, 8, 8, 16)
    assert h2 > 0


@pytest.mark.parametrize("kw,C,g,topk,flags,path", [
    (dict(), 128, 8, 32, 0, ssa.SSA_PATH_PIPELINE),                   # the 128K batch workload
    (dict(B=2, n_max=524288), 256, 8, 64, 0, ssa.SSA_PATH_PIPELINE),  # 512K
    (dict(), 128, 8, 32, ssa.SSA_DEBUG_FUSED_PATH, ssa.SSA_PATH_FUSED),
    (dict(d=128), 128, 8, 32, 0, ssa.SSA_PATH_FUSED),                 # d = 128
    (dict(Hq=64, Hkv=4), 128, 8, 32, 0, ssa.SSA_PATH_FUSED),          # G = 16
    (dict(dtype=ssa.SSA_FP32), 128, 8, 32, 0, ssa.SSA_PATH_GENERIC),
    (dict(B=200, n_max=8192), 128, 8, 32, 0, ssa.SSA_PATH_GENERIC),   # B > 128
])
def test_decode_path(kw, C, g, topk, flags, path):
    ssa.ssa_set_debug_flags(flags)
    try:
        assert ssa.ssa_decode_path(shape(**kw), C, g, topk) == path
    finally:
        ssa.ssa_set_debug_flags(0)


def test_decode_path_rejects_bad_sizes():
    v = ctypes.c_int32(-1)
    assert ssa.lib.ssa_decode_path(ctypes.byref(shape(d=96)), 128, 8, 32,
                                   ctypes.byref(v)) == ssa.SSA_ERR_UNSUPPORTED
    assert ssa.lib.ssa_decode_path(ctypes.byref(shape()), 128, 8, 32, None) == ssa.SSA_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,C,g,topk,code", [
    (dict(Hq=30), 128, 8, 32, ssa.SSA_ERR_INVALID_ARG),          # Hq % Hkv
    (dict(d=96), 128, 8, 32, ssa.SSA_ERR_UNSUPPORTED),           # bf16 head dim
    (dict(dtype=7), 128, 8, 32, ssa.SSA_ERR_INVALID_ARG),        # dtype
    (dict(n_max=1000), 128, 8, 32, ssa.SSA_ERR_INVALID_ARG),     # n_max % C
    (dict(), 0, 8, 32, ssa.SSA_ERR_INVALID_ARG),                 # C
    (dict(), 128, 0, 32, ssa.SSA_ERR_INVALID_ARG),               # g
    (dict(), 128, 8, -1, ssa.SSA_ERR_INVALID_ARG),               # topk
    (dict(), 128, 8, 5000, ssa.SSA_ERR_UNSUPPORTED),             # topk cap
    (dict(Hq=64, Hkv=2), 128, 8, 32, ssa.SSA_ERR_UNSUPPORTED),   # group > 16
])
def test_workspace_size_rejects(kw, C, g, topk, code):
    n = ctypes.c_size_t(0)
    st = ssa.lib.ssa_workspace_size(ctypes.byref(shape(**kw)), C, g, topk, ctypes.byref(n))
    assert st == code, (st, ssa.lib.ssa_last_error())
    assert ssa.lib.ssa_last_error()


def test_null_pointers_rejected_before_cuda():
    sh = shape()
    st = ssa.lib.ssa_decode(ctypes.byref(sh), None, None, None, None, None, None, 128, 8, 32,
                            None, None, None, 0, None)
    assert st == ssa.SSA_ERR_INVALID_ARG
    st = ssa.lib.ssa_decode(None, 16, 16, 16, 16, 16, 16, 128, 8, 32, 16, 16, None, 0, None)
    assert st == ssa.SSA_ERR_INVALID_ARG
    st = ssa.lib.ssa_score_gists(ctypes.byref(sh), None, 16, 16, 128, 8, 16, None)
    assert st == ssa.SSA_ERR_INVALID_ARG
    st = ssa.lib.ssa_topk_chunks(ctypes.byref(sh), None, 16, 128, 32, 16, None)
    assert st == ssa.SSA_ERR_INVALID_ARG


def test_misaligned_bf16_tensor_rejected():
    sh = shape()
    st = ssa.lib.ssa_decode(ctypes.byref(sh), 16, 18, 16, 16, 16, 16, 128, 8, 32, 16, 16, None, 0,
                            None)
    assert st == ssa.SSA_ERR_UNSUPPORTED


def test_small_workspace_rejected():
    sh = shape()
    need = ssa.ssa_workspace_size(sh, 128, 8, 32)
    st = ssa.lib.ssa_decode(ctypes.byref(sh), 256, 256, 256, 256, 256, 256, 128, 8, 32, 256, 256,
                            256, need - 1, None)
    assert st == ssa.SSA_ERR_WORKSPACE
    st = ssa.lib.ssa_decode(ctypes.byref(sh), 256, 256, 256, 256, 256, 256, 128, 8, 32, 256, 256,
                            None, 64, None)
    assert st == ssa.SSA_ERR_WORKSPACE


def test_h2_argument_checks():
    sh = shape(B=8)
    n = ctypes.c_size_t(0)
    assert ssa.lib.ssa_workspace_size_h2(ctypes.byref(sh), 64, 8, 0, 8, 8, 16,
                                         ctypes.byref(n)) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_workspace_size_h2(ctypes.byref(sh), 64, 8, 200, 8, 8, 16,
                                         ctypes.byref(n)) == ssa.SSA_ERR_UNSUPPORTED  # J*g > 1024
    assert ssa.lib.ssa_workspace_size_h2(ctypes.byref(sh), 64, 8, 16, 8, -1, 16,
                                         ctypes.byref(n)) == ssa.SSA_ERR_INVALID_ARG


@pytest.mark.parametrize("context,select,code", [
    (2, 0, ssa.SSA_ERR_INVALID_ARG), (0, -1, ssa.SSA_ERR_INVALID_ARG), (1, 1, ssa.SSA_OK)])
def test_variant_workspace_and_bad_readings(context, select, code):
    n = ctypes.c_size_t(0)
    st = ssa.lib.ssa_workspace_size_variant(ctypes.byref(shape()), 128, 8, 32, context, select,
                                            ctypes.byref(n))
    assert st == code
    if code == ssa.SSA_OK:
        # per-head scores (B*Hq rows) and per-head selections
        assert n.value >= 4 * 32 * 1024 * 4 + 4 * 32 * 32 * 4


def test_hier_workspace_and_bad_levels():
    sh = shape(B=1, n_max=1 << 20)
    n = ssa.ssa_workspace_size_hier(sh, 64, 8, 16, [8, 8], [16, 8, 4])
    # candidate scores of every level: 8 pairs x (16384 + 1024 + 64) floats
    assert n >= 8 * (16384 + 1024 + 64) * 4
    v = ctypes.c_size_t(0)
    nine = (ctypes.c_int32 * 9)(*([8] * 9))
    assert ssa.lib.ssa_workspace_size_hier(ctypes.byref(sh), 64, 8, 16, 9, nine, nine,
                                           ctypes.byref(v)) == ssa.SSA_ERR_INVALID_ARG
    bad_g = (ctypes.c_int32 * 2)(0, 8)
    tk = (ctypes.c_int32 * 3)(16, 8, 4)
    assert ssa.lib.ssa_workspace_size_hier(ctypes.byref(sh), 64, 8, 16, 3, bad_g, tk,
                                           ctypes.byref(v)) == ssa.SSA_ERR_INVALID_ARG
