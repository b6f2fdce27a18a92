"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function
include/swiglu_ffn.h declares, validates arguments before touching the GPU, and its host
subsample generator matches the oracle bit for bit."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle as O
from swiglu_feed_forward_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_every_declared_function_is_exported_and_bound(lib):
    names = declared_functions()
    assert {"swiglu_ffn_fwd", "swiglu_ffn_bwd", "grouped_topk_select", "sparse_swiglu_ffn_fwd"} <= names
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
        assert n in _lib.SIGNATURES, f"{n} has no Python binding"


def test_status_strings(lib):
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.swf_status_string(code).decode().startswith(name)


def test_shape_rules(lib):
    BF, F32 = _lib.SWF_BF16, _lib.SWF_F32
    sup = lambda op, *a: lib.swf_supported(_lib.OPS[op], *a)
    assert sup("fwd", 16384, 768, 2048, 0, 0, 0, BF) == 0
    assert sup("fwd", 64, 128, 352, 0, 0, 0, F32) == 0
    assert sup("fwd", 64, 120, 352, 0, 0, 0, BF) == 2       # d_model not a multiple of 16
    assert sup("fwd", 64, 100, 350, 0, 0, 0, F32) == 0      # fp32 takes any size
    assert sup("fwd", 0, 128, 352, 0, 0, 0, F32) == 1
    assert sup("select", 16384, 1024, 4096, 64, 8, 8, BF) == 0
    assert sup("select", 16384, 1024, 4096, 48, 8, 8, BF) == 2   # not a power of two
    assert sup("select", 16384, 1024, 4096, 128, 8, 8, BF) == 2  # > 64
    assert sup("select", 16384, 1024, 4096, 8, 8, 8, BF) == 2    # < 16
    assert sup("select", 16384, 1024, 4096, 64, 65, 8, BF) == 2  # K > groups
    assert sup("select", 16384, 1024, 4096, 64, 8, 65, BF) == 2  # spg > G
    assert sup("sparse_fwd", 16384, 1024, 64, 64, 1, 0, BF) == 2  # one group only
    assert sup("sparse_fwd", 2 ** 28, 1024, 4096, 64, 8, 0, BF) == 2  # M*K >= 2^31


def test_workspace_and_plan(lib):
    BF = _lib.SWF_BF16
    assert lib.swf_workspace_bytes(_lib.OPS["fwd"], 16384, 768, 2048, 0, 0, BF) == 0
    assert lib.swf_workspace_bytes(_lib.OPS["fwd_infer"], 16384, 768, 2048, 0, 0, BF) >= 16384 * 2048 * 2
    assert lib.swf_workspace_bytes(_lib.OPS["bwd"], 16384, 768, 2048, 0, 0, BF) >= 16384 * 4096 * 2
    info = _lib.swf_plan_info()
    assert lib.swf_plan(_lib.OPS["bwd"], 32768, 2048, 5504, 0, 0, 0, BF, C.byref(info)) == 0
    assert info.path == 1 and info.flops == 12 * 32768 * 2048 * 5504 and info.deterministic == 1
    assert lib.swf_plan(_lib.OPS["fwd"], 64, 128, 352, 0, 0, 0, _lib.SWF_F32, C.byref(info)) == 0
    assert info.path == 0


def test_argument_errors_return_before_any_launch(lib):
    BF = _lib.SWF_BF16
    p = C.c_void_p(0x10000)
    null = None
    # null pointer
    assert lib.swiglu_ffn_fwd(null, p, p, p, p, p, p, p, 64, 128, 352, BF, None) == 1
    # unaligned pointer
    q = C.c_void_p(0x10008)
    assert lib.swiglu_ffn_fwd(q, p, p, p, p, p, p, p, 64, 128, 352, BF, None) == 3
    # unsupported shape
    assert lib.swiglu_ffn_fwd(p, p, p, p, p, p, p, p, 64, 120, 352, BF, None) == 2
    # workspace too small
    assert lib.swiglu_ffn_fwd_infer(p, p, p, p, p, p, 16, 64, 128, 352, BF, None) == 4
    assert lib.swiglu_ffn_bwd(p, p, p, p, p, p, p, p, p, p, p, p, p, 16, 64, 128, 352, BF, None) == 4
    # bad enum
    assert lib.swiglu_ffn_fwd(p, p, p, p, p, p, p, p, 64, 128, 352, 7, None) == 1
    assert lib.swf_selftest_wait_timeout(0, None) == 1


def test_mhffn_argument_errors(lib):
    BF, F32 = _lib.SWF_BF16, _lib.SWF_F32
    p, q = C.c_void_p(0x10000), C.c_void_p(0x10008)
    f = lib.flash_mhffn_fwd
    assert f(None, p, p, p, p, p, 256, 16, 128, 15, 384, BF, None) == 1   # null pointer
    assert f(p, p, p, p, p, p, 0, 16, 128, 15, 384, BF, None) == 1        # no tokens
    assert f(p, p, p, p, p, p, 256, 16, 64, 15, 384, BF, None) == 2       # d_h other than 128
    assert f(p, p, p, p, p, p, 256, 16, 128, 15, 96, BF, None) == 2       # d_e not a multiple of 64
    assert f(p, p, p, p, p, p, 256, 16, 128, 15, 384, F32, None) == 2     # fp32
    assert f(p, p, p, p, q, p, 256, 16, 128, 15, 384, BF, None) == 3      # unaligned router
    assert f(p, p, p, p, p, p, 256, 16, 128, 15, 384, 9, None) == 1       # bad dtype
    b = lib.flash_mhffn_bwd
    assert b(p, p, p, p, p, None, p, p, p, p, p, p, 1 << 30, 256, 16, 128, 15, 384, BF, None) == 1  # null d_o
    assert b(p, p, p, p, p, p, p, p, p, p, p, p, 1 << 30, 256, 16, 128, 15, 320, BF, None) == 2     # d_e % 128
    assert b(p, p, p, p, p, p, p, p, p, p, p, None, 0, 256, 16, 128, 15, 384, BF, None) == 4        # no workspace
    assert lib.flash_mhffn_bwd_workspace_bytes(256, 16, 128, 15, 384, BF) > 256 * 5760 * 8
    assert lib.flash_mhffn_bwd_workspace_bytes(256, 16, 64, 15, 384, BF) == 0
    # the dS_g | dS_u and P planes are held for at most four heads at a time
    planes = lambda g: g * 4096 * 5760 * 2 * 3
    w2, w4, w8 = (lib.flash_mhffn_bwd_workspace_bytes(4096, h, 128, 15, 384, BF) for h in (2, 4, 8))
    assert planes(2) <= w2 < planes(4) <= w4 and w8 - w4 < planes(1)
    g = lib.flash_mhffn_prologue
    assert g(None, p, None, p, p, p, 256, 2048, 16, 128, 15, 1e-6, BF, None) == 1  # null x
    assert g(p, p, None, p, p, p, 256, 2048, 16, 128, 15, -1.0, BF, None) == 1     # eps < 0
    assert g(p, p, None, p, p, p, 256, 2048, 16, 64, 15, 1e-6, BF, None) == 2      # d_h 64
    assert g(p, p, None, p, p, p, 256, 2040, 16, 128, 15, 1e-6, BF, None) == 2     # d_model % 16
    assert g(p, p, None, p, p, p, 256, 2048, 16, 128, 17, 1e-6, BF, None) == 2     # 272 router columns
    assert g(p, p, q, p, p, p, 256, 2048, 16, 128, 15, 1e-6, BF, None) == 3        # unaligned gain


@pytest.mark.parametrize("d_ff,G,spg,seed", [(4096, 64, 8, 3), (512, 32, 8, 0), (256, 16, 16, 7),
                                             (3200, 32, 1, 2 ** 63 + 5)])
def test_subsample_index_matches_oracle(lib, d_ff, G, spg, seed):
    ng = d_ff // G
    out = np.empty((ng, spg), dtype=np.int32)
    st = lib.swf_make_subsample_index(d_ff, G, spg, seed, out.ctypes.data_as(C.c_void_p))
    assert st == 0
    np.testing.assert_array_equal(out, O.make_subsample_index(d_ff, G, spg, seed))


def test_subsample_index_errors(lib):
    out = np.empty(64, dtype=np.int32)
    ptr = out.ctypes.data_as(C.c_void_p)
    assert lib.swf_make_subsample_index(4096, 64, 0, 0, ptr) == 1
    assert lib.swf_make_subsample_index(4096, 64, 65, 0, ptr) == 2
    assert lib.swf_make_subsample_index(4000, 64, 8, 0, ptr) == 2
    assert lib.swf_make_subsample_index(4096, 64, 8, 0, None) == 1


def test_group_idx_validation_rejects_bad_arguments_on_the_host(lib):
    """swf_validate_group_idx checks its arguments before touching the GPU; the debug switch
    takes only 0 or 1 and reports what it was set to."""
    bad = C.c_int64(-1)
    assert lib.swf_validate_group_idx(None, 10, 2, 8, C.byref(bad), None) == 1       # null
    assert lib.swf_validate_group_idx(C.c_void_p(16), 0, 2, 8, C.byref(bad), None) == 1  # M = 0
    assert lib.swf_validate_group_idx(C.c_void_p(16), 10, 0, 8, C.byref(bad), None) == 1  # K = 0
    assert lib.swf_validate_group_idx(C.c_void_p(20), 10, 2, 8, C.byref(bad), None) == 3  # misaligned
    assert lib.swf_validate_group_idx(C.c_void_p(16), 1 << 30, 4, 8, C.byref(bad), None) == 2  # M*K >= 2^31
    assert bad.value == -1  # nothing written
    prev = lib.swf_get_debug()
    try:
        assert lib.swf_set_debug(2) == 1
        assert lib.swf_set_debug(1) == 0 and lib.swf_get_debug() == 1
        assert lib.swf_set_debug(0) == 0 and lib.swf_get_debug() == 0
    finally:
        lib.swf_set_debug(prev)
