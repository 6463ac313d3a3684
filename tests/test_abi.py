"""The C-ABI library loads, exports every declared entry point, and rejects
bad arguments with the documented status codes before touching a device.
Runs without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def cowa():
    from structured_sparse_attention_block_b200 import build
    build.build()
    import structured_sparse_attention_block_b200 as m
    return m


def declared_functions():
    text = open(os.path.join(ROOT, "include", "cowa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cowa_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(cowa):
    names = declared_functions()
    assert "cowa_fwd" in names and "cowa_bwd" in names and "cowa_decode" in names
    lib = ctypes.CDLL(cowa.library_path())
    for n in names:
        assert hasattr(lib, n), "missing export %s" % n


def test_checking_build_exports_the_same_symbols(cowa):
    """The COWA_DEBUG variant (index checks in the kernels) is a drop-in
    replacement: it builds from the same sources and exports every entry
    point the header declares."""
    from structured_sparse_attention_block_b200 import build
    path = build.build(debug=True)
    assert path.endswith("libcowa_debug.so") and path != cowa.library_path()
    lib = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(lib, n), "missing export %s in the checking build" % n


def test_status_strings_and_version(cowa):
    lib = cowa.lib()
    assert lib.cowa_abi_version() == 1
    for code, name in cowa._STATUS.items():
        assert lib.cowa_status_string(code).decode() == name


@pytest.mark.parametrize("Lk,Hkv,S,N,W", [(512, 2, 16, 64, 224), (8192, 4, 64, 1024, 1792),
                                          (32768, 8, 128, 4096, 3584), (131072, 8, 128, 8192, 15360),
                                          (100, 4, 0, 200, 0), (65, 8, 0, 0, 9)])
def test_default_quad(cowa, Lk, Hkv, S, N, W):
    assert cowa.cowa_default_quad(Lk, Hkv, S, N) == (S, N, 0, W)


def make_shape(cowa, B=1, Lq=128, Lk=128, Hq=4, Hkv=2, d=64, off=0, strides=None):
    st = strides or {}
    def s(name, H):
        v = st.get(name, (Lq if name in "qo" else Lk) * H * d)
        return (ctypes.c_int64 * 3)(v, H * d, d)
    return cowa.Shape(B, Lq, Lk, Hq, Hkv, d, s("q", Hq), s("k", Hkv), s("v", Hkv), s("o", Hq), off)


def call_fwd(cowa, shape, quad=(1, 2, 0, 3), ptr=16):
    lib = cowa.lib()
    p = ctypes.c_void_p(ptr)
    return lib.cowa_fwd(ctypes.byref(shape), cowa.Quad(*quad), 0.0, p, p, p, p, p, p, 1 << 20, None)


def test_argument_errors(cowa):
    assert call_fwd(cowa, make_shape(cowa), quad=(-1, 2, 0, 3)) == 1
    assert call_fwd(cowa, make_shape(cowa, d=96)) == 2
    assert call_fwd(cowa, make_shape(cowa, Hq=3, Hkv=2)) == 1
    assert call_fwd(cowa, make_shape(cowa, strides={"k": 1001})) == 3
    assert call_fwd(cowa, make_shape(cowa), ptr=0) == 1
    assert call_fwd(cowa, make_shape(cowa), ptr=24) == 3
    assert "not 16-byte aligned" in cowa.lib().cowa_last_error_detail().decode()
    lib = cowa.lib()
    shp = make_shape(cowa, Lq=2)
    p = ctypes.c_void_p(16)
    st = lib.cowa_decode(ctypes.byref(shp), cowa.Quad(1, 2, 0, 3), 0.0, p, p, p, p, p, p, p, 1 << 20, None)
    assert st == 1  # decode needs Lq == 1


def test_empty_problem_is_a_no_op(cowa):
    # nothing to compute: returns OK without needing a device or pointers
    shape = make_shape(cowa, B=0)
    lib = cowa.lib()
    assert lib.cowa_fwd(ctypes.byref(shape), cowa.Quad(1, 2, 0, 3), 0.0, *([None] * 5), None, 0, None) == 0


def test_workspace_sizes(cowa):
    lib = cowa.lib()
    shape = make_shape(cowa, Lq=1000, Lk=1000)
    assert lib.cowa_fwd_workspace_size(ctypes.byref(shape), cowa.Quad(1, 2, 0, 3)) >= 2 * 8 * 8 * 4
    assert lib.cowa_bwd_workspace_size(ctypes.byref(shape), cowa.Quad(1, 2, 0, 3)) >= 4 * 1000 * 4
    assert lib.cowa_fwd_workspace_size(ctypes.byref(shape), cowa.Quad(-1, 2, 0, 3)) == 0


def test_oracle_is_not_reachable_from_the_product():
    """The package never imports the oracle (test infrastructure only)."""
    pkg = os.path.join(ROOT, "structured_sparse_attention_block_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle|#include\s+\S*oracle|cowa_ref_",
                                     text, flags=re.M), f


def test_trace_argument_errors(cowa):
    lib = cowa.lib()
    assert lib.cowa_trace_start(-1, None) == 1
    assert lib.cowa_trace_start(1 << 21, None) == 1
    assert lib.cowa_trace_start(4, b"x" * 64) == 1
    assert lib.cowa_trace_stop() == 0
    assert lib.cowa_trace_size() == 0
    name, ms = ctypes.c_char_p(), ctypes.c_float()
    assert lib.cowa_trace_entry(0, ctypes.byref(name), ctypes.byref(ms)) == 1


def test_wcache_rows_and_argument_errors(cowa):
    lib = cowa.lib()
    assert cowa.cowa_wcache_rows((128, 8192, 0, 15360), 16) == 128 + 8192 + 15360 + 32
    assert cowa.cowa_wcache_rows((1, 2, 0, 3), 0) == 0
    assert cowa.cowa_wcache_rows((-1, 2, 0, 3), 4) == 0
    p = ctypes.c_void_p(16)
    shp = make_shape(cowa, Lq=1, Lk=1 + 2 + 3 + 8)
    # a windowed decode whose cache rows do not match the quadruple and horizon
    st = lib.cowa_decode_windowed(ctypes.byref(make_shape(cowa, Lq=1, Lk=99)), cowa.Quad(1, 2, 0, 3), 0.0, 4,
                                  p, p, p, p, p, p, p, p, 1 << 20, None)
    assert st == 1 and "rows" in lib.cowa_last_error_detail().decode()
    st = lib.cowa_decode_windowed(ctypes.byref(shp), cowa.Quad(1, 2, 0, 3), 0.0, 4, None, p, p, p, p, p, p, p,
                                  1 << 20, None)
    assert st == 1  # origin is NULL
    assert lib.cowa_wcache_build(ctypes.byref(make_shape(cowa, d=96)), cowa.Quad(1, 2, 0, 3), 4, p, p, p, p, p,
                                 None) == 2
    assert lib.cowa_wcache_append(ctypes.byref(make_shape(cowa)), cowa.Quad(1, 2, 0, 3), 4, p, None, p, p, p, p,
                                  None) == 1  # pos is NULL


def test_varlen_argument_errors(cowa):
    lib = cowa.lib()
    s2 = lambda a, b: (ctypes.c_int64 * 2)(a, b)
    def vshape(B=2, tq=100, tk=100, mq=60, mk=60, Hq=4, Hkv=2, d=64, qs=(256, 64)):
        return cowa.VarlenShape(B, tq, tk, mq, mk, Hq, Hkv, d, s2(*qs), s2(128, 64), s2(128, 64), s2(256, 64), 0)
    p = ctypes.c_void_p(16)
    call = lambda sh: lib.cowa_fwd_varlen(ctypes.byref(sh), cowa.Quad(1, 2, 0, 3), 0.0, p, p, p, p, p, p, p, p,
                                          1 << 20, None)
    assert call(vshape(mq=101)) == 1          # longest sequence above the token count
    assert call(vshape(d=96)) == 2
    assert call(vshape(Hq=3)) == 1
    assert call(vshape(qs=(250, 64))) == 3    # token stride not a multiple of 8
    assert call(vshape(tk=0, mk=0)) == 2      # no keys at all
    assert lib.cowa_fwd_varlen(ctypes.byref(vshape()), cowa.Quad(1, 2, 0, 3), 0.0, None, p, p, p, p, p, p, p,
                               1 << 20, None) == 1  # cu_q is NULL


def test_selftest_refused_without_a_device(cowa):
    """With no sm_100 device the timeout self-test launches nothing and
    returns a status (the GPU test covers the launch itself)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present: tests/test_timeout_gpu.py runs the self-test")
    assert cowa.lib().cowa_selftest_wait_timeout(None) in (2, 5)  # UNSUPPORTED or CUDA
