"""cowa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin inside a runtime that owns all device memory and hands
over only input and output buffers, or a serving loop where cudaMalloc is not
allowed) get a decode whose split scratch is a fixed array inside the
library.  These tests call it through the C ABI and compare it with
cowa_decode, which takes a caller workspace, and with the fp64 oracle, on two
calls in a row (the second call finds the first call's partials still in the
array), check that
a call leaves device memory as it found it (neither torch's allocator nor the
driver's free-memory count moves), call it once through the Python wrapper,
and check that a shape too large for the array is refused before anything
runs.
"""
import ctypes

import pytest
import torch

import numpy as np

from helpers import LSE_ABS, assert_lse, assert_o, to64

pytestmark = pytest.mark.gpu


def noalloc_status(cowa, q, kc, vc, sl, quad, out, lse):
    shape = cowa._shape(q, kc, vc, out, 0)
    return cowa.lib().cowa_decode_noalloc(
        ctypes.byref(shape), cowa._quad(quad), ctypes.c_float(0.0), cowa._ptr(q), cowa._ptr(kc),
        cowa._ptr(vc), cowa._ptr(sl), cowa._ptr(out), cowa._ptr(lse),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_decode_on_two_calls_in_a_row(oracle_mod):
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import bf16_bits, decode_inputs
    quad = (64, 512, 0, 896)
    runs = [(0, [4096, 4000, 129, 1]), (1, [77, 4096, 2048, 3000])]
    for seed, seqlens in runs:
        q, kc, vc, sl = decode_inputs(4, 4096, 16, 4, 128, seed=seed, seqlens=seqlens)
        o_ref, lse_ref = cowa.cowa_decode(q, kc, vc, sl, quad)
        out = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        assert noalloc_status(cowa, q, kc, vc, sl, quad, out, lse) == 0
        torch.cuda.synchronize()
        cowa.cowa_get_device_error()
        assert_o(out[:, 0], to64(o_ref[:, 0]), what="noalloc O")
        diff = (lse - lse_ref).abs().max().item()
        assert diff <= LSE_ABS
        # and against the oracle's decode of the same inputs
        o64, lse64 = oracle_mod.decode(bf16_bits(q[:, 0]), bf16_bits(kc), bf16_bits(vc), np.array(seqlens), quad)
        assert_o(out[:, 0], o64, what="noalloc O vs oracle")
        assert_lse(lse, lse64)


def test_noalloc_leaves_device_memory_unchanged():
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import decode_inputs
    quad = (64, 512, 0, 896)
    q, kc, vc, sl = decode_inputs(4, 4096, 16, 4, 128, seed=5, seqlens=[4096, 3000, 100, 1])
    out = torch.empty((4, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((4, 16), dtype=torch.float32, device="cuda")
    assert noalloc_status(cowa, q, kc, vc, sl, quad, out, lse) == 0  # first call: set-up
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert noalloc_status(cowa, q, kc, vc, sl, quad, out, lse) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0


def test_noalloc_python_wrapper():
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import decode_inputs
    quad = (16, 128, 0, 300)
    q, kc, vc, sl = decode_inputs(3, 1000, 8, 2, 64, seed=6, seqlens=[1000, 513, 2])
    o_ref, lse_ref = cowa.cowa_decode(q, kc, vc, sl, quad)
    out = torch.full_like(o_ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    o, l2 = cowa.cowa_decode_noalloc(q, kc, vc, sl, quad, out, lse)
    torch.cuda.synchronize()
    assert o.data_ptr() == out.data_ptr() and l2.data_ptr() == lse.data_ptr()
    assert_o(out[:, 0], to64(o_ref[:, 0]), what="noalloc O (wrapper)")
    assert (lse - lse_ref).abs().max().item() <= LSE_ABS


def test_noalloc_refuses_shapes_beyond_the_static_scratch():
    import structured_sparse_attention_block_b200 as cowa
    # 64 sequences x 64 query heads x d=128 need more split scratch than 4 MiB
    shape = cowa.Shape(64, 1, 1 << 16, 64, 8, 128, (ctypes.c_int64 * 3)(64 * 128, 64 * 128, 128),
                       (ctypes.c_int64 * 3)((1 << 16) * 8 * 128, 8 * 128, 128),
                       (ctypes.c_int64 * 3)((1 << 16) * 8 * 128, 8 * 128, 128),
                       (ctypes.c_int64 * 3)(64 * 128, 64 * 128, 128), 0)
    quad = cowa.Quad(128, 8192, 0, 7168)
    lib = cowa.lib()
    torch.cuda.init()
    assert lib.cowa_decode_workspace_size(ctypes.byref(shape), quad) > (4 << 20)
    st = lib.cowa_decode_noalloc(ctypes.byref(shape), quad, 0.0, *([None] * 6), None)
    assert st == 4
    assert "static limit" in lib.cowa_last_error_detail().decode()
