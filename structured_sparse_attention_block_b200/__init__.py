"""CoWindow Attention (CoWA) for B200: Python binding of ``libcowa.so``.

Argument marshalling only.  Every step of the operator runs in the library's
sm_100a kernels; PyTorch provides device memory and the current stream.
There is no CPU or eager fallback: if the library is missing or the tensors
are not on a CUDA device, the calls raise.

Entry points (same names as the C ABI in ``include/cowa.h``):

* ``cowa_fwd(q, k, v, quad)`` -> ``(o, lse)``: training / prefill forward,
  q [B, Lq, Hq, d], k/v [B, Lk, Hkv, d] bf16; lse [B, Hq, Lq] fp32.
* ``cowa_bwd(q, k, v, o, lse, dout, quad)`` -> ``(dq, dk, dv)``.
* ``cowa_decode(q, k_cache, v_cache, seqlens, quad)`` -> ``(o, lse)``:
  one new token per sequence, q [B, 1, Hq, d], caches [B, Lcap, Hkv, d],
  seqlens int32 [B] on the device.
* ``cowa_default_quad(Lk, Hkv, S, N)``: G = 0, W = ceil((Lk - N) / Hkv).
* ``cowa_tile_classes(...)``: the visible-tile map the kernels use.

The window quadruple ``quad`` is ``(S, N, G, W)``: sink width, near width,
gap and long-range width ("CoWindow Attention: Full Causal Coverage Is a
Collective Property", paper digest, method key points).
"""
import ctypes
import os

import torch

__all__ = ["CowaError", "cowa_fwd", "cowa_bwd", "cowa_decode", "cowa_default_quad",
           "cowa_tile_classes", "cowa_fwd_workspace_size", "cowa_bwd_workspace_size",
           "cowa_decode_workspace_size", "cowa_get_device_error", "cowa_launch_count",
           "cowa_decode_noalloc", "cowa_trace_start", "cowa_trace_stop", "cowa_trace_entries",
           "cowa_wcache_rows", "cowa_wcache_build", "cowa_wcache_append", "cowa_decode_windowed",
           "cowa_fwd_varlen", "cowa_bwd_varlen", "cowa_selftest_wait_timeout",
           "cowa_mala_fwd", "cowa_mala_bwd",
           "library_path", "lib"]

_HERE = os.path.dirname(os.path.abspath(__file__))
# COWA_DEBUG=1 selects the checking build (index checks in the kernels,
# failed checks reported as COWA_ERR_DEVICE); see build.py
_LIB_PATH = os.path.join(_HERE, "libcowa_debug.so" if os.environ.get("COWA_DEBUG") == "1" else "libcowa.so")
_lib = None

COWA_OK = 0
_STATUS = {0: "COWA_OK", 1: "COWA_ERR_INVALID_ARG", 2: "COWA_ERR_UNSUPPORTED",
           3: "COWA_ERR_ALIGNMENT", 4: "COWA_ERR_WORKSPACE", 5: "COWA_ERR_CUDA",
           6: "COWA_ERR_TIMEOUT", 7: "COWA_ERR_DEVICE"}


class CowaError(RuntimeError):
    def __init__(self, status, detail):
        self.status = status
        super().__init__("%s: %s" % (_STATUS.get(status, status), detail))


class Quad(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("N", ctypes.c_int32), ("G", ctypes.c_int32),
                ("W", ctypes.c_int32)]


class VarlenShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
                ("max_q", ctypes.c_int64), ("max_k", ctypes.c_int64), ("Hq", ctypes.c_int64),
                ("Hkv", ctypes.c_int64), ("d", ctypes.c_int64),
                ("q_stride", ctypes.c_int64 * 2), ("k_stride", ctypes.c_int64 * 2),
                ("v_stride", ctypes.c_int64 * 2), ("o_stride", ctypes.c_int64 * 2),
                ("kv_head_offset", ctypes.c_int64)]


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("Lq", ctypes.c_int64), ("Lk", ctypes.c_int64),
                ("Hq", ctypes.c_int64), ("Hkv", ctypes.c_int64), ("d", ctypes.c_int64),
                ("q_stride", ctypes.c_int64 * 3), ("k_stride", ctypes.c_int64 * 3),
                ("v_stride", ctypes.c_int64 * 3), ("o_stride", ctypes.c_int64 * 3),
                ("kv_head_offset", ctypes.c_int64)]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded ``libcowa.so`` (``libcowa_debug.so`` under COWA_DEBUG=1);
    raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                "%s is missing: build it with `python -m structured_sparse_attention_block_b200.build%s`"
                % (_LIB_PATH, " --debug" if _LIB_PATH.endswith("_debug.so") else ""))
        L = ctypes.CDLL(_LIB_PATH)
        vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
        SP = ctypes.POINTER(Shape)
        L.cowa_status_string.restype = ctypes.c_char_p
        L.cowa_status_string.argtypes = [ctypes.c_int]
        L.cowa_last_error_detail.restype = ctypes.c_char_p
        L.cowa_abi_version.restype = ctypes.c_int
        L.cowa_launch_count.restype = ctypes.c_uint64
        L.cowa_default_quad.restype = Quad
        L.cowa_default_quad.argtypes = [i64, i64, i32, i32]
        for name in ("cowa_fwd_workspace_size", "cowa_bwd_workspace_size",
                     "cowa_decode_workspace_size"):
            f = getattr(L, name)
            f.restype = sz
            f.argtypes = [SP, Quad]
        L.cowa_fwd.restype = ctypes.c_int
        L.cowa_fwd.argtypes = [SP, Quad, ctypes.c_float, vp, vp, vp, vp, vp, vp, sz, vp]
        L.cowa_bwd.restype = ctypes.c_int
        L.cowa_bwd.argtypes = [SP, Quad, ctypes.c_float] + [vp] * 9 + [vp, sz, vp]
        L.cowa_decode.restype = ctypes.c_int
        L.cowa_decode.argtypes = [SP, Quad, ctypes.c_float] + [vp] * 6 + [vp, sz, vp]
        L.cowa_mala_keep_bytes.restype = sz
        L.cowa_mala_keep_bytes.argtypes = [SP]
        L.cowa_mala_fwd.restype = ctypes.c_int
        L.cowa_mala_fwd.argtypes = [SP, ctypes.c_float, ctypes.c_float] + [vp] * 7
        L.cowa_mala_bwd_workspace_size.restype = sz
        L.cowa_mala_bwd_workspace_size.argtypes = [SP]
        L.cowa_mala_bwd.restype = ctypes.c_int
        L.cowa_mala_bwd.argtypes = [SP, ctypes.c_float] + [vp] * 10 + [vp, sz, vp]
        L.cowa_decode_noalloc.restype = ctypes.c_int
        L.cowa_decode_noalloc.argtypes = [SP, Quad, ctypes.c_float] + [vp] * 6 + [vp]
        L.cowa_schedule_workspace_size.restype = sz
        L.cowa_schedule_workspace_size.argtypes = [i64, i64, i32, i32]
        L.cowa_tile_classes.restype = ctypes.c_int
        L.cowa_tile_classes.argtypes = [i64, i64, i64, Quad, i32, i32, ctypes.c_int, vp, vp, sz, vp]
        L.cowa_get_device_error.restype = ctypes.c_int
        L.cowa_get_device_error.argtypes = [vp]
        L.cowa_selftest_wait_timeout.restype = ctypes.c_int
        L.cowa_selftest_wait_timeout.argtypes = [vp]
        VP = ctypes.POINTER(VarlenShape)
        for name in ("cowa_fwd_varlen_workspace_size", "cowa_bwd_varlen_workspace_size"):
            f = getattr(L, name)
            f.restype = sz
            f.argtypes = [VP, Quad]
        L.cowa_fwd_varlen.restype = ctypes.c_int
        L.cowa_fwd_varlen.argtypes = [VP, Quad, ctypes.c_float] + [vp] * 7 + [vp, sz, vp]
        L.cowa_bwd_varlen.restype = ctypes.c_int
        L.cowa_bwd_varlen.argtypes = [VP, Quad, ctypes.c_float] + [vp] * 11 + [vp, sz, vp]
        L.cowa_wcache_rows.restype = i64
        L.cowa_wcache_rows.argtypes = [Quad, i32]
        L.cowa_wcache_build.restype = ctypes.c_int
        L.cowa_wcache_build.argtypes = [SP, Quad, i32, vp, vp, vp, vp, vp, vp]
        L.cowa_wcache_append.restype = ctypes.c_int
        L.cowa_wcache_append.argtypes = [SP, Quad, i32, vp, vp, vp, vp, vp, vp, vp]
        L.cowa_decode_windowed.restype = ctypes.c_int
        L.cowa_decode_windowed.argtypes = [SP, Quad, ctypes.c_float, i32] + [vp] * 7 + [vp, sz, vp]
        L.cowa_trace_start.restype = ctypes.c_int
        L.cowa_trace_start.argtypes = [i64, ctypes.c_char_p]
        L.cowa_trace_stop.restype = ctypes.c_int
        L.cowa_trace_size.restype = i64
        L.cowa_trace_dropped.restype = i64
        L.cowa_trace_entry.restype = ctypes.c_int
        L.cowa_trace_entry.argtypes = [i64, ctypes.POINTER(ctypes.c_char_p),
                                       ctypes.POINTER(ctypes.c_float)]
        _lib = L
    return _lib


def _check(status):
    if status != COWA_OK:
        raise CowaError(status, lib().cowa_last_error_detail().decode())


def _quad(quad) -> Quad:
    if isinstance(quad, Quad):
        return quad
    S, N, G, W = (int(x) for x in quad)
    return Quad(S, N, G, W)


def cowa_default_quad(Lk, Hkv, S, N):
    """(S, N, 0, ceil((Lk - N) / Hkv)) with W clamped at 0; Hkv is the global count."""
    q = lib().cowa_default_quad(int(Lk), int(Hkv), int(S), int(N))
    return (q.S, q.N, q.G, q.W)


def _bf16_cuda(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != torch.bfloat16:
        raise TypeError("%s must be bfloat16 (got %s)" % (name, t.dtype))
    if t.dim() != 4 or (t.numel() > 0 and t.stride(3) != 1):
        raise ValueError("%s must be [B, L, H, d] with a contiguous last dimension" % name)


def _strides(t):
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def _shape(q, k, v, o, kv_head_offset):
    B, Lq, Hq, d = q.shape
    _, Lk, Hkv, _ = k.shape
    return Shape(B, Lq, Lk, Hq, Hkv, d, _strides(q), _strides(k), _strides(v), _strides(o),
                 int(kv_head_offset))


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() > 0 else None


def _workspace(nbytes, device, workspace):
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small: need %d bytes" % nbytes)
        return workspace
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def cowa_fwd_workspace_size(q, k, quad, kv_head_offset=0):
    return int(lib().cowa_fwd_workspace_size(ctypes.byref(_shape(q, k, k, q, kv_head_offset)), _quad(quad)))


def cowa_bwd_workspace_size(q, k, quad, kv_head_offset=0):
    return int(lib().cowa_bwd_workspace_size(ctypes.byref(_shape(q, k, k, q, kv_head_offset)), _quad(quad)))


def cowa_decode_workspace_size(q, k_cache, quad, kv_head_offset=0):
    q4 = q if q.dim() == 4 else q.unsqueeze(1)
    return int(lib().cowa_decode_workspace_size(
        ctypes.byref(_shape(q4, k_cache, k_cache, q4, kv_head_offset)), _quad(quad)))


def cowa_fwd(q, k, v, quad, softmax_scale=None, kv_head_offset=0, out=None, lse=None,
             workspace=None):
    """CoWA forward.  Returns ``(o, lse)``; see the module docstring."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16_cuda(t, n)
    B, Lq, Hq, d = q.shape
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    _bf16_cuda(out, "out")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Lq):
        raise ValueError("lse must be contiguous fp32 [B, Hq, Lq]")
    shape = _shape(q, k, v, out, kv_head_offset)
    qd = _quad(quad)
    L = lib()
    need = L.cowa_fwd_workspace_size(ctypes.byref(shape), qd)
    if need == 0:
        _raise_size_error(L)
    ws = _workspace(need, q.device, workspace)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(L.cowa_fwd(ctypes.byref(shape), qd, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                      _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)))
    return out, lse


def cowa_mala_fwd(q, k, v, tau, softmax_scale=None, out=None, lse=None, keep=None):
    """MALA forward (full causal scoring; blocks of 128 query rows x 64 keys
    kept when some row gives them at least ``tau`` of its softmax mass).
    Returns ``(o, lse, keep)`` with keep uint8 [B, Hq, ceil(Lq/128),
    ceil(Lk/64)]; see ``cowa_mala_fwd`` in include/cowa.h."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16_cuda(t, n)
    B, Lq, Hq, d = q.shape
    Lk = k.shape[1]
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    kshape = (B, Hq, -(-Lq // 128), -(-Lk // 64))
    if keep is None:
        keep = torch.empty(kshape, dtype=torch.uint8, device=q.device)
    _bf16_cuda(out, "out")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Lq):
        raise ValueError("lse must be contiguous fp32 [B, Hq, Lq]")
    if keep.dtype != torch.uint8 or not keep.is_contiguous() or tuple(keep.shape) != kshape:
        raise ValueError("keep must be contiguous uint8 %s" % (kshape,))
    shape = _shape(q, k, v, out, 0)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(lib().cowa_mala_fwd(ctypes.byref(shape), float(tau), scale, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                               _ptr(lse), _ptr(keep), _stream(q.device)))
    return out, lse, keep


def cowa_mala_bwd(q, k, v, o, lse, keep, dout, softmax_scale=None, dq=None, dk=None, dv=None,
                  workspace=None):
    """MALA backward with the forward's block decisions held fixed.  Returns
    ``(dq, dk, dv)``; dO uses o's strides, each gradient its input's."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _bf16_cuda(t, n)
    if dout.stride() != o.stride():
        raise ValueError("dout must have the strides of o")
    dq = torch.empty_strided(q.shape, q.stride(), dtype=q.dtype, device=q.device) if dq is None else dq
    dk = torch.empty_strided(k.shape, k.stride(), dtype=k.dtype, device=k.device) if dk is None else dk
    dv = torch.empty_strided(v.shape, v.stride(), dtype=v.dtype, device=v.device) if dv is None else dv
    for t, ref, n in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        _bf16_cuda(t, n)
        if t.stride() != ref.stride() or t.shape != ref.shape:
            raise ValueError("%s must match the shape and strides of its input" % n)
    B, Lq, Hq, d = q.shape
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Lq):
        raise ValueError("lse must be contiguous fp32 [B, Hq, Lq]")
    kshape = (B, Hq, -(-Lq // 128), -(-k.shape[1] // 64))
    if keep.dtype != torch.uint8 or not keep.is_contiguous() or tuple(keep.shape) != kshape:
        raise ValueError("keep must be contiguous uint8 %s" % (kshape,))
    shape = _shape(q, k, v, o, 0)
    L = lib()
    need = L.cowa_mala_bwd_workspace_size(ctypes.byref(shape))
    if need == 0:
        _raise_size_error(L)
    ws = _workspace(need, q.device, workspace)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(L.cowa_mala_bwd(ctypes.byref(shape), scale, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(keep),
                           _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream(q.device)))
    return dq, dk, dv


def _raise_size_error(L):
    """A workspace query returned 0: the arguments were rejected."""
    detail = L.cowa_last_error_detail().decode()
    raise CowaError(1, detail or "invalid arguments")


def cowa_bwd(q, k, v, o, lse, dout, quad, softmax_scale=None, kv_head_offset=0,
             dq=None, dk=None, dv=None, workspace=None):
    """CoWA backward.  Returns ``(dq, dk, dv)``; dO uses o's strides, dQ q's,
    dK k's and dV v's (pass dq/dk/dv to choose them)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _bf16_cuda(t, n)
    if dout.stride() != o.stride():
        raise ValueError("dout must have the strides of o")
    # the C ABI gives each gradient the strides of its input
    dq = torch.empty_strided(q.shape, q.stride(), dtype=q.dtype, device=q.device) if dq is None else dq
    dk = torch.empty_strided(k.shape, k.stride(), dtype=k.dtype, device=k.device) if dk is None else dk
    dv = torch.empty_strided(v.shape, v.stride(), dtype=v.dtype, device=v.device) if dv is None else dv
    for t, ref, n in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        _bf16_cuda(t, n)
        if t.stride() != ref.stride() or t.shape != ref.shape:
            raise ValueError("%s must match the shape and strides of its input" % n)
    B, Lq, Hq, d = q.shape
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Lq):
        raise ValueError("lse must be contiguous fp32 [B, Hq, Lq]")
    shape = _shape(q, k, v, o, kv_head_offset)
    qd = _quad(quad)
    L = lib()
    need = L.cowa_bwd_workspace_size(ctypes.byref(shape), qd)
    if need == 0:
        _raise_size_error(L)
    ws = _workspace(need, q.device, workspace)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(L.cowa_bwd(ctypes.byref(shape), qd, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                      _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                      _stream(q.device)))
    return dq, dk, dv


def cowa_decode(q, k_cache, v_cache, seqlens, quad, softmax_scale=None, kv_head_offset=0,
                out=None, lse=None, workspace=None):
    """CoWA single-token decode.  q [B, 1, Hq, d] (or [B, Hq, d]); returns
    ``(o [B, 1, Hq, d], lse [B, Hq])``."""
    q4 = q if q.dim() == 4 else q.unsqueeze(1)
    for t, n in ((q4, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16_cuda(t, n)
    if seqlens.dtype != torch.int32 or not seqlens.is_cuda or not seqlens.is_contiguous():
        raise TypeError("seqlens must be a contiguous int32 CUDA tensor")
    B, _, Hq, d = q4.shape
    if out is None:
        out = torch.empty((B, 1, Hq, d), dtype=torch.bfloat16, device=q4.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q4.device)
    _bf16_cuda(out, "out")
    shape = _shape(q4, k_cache, v_cache, out, kv_head_offset)
    qd = _quad(quad)
    L = lib()
    need = L.cowa_decode_workspace_size(ctypes.byref(shape), qd)
    if need == 0:
        _raise_size_error(L)
    ws = _workspace(need, q4.device, workspace)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(L.cowa_decode(ctypes.byref(shape), qd, scale, _ptr(q4), _ptr(k_cache), _ptr(v_cache),
                         _ptr(seqlens), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                         _stream(q4.device)))
    return out, lse


def _packed(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16:
        raise TypeError("%s must be a bf16 CUDA tensor" % name)
    if t.dim() != 3 or (t.numel() > 0 and t.stride(2) != 1):
        raise ValueError("%s must be [total, H, d] with a contiguous last dimension" % name)


def _varlen_shape(q, k, v, o, cu_q, max_q, max_k, kv_head_offset):
    s2 = lambda t: (ctypes.c_int64 * 2)(t.stride(0), t.stride(1))
    return VarlenShape(cu_q.numel() - 1, q.shape[0], k.shape[0], int(max_q), int(max_k), q.shape[1], k.shape[1],
                       q.shape[2], s2(q), s2(k), s2(v), s2(o), int(kv_head_offset))


def cowa_fwd_varlen(q, k, v, cu_q, cu_k, max_q, max_k, quad, softmax_scale=None, kv_head_offset=0,
                    out=None, lse=None, workspace=None):
    """CoWA forward over a packed batch: q [total_q, Hq, d], k/v [total_k, Hkv, d],
    cu_q / cu_k int32 CUDA [B + 1] offsets, max_q / max_k the longest
    sequences.  Returns ``(o [total_q, Hq, d], lse [Hq, total_q])``."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _packed(t, n)
    _int32_cuda(cu_q, "cu_q")
    _int32_cuda(cu_k, "cu_k")
    if cu_k.numel() != cu_q.numel():
        raise ValueError("cu_q and cu_k must have the same length")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    _packed(out, "out")
    shape = _varlen_shape(q, k, v, out, cu_q, max_q, max_k, kv_head_offset)
    qd = _quad(quad)
    L = lib()
    need = L.cowa_fwd_varlen_workspace_size(ctypes.byref(shape), qd)
    if need == 0:
        _raise_size_error(L)
    ws = _workspace(need, q.device, workspace)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(L.cowa_fwd_varlen(ctypes.byref(shape), qd, scale, _ptr(cu_q), _ptr(cu_k), _ptr(q), _ptr(k), _ptr(v),
                             _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)))
    return out, lse


def cowa_bwd_varlen(q, k, v, o, lse, dout, cu_q, cu_k, max_q, max_k, quad, softmax_scale=None,
                    kv_head_offset=0, workspace=None):
    """CoWA backward over a packed batch; returns ``(dq, dk, dv)`` shaped like
    q, k, v (dO must have o's strides)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _packed(t, n)
    _int32_cuda(cu_q, "cu_q")
    _int32_cuda(cu_k, "cu_k")
    if dout.stride() != o.stride():
        raise ValueError("dout must have the strides of o")
    dq = torch.empty_strided(q.shape, q.stride(), dtype=q.dtype, device=q.device)
    dk = torch.empty_strided(k.shape, k.stride(), dtype=k.dtype, device=k.device)
    dv = torch.empty_strided(v.shape, v.stride(), dtype=v.dtype, device=v.device)
    shape = _varlen_shape(q, k, v, o, cu_q, max_q, max_k, kv_head_offset)
    qd = _quad(quad)
    L = lib()
    need = L.cowa_bwd_varlen_workspace_size(ctypes.byref(shape), qd)
    if need == 0:
        _raise_size_error(L)
    ws = _workspace(need, q.device, workspace)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(L.cowa_bwd_varlen(ctypes.byref(shape), qd, scale, _ptr(cu_q), _ptr(cu_k), _ptr(q), _ptr(k), _ptr(v),
                             _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                             _stream(q.device)))
    return dq, dk, dv


def _int32_cuda(t, name):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError("%s must be a contiguous int32 CUDA tensor" % name)


def cowa_wcache_rows(quad, horizon) -> int:
    """Rows of a windowed decode cache serving ``horizon`` query positions."""
    return int(lib().cowa_wcache_rows(_quad(quad), int(horizon)))


def cowa_wcache_build(k_cache, v_cache, origin, quad, horizon, kv_head_offset=0):
    """Windowed decode cache ``(k_win, v_win)`` [B, rows, Hkv, d] from a full
    cache [B, L, Hkv, d] for query positions [origin[b], origin[b] + horizon)
    of each sequence (origin: int32 CUDA [B]; keys 0..origin[b] must be in
    the full cache)."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16_cuda(t, n)
    _int32_cuda(origin, "origin")
    B, Lk, Hkv, d = k_cache.shape
    rows = cowa_wcache_rows(quad, horizon)
    if rows <= 0:
        raise ValueError("bad quadruple or horizon")
    kw = torch.empty((B, rows, Hkv, d), dtype=torch.bfloat16, device=k_cache.device)
    vw = torch.empty_like(kw)
    shape = Shape(B, 1, Lk, Hkv, Hkv, d, _strides(k_cache), _strides(k_cache), _strides(v_cache),
                  _strides(k_cache), int(kv_head_offset))
    _check(lib().cowa_wcache_build(ctypes.byref(shape), _quad(quad), int(horizon), _ptr(origin),
                                   _ptr(k_cache), _ptr(v_cache), _ptr(kw), _ptr(vw), _stream(k_cache.device)))
    return kw, vw


def cowa_wcache_append(k_win, v_win, k_new, v_new, pos, origin, quad, horizon, kv_head_offset=0):
    """Write the K/V rows k_new/v_new [B, Hkv, d] of the tokens at positions
    pos (int32 CUDA [B]) into the windowed cache (in place)."""
    for t, n in ((k_win, "k_win"), (v_win, "v_win")):
        _bf16_cuda(t, n)
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 3 \
                or t.stride(2) != 1:
            raise TypeError("%s must be a bf16 CUDA tensor [B, Hkv, d] with a contiguous last dimension" % n)
    _int32_cuda(pos, "pos")
    _int32_cuda(origin, "origin")
    B, rows, Hkv, d = k_win.shape
    ks = (ctypes.c_int64 * 3)(k_new.stride(0), 0, k_new.stride(1))
    vs = (ctypes.c_int64 * 3)(v_new.stride(0), 0, v_new.stride(1))
    shape = Shape(B, 1, rows, Hkv, Hkv, d, ks, ks, vs, ks, int(kv_head_offset))
    _check(lib().cowa_wcache_append(ctypes.byref(shape), _quad(quad), int(horizon), _ptr(origin), _ptr(pos),
                                    _ptr(k_new), _ptr(v_new), _ptr(k_win), _ptr(v_win), _stream(k_win.device)))


def cowa_decode_windowed(q, k_win, v_win, seqlens, origin, quad, horizon, softmax_scale=None,
                         kv_head_offset=0, out=None, lse=None, workspace=None):
    """CoWA decode over a windowed cache; the query of sequence b sits at
    seqlens[b] - 1, inside [origin[b], origin[b] + horizon).  Returns
    ``(o [B, 1, Hq, d], lse [B, Hq])``."""
    q4 = q if q.dim() == 4 else q.unsqueeze(1)
    for t, n in ((q4, "q"), (k_win, "k_win"), (v_win, "v_win")):
        _bf16_cuda(t, n)
    _int32_cuda(seqlens, "seqlens")
    _int32_cuda(origin, "origin")
    B, _, Hq, d = q4.shape
    if out is None:
        out = torch.empty((B, 1, Hq, d), dtype=torch.bfloat16, device=q4.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q4.device)
    _bf16_cuda(out, "out")
    shape = _shape(q4, k_win, v_win, out, kv_head_offset)
    qd = _quad(quad)
    L = lib()
    need = L.cowa_decode_workspace_size(ctypes.byref(shape), qd)
    if need == 0:
        _raise_size_error(L)
    ws = _workspace(need, q4.device, workspace)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(L.cowa_decode_windowed(ctypes.byref(shape), qd, scale, int(horizon), _ptr(origin), _ptr(q4),
                                  _ptr(k_win), _ptr(v_win), _ptr(seqlens), _ptr(out), _ptr(lse), _ptr(ws),
                                  ws.numel(), _stream(q4.device)))
    return out, lse


def cowa_decode_noalloc(q, k_cache, v_cache, seqlens, quad, out, lse, softmax_scale=None,
                        kv_head_offset=0):
    """Decode that allocates no device memory, for callers that cannot
    allocate (for example a plugin inside a runtime that owns all device
    memory).  The caller passes every buffer, out [B, 1, Hq, d] bf16 and
    lse [B, Hq] fp32 included; the split scratch is a fixed array inside the
    library (``COWA_DECODE_NOALLOC_SCRATCH_BYTES``, 4 MiB per GPU).  Calls on
    one device must not overlap on the GPU.  Returns ``(out, lse)``."""
    q4 = q if q.dim() == 4 else q.unsqueeze(1)
    for t, n in ((q4, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (out, "out")):
        _bf16_cuda(t, n)
    if seqlens.dtype != torch.int32 or not seqlens.is_cuda or not seqlens.is_contiguous():
        raise TypeError("seqlens must be a contiguous int32 CUDA tensor")
    B, _, Hq, d = q4.shape
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq):
        raise ValueError("lse must be contiguous fp32 [B, Hq]")
    shape = _shape(q4, k_cache, v_cache, out, kv_head_offset)
    scale = 0.0 if softmax_scale is None else float(softmax_scale)
    _check(lib().cowa_decode_noalloc(ctypes.byref(shape), _quad(quad), scale, _ptr(q4), _ptr(k_cache),
                                     _ptr(v_cache), _ptr(seqlens), _ptr(out), _ptr(lse),
                                     _stream(q4.device)))
    return out, lse


def cowa_tile_classes(Lq, Lk, kv_head, quad, BM, BN=64, transposed=False, device="cuda"):
    """uint8 [ceil(Lq/BM), ceil(Lk/BN)]: 0 skipped, 1 masked, 2 unmasked tile."""
    L = lib()
    nqt, nkt = -(-Lq // BM), -(-Lk // BN)
    out = torch.empty((nqt, nkt), dtype=torch.uint8, device=device)
    need = L.cowa_schedule_workspace_size(Lq, Lk, BM, BN)
    ws = torch.empty(max(int(need), 1), dtype=torch.uint8, device=device)
    _check(L.cowa_tile_classes(Lq, Lk, kv_head, _quad(quad), BM, BN, int(bool(transposed)),
                               _ptr(out), _ptr(ws), ws.numel(), _stream(torch.device(device))))
    return out


def cowa_launch_count() -> int:
    """Kernels the library has launched in this process (all devices)."""
    return int(lib().cowa_launch_count())


def cowa_trace_start(capacity: int, only: str = None) -> None:
    """Record a CUDA event pair around each of the next ``capacity`` library
    launches on the current device -- of the kernel named ``only``, if given
    (0 turns tracing off)."""
    _check(lib().cowa_trace_start(int(capacity), only.encode() if only else None))


def cowa_trace_stop() -> None:
    _check(lib().cowa_trace_stop())


def cowa_trace_entries():
    """(kernel name, milliseconds) of every traced launch, in launch order,
    and the number of launches that were not recorded."""
    L = lib()
    out = []
    name, ms = ctypes.c_char_p(), ctypes.c_float()
    for i in range(int(L.cowa_trace_size())):
        _check(L.cowa_trace_entry(i, ctypes.byref(name), ctypes.byref(ms)))
        out.append((name.value.decode(), float(ms.value)))
    return out, int(L.cowa_trace_dropped())


def cowa_selftest_wait_timeout(device=None):
    """Launch the timeout self-test: a block whose bounded wait on a barrier
    that nothing completes runs out after 2 s and records COWA_ERR_TIMEOUT,
    which the next cowa_get_device_error raises."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(lib().cowa_selftest_wait_timeout(_stream(dev)))


def cowa_get_device_error(device=None):
    """Synchronise and raise if a kernel recorded a device-side error."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(lib().cowa_get_device_error(_stream(dev)))
