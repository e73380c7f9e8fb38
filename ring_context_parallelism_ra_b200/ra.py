"""ctypes binding of libra.so (the C ABI in include/ra.h).

Argument marshalling only: checks that tensors are CUDA, contiguous and of the
right dtype, allocates outputs with torch when the caller passes none, and
hands raw pointers plus the current CUDA stream to the library.  Every step
of the computation runs in the library's kernels.  If libra.so is missing or
fails to load, every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import numpy as np
import torch

__all__ = [
    "RAError", "library_path", "lib", "Shape", "block_partial", "block_partial_strided",
    "lse_merge", "ring_forward", "ring_forward_striped",
    "ring_forward_host", "ring_forward_host_workspace_bytes", "decode_workspace_bytes", "decode_partial", "decode_partials",
    "decode_partial_noalloc",
    "decode_merge",
    "decode_pass_q", "backward_workspace_bytes", "backward_delta", "ring_backward",
    "ring_backward_striped", "block_backward",
    "block_class", "block_class_device", "get_status", "set_wait_limit_ns",
    "check_wait_timeout", "launch_count", "status_string", "EXPORTED",
]

RA_OK, RA_ERR_INVALID, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_TIMEOUT = 0, -1, -2, -3, -4
RA_F32, RA_BF16 = 0, 1

# Every symbol include/ra.h declares.
EXPORTED = (
    "ra_block_partial", "ra_block_partial_strided", "ra_lse_merge", "ra_ring_forward",
    "ra_ring_forward_striped", "ra_ring_forward_host_workspace_bytes", "ra_ring_forward_host",
    "ra_decode_workspace_bytes",
    "ra_decode_partial", "ra_decode_partials", "ra_decode_partial_noalloc", "ra_decode_merge",
    "ra_backward_workspace_bytes", "ra_backward_delta", "ra_ring_backward",
    "ra_ring_backward_striped", "ra_block_backward", "ra_block_class", "ra_block_class_device",
    "ra_get_status", "ra_set_wait_limit_ns", "ra_check_wait_timeout", "ra_status_string",
    "ra_launch_count", "ra_shutdown",
)


class RAError(RuntimeError):
    def __init__(self, func: str, status: int):
        self.status = status
        super().__init__(f"{func}: {status_string(status)} ({status})")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("n_q", ctypes.c_int), ("n_k", ctypes.c_int), ("d_qk", ctypes.c_int),
                ("d_v", ctypes.c_int), ("dtype", ctypes.c_int)]


_LIB = None
_LOCK = threading.Lock()


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libra.so")


def lib() -> ctypes.CDLL:
    """Load libra.so once; raise if it is absent (build it with ``build.py``)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    with _LOCK:
        if _LIB is not None:
            return _LIB
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run `python -m ring_context_parallelism_ra_b200.build`")
        L = ctypes.CDLL(path)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        sp = ctypes.POINTER(Shape)
        sig = {
            "ra_block_partial": (i, [vp, vp, vp, sp, i, i, i, f, vp, vp, vp]),
            "ra_block_partial_strided": (i, [vp, vp, vp, sp, i, i, i, i, f, vp, vp, vp]),
            "ra_ring_forward_striped": (i, [vp, vp, vp, i, i, f, vp, vp, sp, vp]),
            "ra_lse_merge": (i, [vp, vp, i, sp, vp, i, vp, vp]),
            "ra_ring_forward": (i, [vp, vp, vp, i, i, f, vp, vp, sp, vp]),
            "ra_ring_forward_host_workspace_bytes": (sz, [sp]),
            "ra_ring_forward_host": (i, [vp, vp, vp, i, i, f, vp, vp, sp, vp, sz, vp]),
            "ra_decode_workspace_bytes": (sz, [sp]),
            "ra_decode_partial": (i, [vp, vp, vp, ctypes.c_longlong, sp, f, vp, vp, vp, sz, vp]),
            "ra_decode_partial_noalloc": (i, [vp, vp, vp, ctypes.c_longlong, sp, f, vp, vp, vp]),
            "ra_decode_partials": (i, [vp, vp, vp, i, sp, f, vp, vp, vp, sz, vp]),
            "ra_decode_merge": (i, [vp, vp, i, sp, vp, i, vp, vp]),
            "ra_backward_workspace_bytes": (sz, [sp]),
            "ra_backward_delta": (i, [vp, vp, sp, vp, vp]),
            "ra_ring_backward": (i, [vp, vp, vp, vp, vp, vp, i, i, f, vp, vp, vp, sp, vp, sz, vp]),
            "ra_ring_backward_striped": (i, [vp, vp, vp, vp, vp, vp, i, i, f, vp, vp, vp, sp, vp,
                                             sz, vp]),
            "ra_block_backward": (i, [vp, vp, vp, vp, vp, vp, sp, i, i, i, i, f, vp, vp, vp, vp,
                                      sz, vp]),
            "ra_block_class": (i, [i, i, i, i, i, i, i, vp]),
            "ra_block_class_device": (i, [i, i, i, i, i, i, i, vp, vp]),
            "ra_get_status": (i, [vp]),
            "ra_set_wait_limit_ns": (i, [ctypes.c_ulonglong]),
            "ra_check_wait_timeout": (i, [ctypes.c_ulonglong, vp]),
            "ra_status_string": (ctypes.c_char_p, [i]),
            "ra_launch_count": (ctypes.c_ulonglong, []),
            "ra_shutdown": (i, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _LIB = L
        return L


def status_string(status: int) -> str:
    return lib().ra_status_string(int(status)).decode()


def _check(func: str, rc: int):
    if rc != RA_OK:
        raise RAError(func, rc)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return RA_F32
    if t == torch.bfloat16:
        return RA_BF16
    raise TypeError(f"unsupported dtype {t}")


def _need(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _shape(q, k, v, n_q=None) -> Shape:
    B, Hq, nq, dqk = q.shape
    Bk, Hkv, nk, dqk2 = k.shape
    if Bk != B or dqk2 != dqk or v.shape[:3] != k.shape[:3]:
        raise ValueError("inconsistent q/k/v shapes")
    return Shape(B, Hq, Hkv, nq if n_q is None else n_q, nk, dqk, v.shape[-1], _dtype_code(q.dtype))


def block_partial(q, k, v, q_offset=0, k_offset=0, causal=True, scale=None, o_part=None,
                  lse_part=None, stream=None):
    """Partial (O normalised over this block, LSE) of one Q range vs one KV range."""
    s = _shape(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    if o_part is None:
        o_part = torch.empty((s.B, s.Hq, s.n_q, s.d_v), device=q.device, dtype=torch.float32)
    if lse_part is None:
        lse_part = torch.empty((s.B, s.Hq, s.n_q), device=q.device, dtype=torch.float32)
    rc = lib().ra_block_partial(_need(q, "q"), _need(k, "k", q.dtype), _need(v, "v", q.dtype),
                                ctypes.byref(s), int(q_offset), int(k_offset), int(bool(causal)),
                                float(scale), _need(o_part, "o_part", torch.float32),
                                _need(lse_part, "lse_part", torch.float32), _stream(stream))
    _check("ra_block_partial", rc)
    return o_part, lse_part


def block_partial_strided(q, k, v, q_offset, k_offset, pos_stride, causal=True, scale=None,
                          o_part=None, lse_part=None, stream=None):
    """Block partial with positions q_offset + t * pos_stride / k_offset + u * pos_stride
    (the (i, j) block of a striped split is q_offset = i, k_offset = j, pos_stride = P)."""
    s = _shape(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    if o_part is None:
        o_part = torch.empty((s.B, s.Hq, s.n_q, s.d_v), device=q.device, dtype=torch.float32)
    if lse_part is None:
        lse_part = torch.empty((s.B, s.Hq, s.n_q), device=q.device, dtype=torch.float32)
    rc = lib().ra_block_partial_strided(_need(q, "q"), _need(k, "k", q.dtype),
                                        _need(v, "v", q.dtype), ctypes.byref(s), int(q_offset),
                                        int(k_offset), int(pos_stride), int(bool(causal)),
                                        float(scale), _need(o_part, "o_part", torch.float32),
                                        _need(lse_part, "lse_part", torch.float32), _stream(stream))
    _check("ra_block_partial_strided", rc)
    return o_part, lse_part


def lse_merge(o_parts, lse_parts, out_dtype=torch.float32, out=None, lse=None, stream=None,
              _name="ra_lse_merge"):
    """Merge P stacked partials o_parts [P,B,H,n,d_v], lse_parts [P,B,H,n]."""
    P, B, H, n, dv = o_parts.shape
    if lse_parts.shape != (P, B, H, n):
        raise ValueError("lse_parts shape mismatch")
    if out is None:
        out = torch.empty((B, H, n, dv), device=o_parts.device, dtype=out_dtype)
    if lse is None:
        lse = torch.empty((B, H, n), device=o_parts.device, dtype=torch.float32)
    s = Shape(B, H, H, n, n, dv, dv, RA_F32)
    fn = getattr(lib(), _name)
    rc = fn(_need(o_parts, "o_parts", torch.float32), _need(lse_parts, "lse_parts", torch.float32),
            int(P), ctypes.byref(s), _need(out, "out", out_dtype), _dtype_code(out_dtype),
            _need(lse, "lse", torch.float32), _stream(stream))
    _check(_name, rc)
    return out, lse


def ring_forward(q, k, v, P, causal=True, scale=None, out=None, lse=None, stream=None):
    """Fused ring over P partitions of one sequence: (O [B,Hq,n,d_v], LSE [B,Hq,n])."""
    s = _shape(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    if out is None:
        out = torch.empty((s.B, s.Hq, s.n_q, s.d_v), device=q.device, dtype=q.dtype)
    if lse is None:
        lse = torch.empty((s.B, s.Hq, s.n_q), device=q.device, dtype=torch.float32)
    rc = lib().ra_ring_forward(_need(q, "q"), _need(k, "k", q.dtype), _need(v, "v", q.dtype),
                               int(P), int(bool(causal)), float(scale), _need(out, "out", q.dtype),
                               _need(lse, "lse", torch.float32), ctypes.byref(s), _stream(stream))
    _check("ra_ring_forward", rc)
    return out, lse


def ring_forward_striped(q, k, v, P, causal=True, scale=None, out=None, lse=None, stream=None):
    """Fused ring over a striped split: row i * (n / P) + r of q, k, v, out and
    lse is token r * P + i."""
    s = _shape(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    if out is None:
        out = torch.empty((s.B, s.Hq, s.n_q, s.d_v), device=q.device, dtype=q.dtype)
    if lse is None:
        lse = torch.empty((s.B, s.Hq, s.n_q), device=q.device, dtype=torch.float32)
    rc = lib().ra_ring_forward_striped(_need(q, "q"), _need(k, "k", q.dtype),
                                       _need(v, "v", q.dtype), int(P), int(bool(causal)),
                                       float(scale), _need(out, "out", q.dtype),
                                       _need(lse, "lse", torch.float32), ctypes.byref(s),
                                       _stream(stream))
    _check("ra_ring_forward_striped", rc)
    return out, lse


def _host(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise TypeError(f"{name} must be a CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def ring_forward_host_workspace_bytes(q, k, v) -> int:
    """Device bytes ``ring_forward_host`` needs for these shapes."""
    s = _shape(q, k, v)
    return int(lib().ra_ring_forward_host_workspace_bytes(ctypes.byref(s)))


def ring_forward_host(q, k, v, P, causal=True, scale=None, out=None, lse=None, workspace=None,
                      stream=None, synchronize=True):
    """``ra_ring_forward_host``: the fused ring on host tensors (pinned memory
    for overlapped copies).  Returns (O, LSE) as host tensors (pinned when
    allocated here); they hold the result once ``stream`` has passed the
    call, which this wrapper waits for unless ``synchronize`` is False."""
    s = _shape(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    if out is None:
        out = torch.empty((s.B, s.Hq, s.n_q, s.d_v), dtype=q.dtype, pin_memory=True)
    if lse is None:
        lse = torch.empty((s.B, s.Hq, s.n_q), dtype=torch.float32, pin_memory=True)
    need = ring_forward_host_workspace_bytes(q, k, v)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    if not workspace.is_cuda:
        raise TypeError("workspace must be a CUDA tensor")
    st = stream if stream is not None else torch.cuda.current_stream()
    rc = lib().ra_ring_forward_host(_host(q, "q"), _host(k, "k", q.dtype), _host(v, "v", q.dtype),
                                    int(P), int(bool(causal)), float(scale),
                                    _host(out, "out", q.dtype), _host(lse, "lse", torch.float32),
                                    ctypes.byref(s), ctypes.c_void_p(workspace.data_ptr()),
                                    ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                    ctypes.c_void_p(st.cuda_stream))
    _check("ra_ring_forward_host", rc)
    if synchronize:
        st.synchronize()
    return out, lse


def backward_workspace_bytes(q, k, v) -> int:
    s = _shape(q, k, v)
    return int(lib().ra_backward_workspace_bytes(ctypes.byref(s)))


def _workspace(q, k, v, workspace):
    need = backward_workspace_bytes(q, k, v)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    return ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(
        workspace.numel() * workspace.element_size())


def backward_delta(out, dout, delta=None, stream=None):
    """D = rowsum(dO * O) per query row: fp32 [B, Hq, n_q]."""
    B, Hq, n, dv = out.shape
    if dout.shape != out.shape:
        raise ValueError("dout must be shaped like out")
    if delta is None:
        delta = torch.empty((B, Hq, n), device=out.device, dtype=torch.float32)
    s = Shape(B, Hq, Hq, n, n, dv, dv, _dtype_code(out.dtype))
    rc = lib().ra_backward_delta(_need(out, "out"), _need(dout, "dout", out.dtype), ctypes.byref(s),
                                 _need(delta, "delta", torch.float32), _stream(stream))
    _check("ra_backward_delta", rc)
    return delta


def _ring_backward(name, q, k, v, out, lse, dout, P, causal, scale, dq, dk, dv, workspace,
                   stream):
    s = _shape(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    wp, wb = _workspace(q, k, v, workspace)
    rc = getattr(lib(), name)(
        _need(q, "q"), _need(k, "k", q.dtype), _need(v, "v", q.dtype), _need(out, "out", q.dtype),
        _need(lse, "lse", torch.float32), _need(dout, "dout", q.dtype), int(P), int(bool(causal)),
        float(scale), _need(dq, "dq", q.dtype), _need(dk, "dk", q.dtype), _need(dv, "dv", q.dtype),
        ctypes.byref(s), wp, wb, _stream(stream))
    _check(name, rc)
    return dq, dk, dv


def ring_backward(q, k, v, out, lse, dout, P, causal=True, scale=None, dq=None, dk=None,
                  dv=None, workspace=None, stream=None):
    """Gradients (dQ, dK, dV) of ring_forward, in the input dtype."""
    return _ring_backward("ra_ring_backward", q, k, v, out, lse, dout, P, causal, scale, dq, dk,
                          dv, workspace, stream)


def ring_backward_striped(q, k, v, out, lse, dout, P, causal=True, scale=None, dq=None, dk=None,
                          dv=None, workspace=None, stream=None):
    """Gradients of ring_forward_striped (striped row order throughout)."""
    return _ring_backward("ra_ring_backward_striped", q, k, v, out, lse, dout, P, causal, scale,
                          dq, dk, dv, workspace, stream)


def block_backward(q, k, v, dout, lse, delta, q_offset=0, k_offset=0, pos_stride=1, causal=True,
                   scale=None, dq_acc=None, dk_acc=None, dv_acc=None, workspace=None,
                   stream=None):
    """Add one block's gradient shares into fp32 accumulators (zeros when not
    given); lse / delta are the query rows' final statistics."""
    s = _shape(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    f32 = torch.float32
    dq_acc = torch.zeros(q.shape, device=q.device, dtype=f32) if dq_acc is None else dq_acc
    dk_acc = torch.zeros(k.shape, device=q.device, dtype=f32) if dk_acc is None else dk_acc
    dv_acc = torch.zeros(v.shape, device=q.device, dtype=f32) if dv_acc is None else dv_acc
    wp, wb = _workspace(q, k, v, workspace)
    rc = lib().ra_block_backward(
        _need(q, "q"), _need(k, "k", q.dtype), _need(v, "v", q.dtype), _need(dout, "dout", q.dtype),
        _need(lse, "lse", f32), _need(delta, "delta", f32), ctypes.byref(s), int(q_offset),
        int(k_offset), int(pos_stride), int(bool(causal)), float(scale),
        _need(dq_acc, "dq_acc", f32), _need(dk_acc, "dk_acc", f32), _need(dv_acc, "dv_acc", f32),
        wp, wb, _stream(stream))
    _check("ra_block_backward", rc)
    return dq_acc, dk_acc, dv_acc


def decode_workspace_bytes(B, Hq, Hkv, n_k, d=128) -> int:
    s = Shape(B, Hq, Hkv, 1, n_k, d, d, RA_BF16)
    return int(lib().ra_decode_workspace_bytes(ctypes.byref(s)))


def decode_partial(q, k, v, token_start=0, token_count=None, scale=None, workspace=None,
                   o_part=None, lse_part=None, stream=None):
    """Pass-Q partial over tokens [token_start, token_start + token_count) of a
    [B, Hkv, S, d] cache (one shard).  Returns (O_p [B,Hq,d], LSE_p [B,Hq])."""
    B, Hq, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query token per sequence")
    _, Hkv, S, dk = k.shape
    token_count = S - token_start if token_count is None else token_count
    if token_start < 0 or token_count <= 0 or token_start + token_count > S:
        raise ValueError("shard outside the cache")
    s = Shape(B, Hq, Hkv, 1, token_count, d, v.shape[-1], _dtype_code(q.dtype))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = int(lib().ra_decode_workspace_bytes(ctypes.byref(s)))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if o_part is None:
        o_part = torch.empty((B, Hq, v.shape[-1]), device=q.device, dtype=torch.float32)
    if lse_part is None:
        lse_part = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    _need(k, "k", q.dtype)
    _need(v, "v", q.dtype)
    esz = k.element_size()
    kp = ctypes.c_void_p(k.data_ptr() + token_start * dk * esz)
    vp = ctypes.c_void_p(v.data_ptr() + token_start * v.shape[-1] * esz)
    rc = lib().ra_decode_partial(_need(q, "q"), kp, vp, ctypes.c_longlong(S), ctypes.byref(s),
                                 float(scale), _need(o_part, "o_part", torch.float32),
                                 _need(lse_part, "lse_part", torch.float32),
                                 ctypes.c_void_p(workspace.data_ptr()),
                                 ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                 _stream(stream))
    _check("ra_decode_partial", rc)
    return o_part, lse_part


def decode_partial_noalloc(q, k, v, token_start=0, token_count=None, scale=None, o_part=None,
                           lse_part=None, stream=None):
    """decode_partial through ra_decode_partial_noalloc: the library keeps the
    chunk partials in its own static device array, so no workspace is passed
    (for callers that cannot allocate device memory).  Pass o_part / lse_part
    to make the call itself allocation-free from Python as well."""
    B, Hq, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query token per sequence")
    _, Hkv, S, dk = k.shape
    token_count = S - token_start if token_count is None else token_count
    if token_start < 0 or token_count <= 0 or token_start + token_count > S:
        raise ValueError("shard outside the cache")
    s = Shape(B, Hq, Hkv, 1, token_count, d, v.shape[-1], _dtype_code(q.dtype))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if o_part is None:
        o_part = torch.empty((B, Hq, v.shape[-1]), device=q.device, dtype=torch.float32)
    if lse_part is None:
        lse_part = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    _need(k, "k", q.dtype)
    _need(v, "v", q.dtype)
    esz = k.element_size()
    kp = ctypes.c_void_p(k.data_ptr() + token_start * dk * esz)
    vp = ctypes.c_void_p(v.data_ptr() + token_start * v.shape[-1] * esz)
    rc = lib().ra_decode_partial_noalloc(_need(q, "q"), kp, vp, ctypes.c_longlong(S),
                                         ctypes.byref(s), float(scale),
                                         _need(o_part, "o_part", torch.float32),
                                         _need(lse_part, "lse_part", torch.float32),
                                         _stream(stream))
    _check("ra_decode_partial_noalloc", rc)
    return o_part, lse_part


def decode_merge(o_parts, lse_parts, out_dtype=torch.bfloat16, out=None, lse=None, stream=None):
    """Reduce P shard partials o_parts [P,B,Hq,d], lse_parts [P,B,Hq]."""
    P, B, H, d = o_parts.shape
    o4 = o_parts.view(P, B, H, 1, d)
    l4 = lse_parts.view(P, B, H, 1)
    out4 = None if out is None else out.view(B, H, 1, d)
    lse4 = None if lse is None else lse.view(B, H, 1)
    o, l = lse_merge(o4, l4, out_dtype, out4, lse4, stream, _name="ra_decode_merge")
    return o.view(B, H, d), l.view(B, H)


def decode_partials(q, k, v, P, scale=None, workspace=None, o_parts=None, lse_parts=None,
                    stream=None):
    """The P shard partials of a [B, Hkv, S, d] cache in one launch (shards of
    S / P tokens, whole 2048-token chunks).  Returns (O_parts [P,B,Hq,d],
    LSE_parts [P,B,Hq])."""
    B, Hq, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query token per sequence")
    _, Hkv, S, _ = k.shape
    s = Shape(B, Hq, Hkv, 1, S, d, v.shape[-1], _dtype_code(q.dtype))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if workspace is None:
        workspace = torch.empty(int(lib().ra_decode_workspace_bytes(ctypes.byref(s))),
                                dtype=torch.uint8, device=q.device)
    if o_parts is None:
        o_parts = torch.empty((P, B, Hq, v.shape[-1]), device=q.device, dtype=torch.float32)
    if lse_parts is None:
        lse_parts = torch.empty((P, B, Hq), device=q.device, dtype=torch.float32)
    _need(k, "k", q.dtype)
    _need(v, "v", q.dtype)
    rc = lib().ra_decode_partials(_need(q, "q"), _need(k, "k"), _need(v, "v"), P, ctypes.byref(s),
                                  float(scale), _need(o_parts, "o_parts", torch.float32),
                                  _need(lse_parts, "lse_parts", torch.float32),
                                  ctypes.c_void_p(workspace.data_ptr()),
                                  ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                  _stream(stream))
    _check("ra_decode_partials", rc)
    return o_parts, lse_parts


def decode_pass_q(q, k, v, P, scale=None, bufs=None):
    """Whole pass-Q decode on one GPU: P shard partials, then the merge.  With
    shards of whole 2048-token chunks the partials come from one launch
    (decode_partials); otherwise one decode_partial call per shard."""
    B, Hq, _, d = q.shape
    S = k.shape[2]
    if S % P:
        raise ValueError("cache length must split into P equal shards")
    L = S // P
    bufs = {} if bufs is None else bufs
    o_parts = bufs.get("o_parts")
    if o_parts is None:
        o_parts = torch.empty((P, B, Hq, d), device=q.device, dtype=torch.float32)
    lse_parts = bufs.get("lse_parts")
    if lse_parts is None:
        lse_parts = torch.empty((P, B, Hq), device=q.device, dtype=torch.float32)
    ws = bufs.get("workspace")
    if P == 1 or L % 2048 == 0:
        if ws is not None and ws.numel() < int(lib().ra_decode_workspace_bytes(
                ctypes.byref(Shape(B, Hq, k.shape[1], 1, S, d, v.shape[-1], _dtype_code(q.dtype))))):
            raise ValueError("workspace smaller than ra_decode_workspace_bytes of the whole cache")
        decode_partials(q, k, v, P, scale, ws, o_parts, lse_parts)
    else:
        for p in range(P):
            decode_partial(q, k, v, p * L, L, scale, ws, o_parts[p], lse_parts[p])
    return decode_merge(o_parts, lse_parts, q.dtype, bufs.get("out"), bufs.get("lse"))


def block_class(n_q, n_k, q_block, k_block, q_offset=0, k_offset=0, causal=True) -> np.ndarray:
    """Host copy of the kernels' tile classification (int8: 0 SKIP, 1 PARTIAL, 2 FULL)."""
    tq, tk = -(-n_q // q_block), -(-n_k // k_block)
    out = np.empty((tq, tk), dtype=np.int8)
    rc = lib().ra_block_class(n_q, n_k, q_block, k_block, q_offset, k_offset, int(bool(causal)),
                              out.ctypes.data_as(ctypes.c_void_p))
    _check("ra_block_class", rc)
    return out


def block_class_device(n_q, n_k, q_block, k_block, q_offset=0, k_offset=0, causal=True,
                       device="cuda", stream=None) -> torch.Tensor:
    tq, tk = -(-n_q // q_block), -(-n_k // k_block)
    out = torch.empty((tq, tk), dtype=torch.int8, device=device)
    rc = lib().ra_block_class_device(n_q, n_k, q_block, k_block, q_offset, k_offset,
                                     int(bool(causal)), ctypes.c_void_p(out.data_ptr()),
                                     _stream(stream))
    _check("ra_block_class_device", rc)
    return out


def get_status(stream=None) -> int:
    return int(lib().ra_get_status(_stream(stream)))


def set_wait_limit_ns(ns: int):
    _check("ra_set_wait_limit_ns", lib().ra_set_wait_limit_ns(int(ns)))


def check_wait_timeout(limit_ns: int, stream=None):
    _check("ra_check_wait_timeout", lib().ra_check_wait_timeout(int(limit_ns), _stream(stream)))


def launch_count() -> int:
    return int(lib().ra_launch_count())
