"""ctypes binding of libla_b200.so (include/la.h), one Python function per
C entry point, with the same names.

Argument marshalling only: shapes become an ``la_desc``, tensors become their
device pointers, the stream is torch's current CUDA stream unless one is
given. All computation happens in the library's CUDA kernels; if the library
cannot be loaded, every call raises (there is no fallback).

Tensors are contiguous [B, H, N, d] (q, k, v, out; float32 or bfloat16),
S [B, H, d, d] and z [B, H, d] float32, m [B, N] int32. ``phi`` is "relu1"
(relu(x)+1) or "identity".
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libla_b200.so")

LA_OK = 0
STATUS_NAMES = {0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED",
                3: "LA_ERR_MISALIGNED", 4: "LA_ERR_WORKSPACE", 5: "LA_ERR_CUDA",
                6: "LA_ERR_MASK_RANGE", 7: "LA_ERR_TIMEOUT"}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
PHIS = {"relu1": 0, "identity": 1, "elu1": 2}
OPS = {"kv_summary": 0, "noncausal": 1, "causal": 2, "prefix": 3, "decode": 4, "noncausal_bwd": 5,
       "causal_bwd": 6}


class LaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


class la_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32), ("phi", ctypes.c_int32),
                ("normalize", ctypes.c_int32)]


_lib = None

_P = ctypes.c_void_p
_SIGS = {
    "la_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(la_desc), ctypes.c_int32, ctypes.c_int32]),
    "la_kv_summary": (ctypes.c_int, [ctypes.POINTER(la_desc), _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "la_noncausal": (ctypes.c_int, [ctypes.POINTER(la_desc), _P, _P, _P, _P, _P, _P, _P,
                                    ctypes.c_size_t, _P]),
    "la_causal_chunked": (ctypes.c_int, [ctypes.POINTER(la_desc), ctypes.c_int32, _P, _P, _P, _P,
                                         _P, ctypes.c_size_t, _P]),
    "la_causal_prefill": (ctypes.c_int, [ctypes.POINTER(la_desc), ctypes.c_int32, _P, _P, _P, _P, _P, _P,
                                         _P, ctypes.c_size_t, _P]),
    "la_noncausal_backward": (ctypes.c_int, [ctypes.POINTER(la_desc), _P, _P, _P, _P, _P, _P, _P, _P,
                                             ctypes.c_size_t, _P]),
    "la_causal_backward": (ctypes.c_int, [ctypes.POINTER(la_desc), _P, _P, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_size_t, _P]),
    "la_prefix_mask": (ctypes.c_int, [ctypes.POINTER(la_desc), ctypes.c_int32, _P, _P, _P, _P, _P,
                                      _P, ctypes.c_size_t, _P]),
    "la_decode_step": (ctypes.c_int, [ctypes.POINTER(la_desc), _P, _P, _P, _P, _P, _P, _P]),
    "la_kv_summary_static": (ctypes.c_int, [ctypes.POINTER(la_desc), _P, _P, _P, _P, _P]),
    "la_last_error": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "la_timing_enable": (ctypes.c_int, [ctypes.c_int32]),
    "la_timing_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float), ctypes.c_int32,
                                      ctypes.POINTER(ctypes.c_int32)]),
    "la_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "la_version": (ctypes.c_int32, []),
}


def lib():
    """The loaded library (raises if it is missing: build it first with
    ``python -m kernelized_linear_attention_phi_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libla_b200.so is not built ({LIB_PATH})")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def make_desc(B, H, N, d, dtype, phi="relu1", normalize=True) -> la_desc:
    return la_desc(int(B), int(H), int(N), int(d), DTYPES.get(dtype, dtype) if not isinstance(dtype, int) else dtype,
                   PHIS[phi] if isinstance(phi, str) else int(phi), int(bool(normalize)))


def _desc_of(x: torch.Tensor, phi, normalize) -> la_desc:
    if x.dim() != 4:
        raise ValueError(f"expected a [B, H, N, d] tensor, got shape {tuple(x.shape)}")
    if x.dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {x.dtype}")
    B, H, N, d = x.shape
    return make_desc(B, H, N, d, x.dtype, phi, normalize)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(t, stream):
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn, status):
    if status != LA_OK:
        raise LaError(fn, status)


def _same(ref, *ts):
    for t in ts:
        if t.dtype != ref.dtype or t.shape != ref.shape or t.device != ref.device:
            raise ValueError("q, k, v and out must share shape, dtype and device")


def _state(S, z, ref):
    """S [B,H,d,d] and z [B,H,d]: contiguous float32 on ref's device (the
    library writes or reads exactly that many floats)."""
    B, H, _, d = ref.shape
    if S.dtype != torch.float32 or tuple(S.shape) != (B, H, d, d) or S.device != ref.device:
        raise ValueError(f"S must be float32 [{B}, {H}, {d}, {d}] on {ref.device}")
    if z.dtype != torch.float32 or tuple(z.shape) != (B, H, d) or z.device != ref.device:
        raise ValueError(f"z must be float32 [{B}, {H}, {d}] on {ref.device}")
    if not S.is_contiguous() or not z.is_contiguous():
        raise ValueError("S and z must be contiguous")


def _ws(ws, ref):
    """A workspace: a contiguous uint8 buffer on ref's device (the library
    checks its size)."""
    if ws.dtype != torch.uint8 or ws.device != ref.device or not ws.is_contiguous():
        raise ValueError(f"the workspace must be a contiguous uint8 tensor on {ref.device}")
    return ws


def la_version() -> int:
    return int(lib().la_version())


def la_status_string(status: int) -> str:
    return lib().la_status_string(int(status)).decode()


def la_workspace_size(desc: la_desc, op, chunk: int = 64) -> int:
    return int(lib().la_workspace_size(ctypes.byref(desc), OPS.get(op, op), int(chunk)))


def workspace(desc: la_desc, op, chunk: int = 64, device="cuda") -> torch.Tensor:
    """A device buffer big enough for ``op`` on ``desc``, with its error word
    zeroed (the library only sets bits in it; la_last_error reads and
    clears)."""
    n = la_workspace_size(desc, op, chunk)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def la_kv_summary(k, v, S_out=None, z_out=None, phi="relu1", ws=None, stream=None):
    """S = sum_j phi(k_j) (x) v_j, z = sum_j phi(k_j) per head. Returns (S, z)."""
    _same(k, v)
    desc = _desc_of(k, phi, True)
    B, H, _, d = k.shape
    if S_out is None:
        S_out = torch.empty(B, H, d, d, dtype=torch.float32, device=k.device)
    if z_out is None:
        z_out = torch.empty(B, H, d, dtype=torch.float32, device=k.device)
    _state(S_out, z_out, k)
    ws = workspace(desc, "kv_summary", device=k.device) if ws is None else _ws(ws, k)
    _check("la_kv_summary", lib().la_kv_summary(
        ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(S_out), _ptr(z_out), _ptr(ws), ws.numel(),
        _stream(k, stream)))
    return S_out, z_out


def la_kv_summary_static(k, v, S_out, z_out, phi="relu1", stream=None):
    """la_kv_summary with the library's own device scratch instead of a
    workspace: for callers that cannot allocate device memory. Allocates
    nothing; S_out [B,H,d,d] and z_out [B,H,d] float32 are the caller's.
    Calls that overlap on the GPU race (they share the scratch)."""
    _same(k, v)
    _state(S_out, z_out, k)
    desc = _desc_of(k, phi, True)
    _check("la_kv_summary_static", lib().la_kv_summary_static(
        ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(S_out), _ptr(z_out), _stream(k, stream)))
    return S_out, z_out


def la_noncausal(q, k, v, out=None, S_out=None, z_out=None, phi="relu1", normalize=True, ws=None,
                 stream=None):
    """Non-causal attention. Returns out (and fills S_out/z_out if given)."""
    if out is None:
        out = torch.empty_like(q)
    _same(q, k, v, out)
    if (S_out is None) != (z_out is None):
        raise ValueError("give both S_out and z_out, or neither")
    if S_out is not None:
        _state(S_out, z_out, q)
    desc = _desc_of(q, phi, normalize)
    ws = workspace(desc, "noncausal", device=q.device) if ws is None else _ws(ws, q)
    _check("la_noncausal", lib().la_noncausal(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(S_out), _ptr(z_out),
        _ptr(ws), ws.numel(), _stream(q, stream)))
    return out


def la_causal_chunked(q, k, v, out=None, chunk=64, phi="relu1", normalize=True, ws=None,
                      stream=None):
    """Causal attention (query i sees keys 0..i). Returns out."""
    if out is None:
        out = torch.empty_like(q)
    _same(q, k, v, out)
    desc = _desc_of(q, phi, normalize)
    ws = workspace(desc, "causal", chunk, device=q.device) if ws is None else _ws(ws, q)
    _check("la_causal_chunked", lib().la_causal_chunked(
        ctypes.byref(desc), int(chunk), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(ws),
        ws.numel(), _stream(q, stream)))
    return out


def la_causal_prefill(q, k, v, out=None, S_out=None, z_out=None, chunk=64, phi="relu1", normalize=True,
                      ws=None, stream=None):
    """Causal attention plus the state after the last token (the cache a
    decode continues from). Returns (out, S, z)."""
    if out is None:
        out = torch.empty_like(q)
    _same(q, k, v, out)
    B, H, _, d = q.shape
    if S_out is None:
        S_out = torch.empty(B, H, d, d, dtype=torch.float32, device=q.device)
    if z_out is None:
        z_out = torch.empty(B, H, d, dtype=torch.float32, device=q.device)
    _state(S_out, z_out, q)
    desc = _desc_of(q, phi, normalize)
    ws = workspace(desc, "causal", chunk, device=q.device) if ws is None else _ws(ws, q)
    _check("la_causal_prefill", lib().la_causal_prefill(
        ctypes.byref(desc), int(chunk), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(S_out), _ptr(z_out),
        _ptr(ws), ws.numel(), _stream(q, stream)))
    return out, S_out, z_out


def la_prefix_mask(q, k, v, m, out=None, chunk=64, phi="relu1", normalize=True, ws=None,
                   stream=None):
    """Prefix-mask attention (query i of sequence b sees keys 0..m[b, i]). Returns out."""
    if out is None:
        out = torch.empty_like(q)
    _same(q, k, v, out)
    B, _, N, _ = q.shape
    if m.dtype != torch.int32 or tuple(m.shape) != (B, N) or m.device != q.device:
        raise ValueError("m must be an int32 [B, N] tensor on the same device")
    if not m.is_contiguous():
        raise ValueError("m must be contiguous")
    desc = _desc_of(q, phi, normalize)
    ws = workspace(desc, "prefix", chunk, device=q.device) if ws is None else _ws(ws, q)
    _check("la_prefix_mask", lib().la_prefix_mask(
        ctypes.byref(desc), int(chunk), _ptr(q), _ptr(k), _ptr(v), _ptr(m), _ptr(out), _ptr(ws),
        ws.numel(), _stream(q, stream)))
    return out


def la_decode_step(q, k, v, S, z, out=None, phi="relu1", normalize=True, stream=None):
    """One decode step on the state (S, z), updated in place. q, k, v: [B, H, 1, d]."""
    if out is None:
        out = torch.empty_like(q)
    _same(q, k, v, out)
    _state(S, z, q)
    desc = _desc_of(q, phi, normalize)
    _check("la_decode_step", lib().la_decode_step(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(z), _ptr(out),
        _stream(q, stream)))
    return out


def la_last_error(ws, stream=None):
    """Synchronizes, reads and clears the workspace error word. Returns
    (status, flags)."""
    flags = ctypes.c_uint32(0)
    st = lib().la_last_error(_ptr(ws), _stream(ws, stream), ctypes.byref(flags))
    return int(st), int(flags.value)


def la_timing_enable(enable=True):
    """Turns the library's per-kernel timing events on or off (on: creates
    them on the current device)."""
    _check("la_timing_enable", lib().la_timing_enable(1 if enable else 0))


def la_timing_read(capacity=16):
    """Durations in ms of the kernels of the last timed call (or graph
    replay), in launch order; waits for that call to finish."""
    buf = (ctypes.c_float * capacity)()
    n = ctypes.c_int32(0)
    _check("la_timing_read", lib().la_timing_read(buf, capacity, ctypes.byref(n)))
    return [float(buf[i]) for i in range(min(n.value, capacity))]


def _backward(name, op, q, k, v, dout, dq, dk, dv, phi, normalize, ws, stream):
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _same(q, k, v, dout, dq, dk, dv)
    desc = _desc_of(q, phi, normalize)
    ws = workspace(desc, op, 64, device=q.device) if ws is None else _ws(ws, q)
    _check(name, getattr(lib(), name)(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
        ws.numel(), _stream(q, stream)))
    return dq, dk, dv


def la_noncausal_backward(q, k, v, dout, dq=None, dk=None, dv=None, phi="relu1", normalize=True, ws=None,
                          stream=None):
    """Gradients (dq, dk, dv) of non-causal attention for upstream dout."""
    return _backward("la_noncausal_backward", "noncausal_bwd", q, k, v, dout, dq, dk, dv, phi, normalize, ws,
                     stream)


def la_causal_backward(q, k, v, dout, dq=None, dk=None, dv=None, phi="relu1", normalize=True, ws=None,
                       stream=None):
    """Gradients (dq, dk, dv) of causal attention for upstream dout."""
    return _backward("la_causal_backward", "causal_bwd", q, k, v, dout, dq, dk, dv, phi, normalize, ws, stream)
