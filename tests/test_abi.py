"""C ABI checks that need no GPU: the library loads, exports every symbol
include/la.h declares, sizes workspaces, and rejects bad requests before it
touches the device (fail-closed validation)."""

import ctypes
import os
import re

import pytest
import torch

from kernelized_linear_attention_phi_b200 import binding as B
from kernelized_linear_attention_phi_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "la.h")).read()
    return sorted(set(re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("la_kv_summary", "la_noncausal", "la_causal_chunked", "la_prefix_mask",
              "la_decode_step", "la_workspace_size", "la_last_error", "la_status_string",
              "la_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # and nothing else: internal symbols stay hidden
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if l.strip())
    assert exported == declared_functions()


def test_status_strings(lib):
    for code, name in B.STATUS_NAMES.items():
        assert B.la_status_string(code) == name
    assert B.la_version() == 100


def desc(B_=2, H=3, N=100, d=64, dtype=1, phi=0, normalize=1):
    return B.la_desc(B_, H, N, d, dtype, phi, normalize)


def test_workspace_sizes(lib):
    for op in ("kv_summary", "noncausal", "causal", "prefix"):
        for d in (16, 32, 64, 128):
            n = B.la_workspace_size(desc(d=d), op, 64)
            assert n > 0 and n % 256 == 0
    assert B.la_workspace_size(desc(), "decode", 64) == 0
    # the state records dominate: at least one (S, z) record per head
    assert B.la_workspace_size(desc(d=128), "kv_summary") >= 2 * 3 * (128 * 128 + 128) * 4
    # invalid or unsupported requests size to 0
    assert B.la_workspace_size(desc(d=48), "noncausal") == 0
    assert B.la_workspace_size(desc(phi=1, normalize=1), "noncausal") == 0
    assert B.la_workspace_size(desc(N=0), "noncausal") == 0
    assert B.la_workspace_size(desc(), "causal", 96) == 0
    assert B.la_workspace_size(desc(), 7, 64) == 0


P16 = ctypes.c_void_p(1 << 20)          # an aligned, never-dereferenced address
P_MIS = ctypes.c_void_p((1 << 20) + 4)  # misaligned
NULL = None


def call_noncausal(lib, dsc, q=P16, ws_bytes=1 << 30, ws=P16):
    return lib.la_noncausal(ctypes.byref(dsc), q, P16, P16, P16, NULL, NULL, ws, ws_bytes, NULL)


def test_validation_statuses(lib):
    assert lib.la_noncausal(None, P16, P16, P16, P16, NULL, NULL, P16, 1 << 30, NULL) == 1
    assert call_noncausal(lib, desc(d=48)) == 2
    assert call_noncausal(lib, desc(phi=1, normalize=1)) == 2
    assert call_noncausal(lib, desc(N=0)) == 1
    assert call_noncausal(lib, desc(dtype=5)) == 1
    assert call_noncausal(lib, desc(normalize=2)) == 1
    assert call_noncausal(lib, desc(), q=NULL) == 1
    assert call_noncausal(lib, desc(), q=P_MIS) == 3
    assert call_noncausal(lib, desc(), ws_bytes=16) == 4
    assert call_noncausal(lib, desc(), ws=NULL) == 4
    dsc = desc()
    # causal / prefix chunk values
    assert lib.la_causal_chunked(ctypes.byref(dsc), 96, P16, P16, P16, P16, P16, 1 << 30, NULL) == 2
    assert lib.la_prefix_mask(ctypes.byref(dsc), 32, P16, P16, P16, P16, P16, P16, 1 << 30, NULL) == 2
    assert lib.la_prefix_mask(ctypes.byref(dsc), 64, P16, P16, P16, NULL, P16, P16, 1 << 30, NULL) == 1
    assert lib.la_prefix_mask(ctypes.byref(dsc), 64, P16, P16, P16, P_MIS, P16, P16, 1 << 30, NULL) == 3
    # decode: N is ignored, other fields validated
    assert lib.la_decode_step(ctypes.byref(desc(N=0)), P16, P16, P16, P16, P16, P_MIS, NULL) == 3
    assert lib.la_decode_step(ctypes.byref(desc(d=8)), P16, P16, P16, P16, P16, P16, NULL) == 2
    assert lib.la_kv_summary(ctypes.byref(dsc), P16, P16, NULL, P16, P16, 1 << 30, NULL) == 1
    assert lib.la_last_error(NULL, NULL, None) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful on a machine with no GPU")
def test_valid_request_without_gpu_reports_cuda_error(lib):
    """A request that passes validation reaches the device check, which fails
    cleanly with LA_ERR_CUDA when no GPU is present (nothing is launched)."""
    assert call_noncausal(lib, desc()) == 5


def test_timing_read_validation(lib):
    """la_timing_read rejects a NULL count, a negative capacity and a NULL
    buffer with room asked for; with nothing recorded it reports 0 kernels."""
    n = ctypes.c_int32(-1)
    buf = (ctypes.c_float * 4)()
    assert lib.la_timing_read(buf, 4, None) == 1
    assert lib.la_timing_read(buf, -1, ctypes.byref(n)) == 1
    assert lib.la_timing_read(None, 4, ctypes.byref(n)) == 1
    assert lib.la_timing_enable(0) == 0
    assert lib.la_timing_read(None, 0, ctypes.byref(n)) == 0 and n.value == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful on a machine with no GPU")
def test_timing_enable_without_gpu_reports_cuda_error(lib):
    assert lib.la_timing_enable(1) == 5
    assert lib.la_timing_enable(0) == 0


def test_causal_prefill_validation(lib):
    """la_causal_prefill: the causal checks plus non-NULL, aligned S_out and
    z_out (nothing is launched)."""
    dsc = desc()
    NULL = None
    assert lib.la_causal_prefill(ctypes.byref(dsc), 64, P16, P16, P16, P16, NULL, P16, P16, 1 << 30, NULL) == 1
    assert lib.la_causal_prefill(ctypes.byref(dsc), 64, P16, P16, P16, P16, P16, NULL, P16, 1 << 30, NULL) == 1
    assert lib.la_causal_prefill(ctypes.byref(dsc), 64, P16, P16, P16, P16, P_MIS, P16, P16, 1 << 30, NULL) == 3
    assert lib.la_causal_prefill(ctypes.byref(dsc), 96, P16, P16, P16, P16, P16, P16, P16, 1 << 30, NULL) == 2


def test_backward_validation(lib):
    """Gradient entry points: the forward checks plus non-NULL, aligned dout,
    dq, dk, dv; their workspace ops have a size, an unknown op has none."""
    dsc = desc()
    NULL = None
    for fn in (lib.la_noncausal_backward, lib.la_causal_backward):
        assert fn(ctypes.byref(dsc), P16, P16, P16, NULL, P16, P16, P16, P16, 1 << 30, NULL) == 1
        assert fn(ctypes.byref(dsc), P16, P16, P16, P16, P16, P16, NULL, P16, 1 << 30, NULL) == 1
        assert fn(ctypes.byref(dsc), P16, P16, P16, P16, P_MIS, P16, P16, P16, 1 << 30, NULL) == 3
        assert fn(ctypes.byref(desc(d=8)), P16, P16, P16, P16, P16, P16, P16, P16, 1 << 30, NULL) == 2
        assert fn(ctypes.byref(dsc), P16, P16, P16, P16, P16, P16, P16, P16, 16, NULL) == 4
    assert B.la_workspace_size(dsc, "noncausal_bwd") > 0
    assert B.la_workspace_size(dsc, "causal_bwd") > 0
    assert lib.la_workspace_size(ctypes.byref(dsc), 7, 64) == 0


def test_gradient_workspace_sizes(lib):
    """The tensor-core non-causal gradient (bf16, d = 64 / 128) keeps the
    record slots of its balanced splits and the totals (S, z), (G, h), but
    not the CUDA-core path's per-token scaled gradient (fp32 [B,H,N,d]) and
    block states: at a long sequence it needs less than the fp32 request of
    the same shape, whose per-token buffer alone exceeds it."""
    B_, H, N = 1, 2, 65536
    per_token = B_ * H * N * 64 * 4  # fp32 gn of the CUDA-core path
    tc = B.la_workspace_size(B.la_desc(B_, H, N, 64, 1, 0, 1), "noncausal_bwd")
    simt = B.la_workspace_size(B.la_desc(B_, H, N, 64, 0, 0, 1), "noncausal_bwd")
    assert 0 < tc < per_token <= simt
    B_, H, N = 2, 3, 4096
    # both gradients hold at least the totals of both states
    for dt in (0, 1):
        for op in ("noncausal_bwd", "causal_bwd"):
            n = B.la_workspace_size(B.la_desc(B_, H, N, 64, dt, 0, 1), op)
            assert n % 256 == 0 and n >= 2 * B_ * H * (64 * 64 + 64) * 4


def test_static_kv_summary_validates_before_any_cuda_call(lib):
    """la_kv_summary_static checks the descriptor and the pointers first, with
    the statuses la_kv_summary gives, before it looks up its scratch array or
    enqueues anything; a valid request then fails cleanly without a GPU."""
    dsc = desc()
    f = lib.la_kv_summary_static
    assert f(None, P16, P16, P16, P16, NULL) == 1
    assert f(ctypes.byref(desc(d=48)), P16, P16, P16, P16, NULL) == 2
    assert f(ctypes.byref(dsc), P16, P16, NULL, P16, NULL) == 1
    assert f(ctypes.byref(dsc), P16, NULL, P16, P16, NULL) == 1
    assert f(ctypes.byref(dsc), P16, P16, P_MIS, P16, NULL) == 3
    assert f(ctypes.byref(dsc), P16, P16, P16, P_MIS, NULL) == 3
    for bad in (dict(d=48), dict(N=0)):
        d_ = desc(**bad)
        assert f(ctypes.byref(d_), P16, P16, NULL, P16, NULL) == \
            lib.la_kv_summary(ctypes.byref(d_), P16, P16, NULL, P16, P16, 1 << 30, NULL)
    if not torch.cuda.is_available():
        assert f(ctypes.byref(dsc), P16, P16, P16, P16, NULL) == 5


def test_binding_rejects_wrong_state_tensors(lib):
    """The binding refuses S / z buffers of the wrong dtype, shape or
    device before calling the library (which would write B*H*(d*d + d)
    floats through them)."""
    k = torch.zeros(2, 3, 256, 64, dtype=torch.bfloat16)
    ok_S = torch.zeros(2, 3, 64, 64)
    ok_z = torch.zeros(2, 3, 64)
    for S, z in ((ok_S.bfloat16(), ok_z), (ok_S[:, :2], ok_z), (ok_S, ok_z[..., :32]),
                 (ok_S.double(), ok_z)):
        with pytest.raises(ValueError):
            B.la_kv_summary_static(k, k, S, z)
        with pytest.raises(ValueError):
            B.la_kv_summary(k, k, S, z)
        with pytest.raises(ValueError):
            B.la_noncausal(k, k, k, torch.empty_like(k), S, z)
    with pytest.raises(ValueError):
        B.la_noncausal(k, k, k, torch.empty_like(k), ok_S, None)
    with pytest.raises(ValueError):  # a workspace must be uint8 bytes
        B.la_causal_chunked(k, k, k, torch.empty_like(k), ws=torch.zeros(16, dtype=torch.float32))
