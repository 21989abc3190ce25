"""chunkwise_recurrence_b200 -- Python binding of libgdr.

libgdr computes the chunkwise-parallel forward pass of the gated delta rule
(DeltaNet, Gated DeltaNet and KDA) on one B200.  This module only marshals
arguments into the C ABI declared in ``include/gdr.h``; every step of the
computation runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams.  There is no CPU fallback: if ``libgdr.so`` is missing the
calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["chunk_fwd", "chunk_fwd_host", "chunk_fwd_noalloc",
           "chunk_fwd_segmented", "chunk_fwd_gdn2", "chunk_fwd_fg2",
           "decode_step", "decode_step_gdn2", "decode_step_fg2",
           "efla_beta", "efla_beta_backward", "backward", "backward_gdn2",
           "backward_fg2",
           "device_error", "status_string",
           "algo_applies", "fused_tc_available",
           "GdrError", "load_library", "LIB_PATH", "GATES", "ALGOS",
           "EXPORTED_SYMBOLS"]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdr.so")

GATES = {"none": 0, "scalar": 1, "channel": 2}
ALGOS = {"auto": 0, "staged": 1, "fused_tc": 2, "recurrent": 3}
DTYPES = {torch.bfloat16: 0, torch.float32: 1}
STATUS = {0: "GDR_OK", 1: "GDR_ERR_INVALID_ARGUMENT", 2: "GDR_ERR_UNSUPPORTED",
          3: "GDR_ERR_CUDA", 4: "GDR_ERR_OUT_OF_MEMORY", 5: "GDR_ERR_TIMEOUT",
          6: "GDR_ERR_RANGE"}
EXPORTED_SYMBOLS = ("gdr_chunk_fwd", "gdr_chunk_fwd_host", "gdr_device_error",
                    "gdr_algo_applies", "gdr_status_string",
                    "gdr_chunk_fwd_noalloc", "gdr_decode_step",
                    "gdr_efla_beta", "gdr_backward",
                    "gdr_chunk_fwd_segmented", "gdr_chunk_fwd_gdn2",
                    "gdr_decode_step_gdn2", "gdr_chunk_fwd_fg2",
                    "gdr_decode_step_fg2", "gdr_backward_gdn2",
                    "gdr_backward_fg2", "gdr_efla_beta_backward")
# size of the static scratch array behind gdr_chunk_fwd_noalloc
NOALLOC_SCRATCH_BYTES = 64 << 20

_lib = None


class GdrError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class _Opts(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("gate", ctypes.c_int),
                ("cu_seqlens", ctypes.c_void_p), ("num_seqs", ctypes.c_int),
                ("algo", ctypes.c_int)]


def load_library(path: str = LIB_PATH):
    """Load libgdr (raises if it has not been built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with "
            "`python -m chunkwise_recurrence_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(path)
    vp, fp, i = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
    for name in ("gdr_chunk_fwd", "gdr_chunk_fwd_host",
                 "gdr_chunk_fwd_noalloc"):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i, i, i, i, i, i, vp,
                      ctypes.POINTER(_Opts)]
    lib.gdr_decode_step.restype = ctypes.c_int
    lib.gdr_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, i, i, i, i,
                                    vp, ctypes.POINTER(_Opts)]
    for name in ("gdr_decode_step_gdn2", "gdr_decode_step_fg2"):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, i, i, i, i, vp,
                      ctypes.POINTER(_Opts)]
    for name in ("gdr_chunk_fwd_gdn2", "gdr_chunk_fwd_fg2"):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, i, i, i, i, i, i, vp,
                      ctypes.POINTER(_Opts)]
    lib.gdr_chunk_fwd_segmented.restype = ctypes.c_int
    lib.gdr_chunk_fwd_segmented.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i,
                                            i, i, i, i, i, i, vp,
                                            ctypes.POINTER(_Opts)]
    lib.gdr_backward.restype = ctypes.c_int
    lib.gdr_backward.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, fp, fp, fp,
                                 fp, fp, fp, i, i, i, i, i, vp,
                                 ctypes.POINTER(_Opts)]
    for name in ("gdr_backward_gdn2", "gdr_backward_fg2"):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, fp, fp, fp, fp, fp,
                      fp, fp, i, i, i, i, i, vp, ctypes.POINTER(_Opts)]
    lib.gdr_efla_beta.restype = ctypes.c_int
    lib.gdr_efla_beta.argtypes = [vp, fp, fp, i, i, i, i, vp]
    lib.gdr_efla_beta_backward.restype = ctypes.c_int
    lib.gdr_efla_beta_backward.argtypes = [vp, fp, fp, fp, fp, i, i, i, i, vp]
    lib.gdr_device_error.restype = ctypes.c_int
    lib.gdr_device_error.argtypes = [vp, i]
    lib.gdr_algo_applies.restype = ctypes.c_int
    lib.gdr_algo_applies.argtypes = [i, i, i, i, i, i]
    lib.gdr_status_string.restype = ctypes.c_char_p
    lib.gdr_status_string.argtypes = [i]
    if path == LIB_PATH:
        _lib = lib
    return lib


def algo_applies(algo: str, dtype: str, gate: str, dk: int, dv: int,
                 chunk: int) -> bool:
    """Whether `algo` can run this dtype ("bf16"/"fp32"), gate and shape."""
    dt = {"bf16": 0, "fp32": 1}[dtype]
    return bool(load_library().gdr_algo_applies(ALGOS[algo], dt, GATES[gate],
                                                dk, dv, chunk))


def fused_tc_available() -> bool:
    """Whether the fused tensor-core kernel serves the headline shape."""
    return algo_applies("fused_tc", "bf16", "scalar", 128, 128, 64)


def status_string(code: int) -> str:
    return load_library().gdr_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shapes(q, v, cu_seqlens):
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, T, H, d]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    nseq = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    return B, T, H, dk, dv, nseq


def _gate_of(log_alpha, gate):
    if gate is not None:
        return gate
    if log_alpha is None:
        return "none"
    return "scalar" if log_alpha.dim() == 3 else "channel"


def chunk_fwd(q, k, v, beta, log_alpha=None, initial_state=None, *,
              chunk: int = 64, gate: str | None = None, cu_seqlens=None,
              out=None, final_state=None, output_final_state: bool = True,
              algo: str = "auto", stream=None):
    """Run ``gdr_chunk_fwd`` on CUDA tensors (layouts as in include/gdr.h).

    Returns (out, final_state); final_state is None if not requested.
    """
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    if out is None:
        out = torch.empty_like(v)
    if final_state is None and output_final_state:
        final_state = torch.empty(nseq, H, dk, dv, dtype=torch.float32,
                                  device=q.device)
    g = _gate_of(log_alpha, gate)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = lib.gdr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                           _ptr(beta), _ptr(initial_state), _ptr(out),
                           _ptr(final_state), B, T, H, dk, dv, chunk,
                           ctypes.c_void_p(stream.cuda_stream),
                           ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd")
    return out, final_state


def chunk_fwd_gdn2(q, k, v, erase_gate, write_gate, log_alpha=None,
                   initial_state=None, *, chunk: int = 64,
                   gate: str | None = None, cu_seqlens=None, out=None,
                   final_state=None, output_final_state: bool = True,
                   algo: str = "auto", stream=None):
    """Run ``gdr_chunk_fwd_gdn2``: the forward pass with Gated DeltaNet-2's
    per-key-channel erase gate (``erase_gate``, the layout of k, fp32) and
    per-value-channel write gate (``write_gate``, the layout of v, fp32) in
    place of beta (see include/gdr.h for the update).  Returns (out,
    final_state)."""
    return _chunk_fwd_two_gates(
        "gdr_chunk_fwd_gdn2", q, k, v, erase_gate, write_gate, log_alpha,
        initial_state, chunk, gate, cu_seqlens, out, final_state,
        output_final_state, algo, stream)


def chunk_fwd_fg2(q, k, v, beta_k, beta_v=None, log_alpha=None,
                  initial_state=None, *, chunk: int = 64,
                  gate: str | None = None, cu_seqlens=None, out=None,
                  final_state=None, output_final_state: bool = True,
                  algo: str = "auto", stream=None):
    """Run ``gdr_chunk_fwd_fg2``: the forward pass with FG^2-GDN's
    per-key-channel learning rate ``beta_k`` (the layout of k, fp32) and,
    for FG^2-GDN+, the per-value-channel target scaling ``beta_v`` (the
    layout of v, fp32; None for FG^2-GDN) in place of beta (see
    include/gdr.h for the update).  Returns (out, final_state)."""
    return _chunk_fwd_two_gates(
        "gdr_chunk_fwd_fg2", q, k, v, beta_k, beta_v, log_alpha,
        initial_state, chunk, gate, cu_seqlens, out, final_state,
        output_final_state, algo, stream)


def _chunk_fwd_two_gates(name, q, k, v, gate_k, gate_v, log_alpha,
                         initial_state, chunk, gate, cu_seqlens, out,
                         final_state, output_final_state, algo, stream):
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    if out is None:
        out = torch.empty_like(v)
    if final_state is None and output_final_state:
        final_state = torch.empty(nseq, H, dk, dv, dtype=torch.float32,
                                  device=q.device)
    g = _gate_of(log_alpha, gate)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = getattr(lib, name)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(gate_k),
        _ptr(gate_v), _ptr(initial_state), _ptr(out), _ptr(final_state),
        B, T, H, dk, dv, chunk, ctypes.c_void_p(stream.cuda_stream),
        ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, name)
    return out, final_state


def chunk_fwd_segmented(q, k, v, beta, log_alpha=None, initial_state=None, *,
                        segments: int, chunk: int = 64,
                        gate: str | None = None, cu_seqlens=None, out=None,
                        final_state=None, output_final_state: bool = True,
                        algo: str = "auto", stream=None):
    """Run ``gdr_chunk_fwd_segmented``: the forward pass with every sequence
    cut into up to ``segments`` pieces whose state maps are computed in
    parallel (context-parallel state passing).  Same inputs and results as
    ``chunk_fwd``."""
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    if out is None:
        out = torch.empty_like(v)
    if final_state is None and output_final_state:
        final_state = torch.empty(nseq, H, dk, dv, dtype=torch.float32,
                                  device=q.device)
    g = _gate_of(log_alpha, gate)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = lib.gdr_chunk_fwd_segmented(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
        _ptr(initial_state), _ptr(out), _ptr(final_state), B, T, H, dk, dv,
        chunk, int(segments), ctypes.c_void_p(stream.cuda_stream),
        ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd_segmented")
    return out, final_state


def chunk_fwd_noalloc(q, k, v, beta, log_alpha=None, initial_state=None, *,
                      out, final_state=None, chunk: int = 64,
                      gate: str | None = None, cu_seqlens=None,
                      algo: str = "auto", stream=None):
    """Run ``gdr_chunk_fwd_noalloc``: like ``chunk_fwd`` but the library
    allocates nothing (its scratch is a static device array shared by every
    call on a device, so calls must not overlap on the GPU).  The caller
    passes preallocated ``out`` (and ``final_state`` if wanted)."""
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    g = _gate_of(log_alpha, gate)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    # the library finds its scratch array through the current device, which
    # must be the device of the stream and the tensors
    with torch.cuda.device(q.device):
        rc = lib.gdr_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v),
                                       _ptr(log_alpha), _ptr(beta),
                                       _ptr(initial_state), _ptr(out),
                                       _ptr(final_state), B, T, H, dk, dv,
                                       chunk,
                                       ctypes.c_void_p(stream.cuda_stream),
                                       ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd_noalloc")
    return out, final_state


def chunk_fwd_host(q, k, v, beta, log_alpha=None, initial_state=None, *,
                   out, final_state=None, chunk: int = 64,
                   gate: str | None = None, cu_seqlens=None,
                   algo: str = "auto", stream=None):
    """Run ``gdr_chunk_fwd_host`` on CPU tensors (pinned for async copies).
    Outputs land in ``out`` / ``final_state`` once ``stream`` is synchronised."""
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    g = _gate_of(log_alpha, gate)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream()
    rc = lib.gdr_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                _ptr(beta), _ptr(initial_state), _ptr(out),
                                _ptr(final_state), B, T, H, dk, dv, chunk,
                                ctypes.c_void_p(stream.cuda_stream),
                                ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_chunk_fwd_host")
    return out, final_state


def decode_step(q, k, v, beta, log_alpha=None, state=None, *, out=None,
                state_out=None, gate: str | None = None, stream=None):
    """Run ``gdr_decode_step`` on CUDA tensors: one token per (sequence, head).

    q, k [N, H, dk]; v [N, H, dv]; beta [N, H]; log_alpha [N, H] (scalar
    gate), [N, H, dk] (channel gate) or None; state [N, H, dk, dv] fp32 or
    None (zero).  ``state_out`` defaults to ``state`` itself (an in-place
    update) when a state is given, else a new tensor.  Returns
    (out [N, H, dv], state_out).
    """
    lib = load_library()
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k, v must be [N, H, d]")
    N, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty_like(v)
    if state_out is None:
        state_out = state if state is not None else torch.empty(
            N, H, dk, dv, dtype=torch.float32, device=q.device)
    g = gate if gate is not None else (
        "none" if log_alpha is None else
        "scalar" if log_alpha.dim() == 2 else "channel")
    opts = _Opts(DTYPES[q.dtype], GATES[g], None, 0, ALGOS["auto"])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = lib.gdr_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                             _ptr(beta), _ptr(state), _ptr(state_out),
                             _ptr(out), N, H, dk, dv,
                             ctypes.c_void_p(stream.cuda_stream),
                             ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_decode_step")
    return out, state_out


def decode_step_gdn2(q, k, v, erase_gate, write_gate, log_alpha=None,
                     state=None, *, out=None, state_out=None,
                     gate: str | None = None, stream=None):
    """Run ``gdr_decode_step_gdn2`` on CUDA tensors: one token per (sequence,
    head) with Gated DeltaNet-2's gates in place of beta.  ``erase_gate``
    [N, H, dk] and ``write_gate`` [N, H, dv] are fp32; everything else is as
    in ``decode_step``.  Returns (out [N, H, dv], state_out)."""
    return _decode_two_gates("gdr_decode_step_gdn2", q, k, v, erase_gate,
                             write_gate, log_alpha, state, out, state_out,
                             gate, stream)


def decode_step_fg2(q, k, v, beta_k, beta_v=None, log_alpha=None,
                    state=None, *, out=None, state_out=None,
                    gate: str | None = None, stream=None):
    """Run ``gdr_decode_step_fg2`` on CUDA tensors: one token per (sequence,
    head) with FG^2-GDN's per-key-channel rate ``beta_k`` [N, H, dk] and
    optional value-side scaling ``beta_v`` [N, H, dv] (fp32) in place of
    beta; everything else is as in ``decode_step``.  Returns (out [N, H,
    dv], state_out)."""
    return _decode_two_gates("gdr_decode_step_fg2", q, k, v, beta_k, beta_v,
                             log_alpha, state, out, state_out, gate, stream)


def _decode_two_gates(name, q, k, v, gate_k, gate_v, log_alpha, state, out,
                      state_out, gate, stream):
    lib = load_library()
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k, v must be [N, H, d]")
    N, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty_like(v)
    if state_out is None:
        state_out = state if state is not None else torch.empty(
            N, H, dk, dv, dtype=torch.float32, device=q.device)
    g = gate if gate is not None else (
        "none" if log_alpha is None else
        "scalar" if log_alpha.dim() == 2 else "channel")
    opts = _Opts(DTYPES[q.dtype], GATES[g], None, 0, ALGOS["auto"])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = getattr(lib, name)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                            _ptr(gate_k), _ptr(gate_v), _ptr(state),
                            _ptr(state_out), _ptr(out), N, H, dk, dv,
                            ctypes.c_void_p(stream.cuda_stream),
                            ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, name)
    return out, state_out


def backward(q, k, v, beta, log_alpha, initial_state, d_out, d_final_state=None,
             *, gate: str | None = None, cu_seqlens=None,
             need_initial_state_grad: bool = True, algo: str = "auto",
             stream=None):
    """Run ``gdr_backward``: gradients of the forward pass (same inputs as
    ``chunk_fwd``) given dL/d out and, optionally, dL/d final_state.
    ``algo``: "auto" / "staged" (the chunked backward) or "recurrent" (the
    reverse token recurrence).  Returns a dict of fp32 CUDA tensors dq, dk,
    dv, dbeta, dlog_alpha (None without a gate) and dinitial_state (None
    unless requested)."""
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    g = _gate_of(log_alpha, gate)
    f32 = lambda t: torch.empty(t.shape, dtype=torch.float32,  # noqa: E731
                                device=q.device)
    gq, gk, gv, gb = f32(q), f32(k), f32(v), f32(beta)
    gla = None if log_alpha is None else f32(log_alpha)
    gs0 = (torch.empty(nseq, H, dk, dv, dtype=torch.float32, device=q.device)
           if need_initial_state_grad else None)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = lib.gdr_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                          _ptr(beta), _ptr(initial_state), _ptr(d_out),
                          _ptr(d_final_state), _ptr(gq), _ptr(gk), _ptr(gv),
                          _ptr(gla), _ptr(gb), _ptr(gs0), B, T, H, dk, dv,
                          ctypes.c_void_p(stream.cuda_stream),
                          ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_backward")
    return dict(dq=gq, dk=gk, dv=gv, dbeta=gb, dlog_alpha=gla,
                dinitial_state=gs0)


def backward_gdn2(q, k, v, erase_gate, write_gate, log_alpha, initial_state,
                  d_out, d_final_state=None, *, gate: str | None = None,
                  cu_seqlens=None, need_initial_state_grad: bool = True,
                  algo: str = "auto", stream=None):
    """Run ``gdr_backward_gdn2``: gradients of ``chunk_fwd_gdn2``'s outputs
    (same inputs) given dL/d out and, optionally, dL/d final_state.  Returns
    a dict of fp32 CUDA tensors dq, dk, dv, derase, dwrite, dlog_alpha
    (None without a gate) and dinitial_state (None unless requested)."""
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    g = _gate_of(log_alpha, gate)
    f32 = lambda t: torch.empty(t.shape, dtype=torch.float32,  # noqa: E731
                                device=q.device)
    gq, gk, gv = f32(q), f32(k), f32(v)
    ge, gw = f32(erase_gate), f32(write_gate)
    gla = None if log_alpha is None else f32(log_alpha)
    gs0 = (torch.empty(nseq, H, dk, dv, dtype=torch.float32, device=q.device)
           if need_initial_state_grad else None)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = lib.gdr_backward_gdn2(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(erase_gate),
        _ptr(write_gate), _ptr(initial_state), _ptr(d_out),
        _ptr(d_final_state), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gla),
        _ptr(ge), _ptr(gw), _ptr(gs0), B, T, H, dk, dv,
        ctypes.c_void_p(stream.cuda_stream), ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_backward_gdn2")
    return dict(dq=gq, dk=gk, dv=gv, derase=ge, dwrite=gw, dlog_alpha=gla,
                dinitial_state=gs0)


def backward_fg2(q, k, v, beta_k, beta_v, log_alpha, initial_state, d_out,
                 d_final_state=None, *, gate: str | None = None,
                 cu_seqlens=None, need_initial_state_grad: bool = True,
                 algo: str = "auto", stream=None):
    """Run ``gdr_backward_fg2``: gradients of ``chunk_fwd_fg2``'s outputs
    (same inputs; ``beta_v`` None for FG^2-GDN) given dL/d out and,
    optionally, dL/d final_state.  Returns a dict of fp32 CUDA tensors dq,
    dk, dv, dbeta_k, dbeta_v (None without beta_v), dlog_alpha (None without
    a gate) and dinitial_state (None unless requested)."""
    lib = load_library()
    B, T, H, dk, dv, nseq = _shapes(q, v, cu_seqlens)
    g = _gate_of(log_alpha, gate)
    f32 = lambda t: torch.empty(t.shape, dtype=torch.float32,  # noqa: E731
                                device=q.device)
    gq, gk, gv, gbk = f32(q), f32(k), f32(v), f32(beta_k)
    gbv = None if beta_v is None else f32(beta_v)
    gla = None if log_alpha is None else f32(log_alpha)
    gs0 = (torch.empty(nseq, H, dk, dv, dtype=torch.float32, device=q.device)
           if need_initial_state_grad else None)
    opts = _Opts(DTYPES[q.dtype], GATES[g],
                 None if cu_seqlens is None else cu_seqlens.data_ptr(),
                 nseq if cu_seqlens is not None else 0, ALGOS[algo])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = lib.gdr_backward_fg2(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta_k),
        _ptr(beta_v), _ptr(initial_state), _ptr(d_out), _ptr(d_final_state),
        _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gla), _ptr(gbk), _ptr(gbv),
        _ptr(gs0), B, T, H, dk, dv, ctypes.c_void_p(stream.cuda_stream),
        ctypes.byref(opts))
    if rc != 0:
        raise GdrError(rc, "gdr_backward_fg2")
    return dict(dq=gq, dk=gk, dv=gv, dbeta_k=gbk, dbeta_v=gbv,
                dlog_alpha=gla, dinitial_state=gs0)


def efla_beta(k, beta, *, out=None, stream=None):
    """Run ``gdr_efla_beta``: the exact-flow step size
    beta' = (1 - exp(-beta |k|^2)) / |k|^2 for keys k [..., H, dk] and beta
    [..., H] (CUDA tensors; ``out`` may be ``beta`` for an in-place update).
    Passing beta' to ``chunk_fwd`` or ``decode_step`` runs the EFLA
    recurrence."""
    lib = load_library()
    dk = k.shape[-1]
    H = k.shape[-2]
    ntok = k.numel() // (H * dk)
    if out is None:
        out = torch.empty_like(beta)
    if stream is None:
        stream = torch.cuda.current_stream(k.device)
    rc = lib.gdr_efla_beta(_ptr(k), _ptr(beta), _ptr(out), ntok, H, dk,
                           DTYPES[k.dtype], ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise GdrError(rc, "gdr_efla_beta")
    return out


def efla_beta_backward(k, beta, d_beta_prime, dk, *, d_beta=None,
                       stream=None):
    """Run ``gdr_efla_beta_backward``: the chain rule through ``efla_beta``.
    Returns d beta [..., H] (fp32) and adds d beta' (d beta' / d |k|^2) 2 k
    into ``dk`` (fp32, the layout of k, e.g. ``backward``'s dk)."""
    lib = load_library()
    dkd = k.shape[-1]
    H = k.shape[-2]
    ntok = k.numel() // (H * dkd)
    if d_beta is None:
        d_beta = torch.empty_like(beta)
    if stream is None:
        stream = torch.cuda.current_stream(k.device)
    rc = lib.gdr_efla_beta_backward(_ptr(k), _ptr(beta), _ptr(d_beta_prime),
                                    _ptr(d_beta), _ptr(dk), ntok, H, dkd,
                                    DTYPES[k.dtype],
                                    ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise GdrError(rc, "gdr_efla_beta_backward")
    return d_beta


def device_error(stream=None, clear: bool = True) -> int:
    """Synchronise ``stream`` and return the library's device error status."""
    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream()
    return lib.gdr_device_error(ctypes.c_void_p(stream.cuda_stream),
                                int(clear))
