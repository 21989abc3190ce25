"""TEST INFRASTRUCTURE ONLY: the fp64 CPU oracle of the gated delta rule.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The product path (``chunkwise_recurrence_b200``)
never imports it and shares no code with it.

Contents
--------
``gdr_fwd``          the plain token-by-token recurrence (C, fp64, threaded over
                     independent (sequence, head) chains) -- the oracle proper.
``decode_step``      one token per (sequence, head): the same recurrence for a
                     single token, applied to a given state.
``efla_fwd``         the exact-flow (EFLA) variant: each token's update is the
                     exact flow of the delta rule's dynamics, integrated with a
                     matrix exponential (small cases only).
``gdr_grads``        fp64 gradients of the recurrence (PyTorch autograd on the
                     plain token loop), the reference for the backward pass.
``gdn2_fwd``         the Gated DeltaNet-2 reading: separate per-key-channel erase
                     and per-value-channel write gates in place of beta (numpy
                     token loop, small cases).
``gdn2_grads``       fp64 gradients of the Gated DeltaNet-2 loop (autograd), the
                     reference for a gate-aware backward pass.
``chunkwise_ref``    an independent fp64 chunkwise reformulation that solves the
                     intra-chunk triangular system with a dense ``solve``; it is a
                     pin for the token loop, not a second oracle for the GPU.

The recurrence, per sequence and head, tokens in order (sources: "DeltaTTT:
Layerwise Optimization for Nonlinear Recurrent Memory", §2 Background and
§4.1; "Delta-Rule Linear Attention" topic page, FG^2-GDN card; the Gated
DeltaNet-2 abstract on the comparative-study page 2607.07953)::

    S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t

with D_t = I (DeltaNet), alpha_t I (Gated DeltaNet) or diag(alpha_t) (KDA).

Parity status: pinned by identities, special cases, brute force and the
independent chunkwise solve (tests/test_oracle.py).  The pages print no worked
numeric example, so no stored value comes from them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

GATES = {"none": 0, "scalar": 1, "channel": 2}


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle (gcc -O2, no fast-math) into a shared library."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-std=c11", src,
           "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def load(path: str | None = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
        _set_sig(lib)
        return lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            _set_sig(lib)
            _lib = lib
    return _lib


def _set_sig(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_gdr_fwd.restype = ctypes.c_int
    lib.oracle_gdr_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                   ctypes.POINTER(ctypes.c_int64),
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int]


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def gdr_fwd(q, k, v, beta, log_alpha=None, gate="scalar", initial_state=None,
            cu_seqlens=None, fixed_base=False, nthreads=0, lib=None):
    """Token-by-token fp64 gated delta rule.

    Fixed length: q, k [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
    log_alpha [B, T, H] (scalar gate) or [B, T, H, dk] (channel gate) or None.
    Varlen: the leading two dims are [1, total] and ``cu_seqlens`` (length
    nseq+1) gives the sequence boundaries.  ``initial_state`` is
    [nseq, H, dk, dv] or None (zero).  Returns (out, final_state, threads_used);
    out has v's shape, final_state is [nseq, H, dk, dv].
    """
    lib = lib or load()
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    g = GATES[gate]
    la = _f64(log_alpha) if g != 0 else None
    if g != 0 and la is None:
        raise ValueError("log_alpha is required for a scalar or channel gate")
    Bq, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(Bq + 1, dtype=np.int64) * T
    else:
        if Bq != 1:
            raise ValueError("varlen input must have a leading batch of 1")
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    nseq = len(cu) - 1
    s0 = _f64(initial_state)
    out = np.zeros(v.shape, dtype=np.float64)
    sT = np.zeros((nseq, H, dk, dv), dtype=np.float64)
    rc = lib.oracle_gdr_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta),
                            _ptr(s0), _ptr(out), _ptr(sT),
                            cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                            nseq, H, dk, dv, g, int(bool(fixed_base)),
                            int(nthreads))
    if rc < 0:
        raise ValueError(f"oracle_gdr_fwd rejected its arguments (code {rc})")
    return out, sT, rc


def decode_step(q, k, v, beta, log_alpha=None, gate="scalar", state=None,
                lib=None):
    """One token per (sequence, head): the recurrence for a single token.

    q, k [N, H, dk]; v [N, H, dv]; beta [N, H]; log_alpha [N, H] (scalar
    gate), [N, H, dk] (channel gate) or None; state [N, H, dk, dv] or None.
    Returns (out [N, H, dv], new state [N, H, dk, dv]).  Decoding applies the
    delta rule's one-token step once per generated token ("Delta-Rule Linear
    Attention" topic page, GDN decode-accelerator card); it is the token loop
    above with one token per sequence, so it reuses it.
    """
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    la = _f64(log_alpha)
    ex = lambda a: None if a is None else a[:, None]  # noqa: E731  [N,1,...]
    out, sT, _ = gdr_fwd(ex(q), ex(k), ex(v), ex(beta), ex(la), gate=gate,
                         initial_state=state, lib=lib)
    return out[:, 0], sT


from .chunkwise_ref import chunkwise_ref  # noqa: E402  (re-export)
from .efla_ref import efla_fwd  # noqa: E402  (re-export)
from .gdn2_ref import gdn2_fwd  # noqa: E402  (re-export)
from .grad_ref import (efla_grads, fg2_grads, gdn2_grads,  # noqa: E402
                       gdr_grads)
from .fg2_ref import fg2_fwd  # noqa: E402  (re-export)
