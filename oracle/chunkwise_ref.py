"""TEST INFRASTRUCTURE ONLY: independent fp64 chunkwise reformulation.

This is a pin for the token-by-token oracle, not a kernel blueprint: it checks
that the chunkwise-parallel form the pages rely on reaches the same result as
the token loop.  "DeltaTTT: Layerwise Optimization for Nonlinear Recurrent
Memory", §2 Background, states that the state-dependent update is affine in
the preceding memory, which is what makes chunkwise evaluation possible; the
Gated DeltaNet-2 abstract (comparative-study page 2607.07953) names the WY form
with the decay absorbed into the erase factors.  The pages print no formula, so
the steps below are derived here from the token recurrence:

For one chunk of rows r = 1..L with incoming state S0 and in-chunk cumulative
log-decay g_r (per key channel; Gamma_r = diag(exp(g_r))):

    S~_r = D_r S_{r-1},  u_r = beta_r (v_r - S~_r^T k_r),  S_r = S~_r + k_r u_r^T
 => S_r = Gamma_r S0 + sum_{i<=r} Gamma_r Gamma_i^-1 k_i u_i^T
 => (I + A) U = diag(beta) V - diag(beta) (K . exp(g)) S0,
    A[r, i] = beta_r k_r^T Gamma_r Gamma_i^-1 k_i  for i < r, else 0
    o_r     = S0^T Gamma_r q_r + sum_{i<=r} (k_i^T Gamma_i^-1 Gamma_r q_r) u_i
    S_L     = Gamma_L S0 + sum_i Gamma_L Gamma_i^-1 k_i u_i^T

The triangular system is solved with a dense ``numpy.linalg.solve``; decay
ratios exp(g_r - g_i) are formed directly (never as a product of exp(g) and
exp(-g)).  Pure fp64 numpy, no blocking beyond the chunk itself.
"""
from __future__ import annotations

import numpy as np


def _chunk(qc, kc, vc, bc, gc, S0):
    """One chunk of one (sequence, head): qc, kc [L, dk]; vc [L, dv];
    bc [L]; gc [L, dk] cumulative log-decay (0 for no gate)."""
    L = kc.shape[0]
    # decay ratio exp(g_r - g_i) per channel, [r, i, c]
    ratio = np.exp(gc[:, None, :] - gc[None, :, :])
    A = bc[:, None] * np.einsum("rc,ric,ic->ri", kc, ratio, kc)
    A = np.tril(A, k=-1)
    rhs = bc[:, None] * (vc - (kc * np.exp(gc)) @ S0)
    U = np.linalg.solve(np.eye(L) + A, rhs)
    P = np.tril(np.einsum("rc,ric,ic->ri", qc, ratio, kc))
    O = (qc * np.exp(gc)) @ S0 + P @ U
    gL = gc[-1]
    S = np.exp(gL)[:, None] * S0 + (kc * np.exp(gL[None, :] - gc)).T @ U
    return O, S


def chunkwise_ref(q, k, v, beta, log_alpha=None, gate="scalar",
                  initial_state=None, cu_seqlens=None, chunk=16):
    """Chunkwise fp64 evaluation; same arguments and result as ``gdr_fwd``."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    beta = np.asarray(beta, np.float64)
    Bq, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(Bq + 1) * T
        flat = lambda x: x.reshape((Bq * T,) + x.shape[2:])  # noqa: E731
    else:
        cu = np.asarray(cu_seqlens, np.int64)
        flat = lambda x: x.reshape((T,) + x.shape[2:])  # noqa: E731
    qf, kf, vf, bf = flat(q), flat(k), flat(v), flat(beta)
    if gate == "none":
        laf = np.zeros(bf.shape + (dk,))
    elif gate == "scalar":
        laf = np.repeat(flat(np.asarray(log_alpha, np.float64))[..., None],
                        dk, axis=-1)
    else:
        laf = flat(np.asarray(log_alpha, np.float64))
    nseq = len(cu) - 1
    out = np.zeros(vf.shape)
    sT = np.zeros((nseq, H, dk, dv))
    for n in range(nseq):
        for h in range(H):
            S = (np.zeros((dk, dv)) if initial_state is None
                 else np.array(initial_state[n, h], np.float64))
            for s in range(int(cu[n]), int(cu[n + 1]), chunk):
                e = min(s + chunk, int(cu[n + 1]))
                gc = np.cumsum(laf[s:e, h, :], axis=0)
                O, S = _chunk(qf[s:e, h], kf[s:e, h], vf[s:e, h], bf[s:e, h],
                              gc, S)
                out[s:e, h] = O
            sT[n, h] = S
    return out.reshape(v.shape), sT
