"""TEST INFRASTRUCTURE ONLY: fp64 reference of the exact-flow (EFLA) delta rule.

EFLA ("Delta-Rule Linear Attention" topic page, EFLA card) reads the delta
rule's token update S <- S - beta k (S^T k - v)^T as one explicit Euler step of
length beta of the flow

    dS/dtau = -k k^T S + k v^T,

and replaces that step with the exact flow over tau in [0, beta].  This module
integrates the flow directly, with the matrix exponential of the augmented
linear system (no closed form of the rank-1 case is used), so that it pins the
library's closed-form step size independently: for X (dk x dv) and the
constant forcing B = k v^T,

    d/dtau [X; I] = [[-k k^T, B], [0, 0]] [X; I]
    =>  [X(beta); I] = expm(beta M) [X(0); I],   X(beta) = E11 X(0) + E12.

As for the delta rule, the decay D_t applies to the state before the flow, and
o_t = S_t^T q_t reads the state after the token's update.  Small cases only:
one (dk + dv)-square matrix exponential per token.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import expm


def efla_fwd(q, k, v, beta, log_alpha=None, gate="scalar",
             initial_state=None):
    """Token loop of the EFLA recurrence, fixed-length batches.

    q, k [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H]; log_alpha [B, T, H]
    (scalar gate), [B, T, H, dk] (channel gate) or None; initial_state
    [B, H, dk, dv] or None.  Returns (out [B, T, H, dv], final state).
    """
    q, k, v, beta = (np.asarray(a, np.float64) for a in (q, k, v, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = (np.zeros((dk, dv)) if initial_state is None else
                 np.array(initial_state[b, h], np.float64))
            for t in range(T):
                if gate == "scalar":
                    S = np.exp(log_alpha[b, t, h]) * S
                elif gate == "channel":
                    S = np.exp(np.asarray(log_alpha[b, t, h]))[:, None] * S
                kt, vt = k[b, t, h], v[b, t, h]
                M = np.zeros((dk + dv, dk + dv))
                M[:dk, :dk] = -np.outer(kt, kt)
                M[:dk, dk:] = np.outer(kt, vt)
                E = expm(beta[b, t, h] * M)
                S = E[:dk, :dk] @ S + E[:dk, dk:]
                out[b, t, h] = S.T @ q[b, t, h]
            sT[b, h] = S
    return out, sT
