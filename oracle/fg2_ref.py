"""TEST INFRASTRUCTURE ONLY: fp64 token loop of the forward pass with
FG^2-GDN's channel-wise learning rate (and FG^2-GDN+'s value-side scaling).

"Delta-Rule Linear Attention" topic page, FG^2-GDN card: the delta rule is
an online gradient-descent update whose learning rate beta_t is one scalar;
FG^2-GDN makes it a vector over channels, the way per-coordinate optimisers
(AdaGrad, Adam) refine SGD, and FG^2-GDN+ scales keys and values
separately so that erasing and writing are set apart.  The card prints no
formula.  The reading taken, per sequence and head:

  * the delta rule's step is one gradient step on the regression loss
    L_t(S) = 1/2 ||S^T k_t - v_t||^2, whose gradient is k_t (S^T k_t - v_t)^T
    ("DeltaTTT" page, sec. 4.1);
  * FG^2-GDN gives each key channel (row of S, the channels KDA's decay acts
    on) its own learning rate: S_t = S~_t - diag(beta_t) grad L_t(S~_t);
  * FG^2-GDN+ adds a per-value-channel scaling c_t of the regression
    target, so the key-side vector alone sets how much is erased and c_t
    sets how much is written relative to it.

    S~_t = D_t S_{t-1}
    u_t  = c_t . v_t - S~_t^T k_t          (c_t = 1 for FG^2-GDN)
    S_t  = S~_t + (beta_t . k_t) u_t^T,    o_t = S_t^T q_t

with D_t = I, alpha_t I or diag(alpha_t).  beta_t = beta_t 1 (and c_t = 1)
gives the delta rule.  One rank-one update per token, with write key
beta_t . k_t and read key k_t.  Plain numpy loops over tokens; small cases
only.  Pinned in tests/test_oracle.py by its reduction to the C oracle, by
a central-difference gradient of L_t taken around the decayed state, by
one-hot keys and by a closed form with one token; plausible mistakes
planted in a copy of this loop each fail at least one of those pins.
"""
from __future__ import annotations

import numpy as np


def fg2_fwd(q, k, v, beta_k, beta_v=None, log_alpha=None, gate="channel",
            initial_state=None, cu_seqlens=None):
    """q, k, beta_k: [B,T,H,dk]; v and beta_v (None: FG^2-GDN, all ones):
    [B,T,H,dv] (packed [1,T,...] with cu_seqlens); log_alpha: None,
    [B,T,H] (scalar) or [B,T,H,dk] (channel).  Returns (out [.., dv],
    final_state [N,H,dk,dv]) in fp64."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    bk = np.asarray(beta_k, np.float64)
    bv = (np.ones_like(v) if beta_v is None
          else np.asarray(beta_v, np.float64))
    la = None if log_alpha is None else np.asarray(log_alpha, np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(b, 0, T) for b in range(B)]
    else:
        cu = np.asarray(cu_seqlens).astype(np.int64)
        spans = [(0, int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]
    out = np.zeros((B, T, H, dv))
    final = np.zeros((len(spans), H, dk, dv))
    for n, (b, t0, t1) in enumerate(spans):
        for h in range(H):
            S = (np.zeros((dk, dv)) if initial_state is None
                 else np.array(initial_state[n, h], np.float64))
            for t in range(t0, t1):
                if gate == "scalar":
                    S = np.exp(la[b, t, h]) * S
                elif gate == "channel":
                    S = np.exp(la[b, t, h])[:, None] * S
                u = bv[b, t, h] * v[b, t, h] - S.T @ k[b, t, h]
                S = S + np.outer(bk[b, t, h] * k[b, t, h], u)
                out[b, t, h] = S.T @ q[b, t, h]
            final[n, h] = S
    return out, final
