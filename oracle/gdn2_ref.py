"""TEST INFRASTRUCTURE ONLY: fp64 token loop of the forward pass with Gated
DeltaNet-2's separate erase and write gates.

Gated DeltaNet-2 (abstract on the comparative-study page 2607.07953) gives
the delta rule a channel-wise erase gate b_t (per key channel) and a
channel-wise write gate w_t (per value channel) in place of the one scalar
gate beta_t, and reduces to KDA when both collapse to the same scalar.  The
pages print no formula; the reading taken (the delta rule's form, erase gate
on the read key, write gate on the target), per sequence and head:

    S~_t = D_t S_{t-1}
    u_t  = w_t . v_t - S~_t^T (b_t . k_t)
    S_t  = S~_t + k_t u_t^T,      o_t = S_t^T q_t

with D_t = I, alpha_t I or diag(alpha_t) as for the other gates.  Plain numpy
loops over tokens; small cases only.  Pinned in tests/test_oracle.py by its
reduction to the C oracle (b_t = w_t = beta_t 1), the no-erase closed form
(b = 0: a decayed sum of write outer products) and one-hot keys (each row of
S then follows its own scalar recurrence); the same file checks that
plausible mistakes planted in a copy of this loop fail those pins.
"""
from __future__ import annotations

import numpy as np


def gdn2_fwd(q, k, v, erase, write, log_alpha=None, gate="channel",
             initial_state=None, cu_seqlens=None):
    """q, k, erase: [B,T,H,dk]; v, write: [B,T,H,dv] (packed [1,T,...] with
    cu_seqlens); log_alpha: None, [B,T,H] (scalar) or [B,T,H,dk] (channel).
    Returns (out [.., dv], final_state [N,H,dk,dv]) in fp64."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    erase, write = np.asarray(erase, np.float64), np.asarray(write, np.float64)
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
                r = S.T @ (erase[b, t, h] * k[b, t, h])
                u = write[b, t, h] * v[b, t, h] - r
                S = S + np.outer(k[b, t, h], u)
                out[b, t, h] = S.T @ q[b, t, h]
            final[n, h] = S
    return out, final
