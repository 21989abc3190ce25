"""TEST INFRASTRUCTURE ONLY: fp64 gradients of the gated delta rule.

The gradient of a scalar loss through the recurrence, computed by PyTorch's
reverse-mode autograd (CPU, float64) on the plain token loop -- the same
definition as the C oracle (sources: "DeltaTTT: Layerwise Optimization for
Nonlinear Recurrent Memory", §2 Background and §4.1; "Delta-Rule Linear
Attention" topic page, FG^2-GDN card).  The loss is sum(out * d_out) +
sum(final_state * d_final_state), so the returned gradients are the
vector-Jacobian products the library's backward pass computes.  Small cases
only (one autograd node per token operation).

``gdn2_grads`` does the same for Gated DeltaNet-2's separate gates (the
update of oracle/gdn2_ref.py: read key b_t . k_t, target w_t . v_t, no beta;
Gated DeltaNet-2 abstract on the comparative-study page 2607.07953, which
credits the model with a gate-aware backward pass), ``efla_grads`` for the
EFLA recurrence (the exact-flow step size formed inside the graph), and
``fg2_grads`` for
FG^2-GDN's per-key-channel rate and FG^2-GDN+'s value scaling (the update of
oracle/fg2_ref.py: write key beta_k . k_t, read key k_t, target
c_t . v_t).
"""
from __future__ import annotations

import numpy as np
import torch


def _loop(q, k, v, beta, log_alpha, gate, s0, cu, erase=None, write=None,
          wkey=None):
    H, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    outs = []
    finals = []
    for n in range(len(cu) - 1):
        for_heads = []
        for h in range(H):
            S = (torch.zeros(dk, dv, dtype=torch.float64) if s0 is None
                 else s0[n, h])
            for t in range(cu[n], cu[n + 1]):
                if gate == "scalar":
                    S = torch.exp(log_alpha[t, h]) * S
                elif gate == "channel":
                    S = torch.exp(log_alpha[t, h])[:, None] * S
                kt = k[t, h]
                if wkey is not None:       # FG^2-GDN (+)
                    tgt = v[t, h] if write is None else write[t, h] * v[t, h]
                    u = tgt - S.T @ kt
                    S = S + torch.outer(wkey[t, h] * kt, u)
                    outs.append(((t, h), S.T @ q[t, h]))
                    continue
                if erase is None:
                    r = S.T @ kt
                    u = beta[t, h] * (v[t, h] - r)
                else:
                    r = S.T @ (erase[t, h] * kt)
                    u = write[t, h] * v[t, h] - r
                S = S + torch.outer(kt, u)
                outs.append(((t, h), S.T @ q[t, h]))
            for_heads.append(S)
        finals.append(torch.stack(for_heads))
    return outs, torch.stack(finals)


def gdr_grads(q, k, v, beta, log_alpha=None, gate="scalar",
              initial_state=None, d_out=None, d_final_state=None,
              cu_seqlens=None):
    return _grads(q, k, v, beta, None, None, log_alpha, gate, initial_state,
                  d_out, d_final_state, cu_seqlens)


def gdn2_grads(q, k, v, erase, write, log_alpha=None, gate="channel",
               initial_state=None, d_out=None, d_final_state=None,
               cu_seqlens=None):
    """Gradients of sum(out * d_out) + sum(final * d_final_state) through the
    Gated DeltaNet-2 loop.  erase has the layout of k, write that of v.
    Returns dq, dk, dv, derase, dwrite, dlog_alpha, dinitial_state, out and
    final_state (dbeta is None)."""
    return _grads(q, k, v, None, erase, write, log_alpha, gate,
                  initial_state, d_out, d_final_state, cu_seqlens)


def efla_grads(q, k, v, beta, log_alpha=None, gate="scalar",
               initial_state=None, d_out=None, d_final_state=None):
    """Gradients of sum(out * d_out) + sum(final * d_final_state) through the
    EFLA recurrence: the delta rule with the exact-flow step size
    beta' = (1 - e^{-beta |k|^2}) / |k|^2 ("Delta-Rule Linear Attention"
    topic page, EFLA card), beta' formed inside the autograd graph so that
    dbeta and dk carry its chain rule.  Fixed-length batches; returns the
    same keys as gdr_grads."""
    t64 = lambda a: None if a is None else torch.tensor(  # noqa: E731
        np.asarray(a, np.float64), requires_grad=True)
    Bq, T = np.shape(q)[:2]
    cu = [i * T for i in range(Bq + 1)]
    flat = lambda a: None if a is None else a.reshape(  # noqa: E731
        (-1,) + tuple(a.shape[2:]))
    tq, tk, tv, tb = t64(q), t64(k), t64(v), t64(beta)
    tla = t64(log_alpha) if gate != "none" else None
    ts0 = t64(initial_state)
    s = (tk * tk).sum(-1)
    bprime = -torch.expm1(-tb * s) / s
    outs, final = _loop(flat(tq), flat(tk), flat(tv), flat(bprime), flat(tla),
                        gate, ts0, cu)
    H, dv = np.shape(v)[2], np.shape(v)[3]
    loss = torch.zeros((), dtype=torch.float64)
    dO = None if d_out is None else torch.tensor(
        np.asarray(d_out, np.float64)).reshape(Bq * T, H, dv)
    out = torch.zeros(Bq * T, H, dv, dtype=torch.float64)
    for (t, h), o in outs:
        if dO is not None:
            loss = loss + (o * dO[t, h]).sum()
        out[t, h] = o.detach()
    if d_final_state is not None:
        loss = loss + (final * torch.tensor(
            np.asarray(d_final_state, np.float64))).sum()
    leaves = [x for x in (tq, tk, tv, tb, tla, ts0) if x is not None]
    grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    gm = dict(zip([id(x) for x in leaves], grads))
    g = lambda x: None if x is None else (  # noqa: E731
        np.zeros(x.shape) if gm[id(x)] is None else gm[id(x)].numpy())
    return dict(dq=g(tq), dk=g(tk), dv=g(tv), dbeta=g(tb),
                dlog_alpha=g(tla), dinitial_state=g(ts0),
                out=out.reshape(np.shape(v)).numpy(),
                final_state=final.detach().numpy())


def fg2_grads(q, k, v, beta_k, beta_v=None, log_alpha=None, gate="channel",
              initial_state=None, d_out=None, d_final_state=None,
              cu_seqlens=None):
    """Gradients of sum(out * d_out) + sum(final * d_final_state) through the
    FG^2-GDN loop (beta_v None: FG^2-GDN; else FG^2-GDN+).  beta_k has the
    layout of k, beta_v that of v.  Returns dq, dk, dv, dbeta_k, dbeta_v
    (None without beta_v), dlog_alpha, dinitial_state, out and
    final_state."""
    r = _grads(q, k, v, None, None, beta_v, log_alpha, gate, initial_state,
               d_out, d_final_state, cu_seqlens, wkey=beta_k)
    r["dbeta_k"] = r.pop("dwkey")
    r["dbeta_v"] = r.pop("dwrite")
    r.pop("derase")
    r.pop("dbeta")
    return r


def _grads(q, k, v, beta, erase, write, log_alpha, gate, initial_state,
           d_out, d_final_state, cu_seqlens, wkey=None):
    """Gradients of sum(out * d_out) + sum(final * d_final_state).

    Layouts as for ``oracle.gdr_fwd`` (fixed length [B, T, H, d] or varlen
    [1, total, H, d] with ``cu_seqlens``).  Returns a dict of numpy arrays
    dq, dk, dv, dbeta, dlog_alpha (None without a gate), dinitial_state
    (None without an initial state), plus out and final_state."""
    t64 = lambda a: None if a is None else torch.tensor(  # noqa: E731
        np.asarray(a, np.float64), requires_grad=True)
    Bq, T = np.shape(q)[:2]
    if cu_seqlens is None:
        cu = [i * T for i in range(Bq + 1)]
    else:
        cu = [int(x) for x in cu_seqlens]
    flat = lambda a: None if a is None else a.reshape(  # noqa: E731
        (-1,) + tuple(a.shape[2:]))
    tq, tk, tv, tb = t64(q), t64(k), t64(v), t64(beta)
    te, tw, twk = t64(erase), t64(write), t64(wkey)
    tla = t64(log_alpha) if gate != "none" else None
    ts0 = t64(initial_state)
    outs, final = _loop(flat(tq), flat(tk), flat(tv), flat(tb), flat(tla),
                        gate, ts0, cu, flat(te), flat(tw), flat(twk))
    H, dv = np.shape(v)[2], np.shape(v)[3]
    out = torch.zeros(Bq * T, H, dv, dtype=torch.float64)
    loss = torch.zeros((), dtype=torch.float64)
    dO = None if d_out is None else torch.tensor(
        np.asarray(d_out, np.float64)).reshape(Bq * T, H, dv)
    for (t, h), o in outs:
        if dO is not None:
            loss = loss + (o * dO[t, h]).sum()
        out[t, h] = o.detach()
    if d_final_state is not None:
        loss = loss + (final * torch.tensor(
            np.asarray(d_final_state, np.float64))).sum()
    leaves = [x for x in (tq, tk, tv, tb, te, tw, twk, tla, ts0)
              if x is not None]
    grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    gm = dict(zip([id(x) for x in leaves], grads))
    g = lambda x: None if x is None else (  # noqa: E731
        np.zeros(x.shape) if gm[id(x)] is None else gm[id(x)].numpy())
    return dict(dq=g(tq), dk=g(tk), dv=g(tv), dbeta=g(tb),
                derase=g(te), dwrite=g(tw), dwkey=g(twk),
                dlog_alpha=g(tla), dinitial_state=g(ts0),
                out=out.reshape(np.shape(v)).numpy(),
                final_state=final.detach().numpy())
