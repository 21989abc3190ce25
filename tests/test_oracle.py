"""Pins for the fp64 CPU oracle (no GPU).

Each pin checks the token-by-token oracle against something other than itself:
hand-worked values, a finite-difference gradient, closed forms of special cases,
a textbook formula, explicit transition-matrix products, and an independent
chunkwise solve.  ``test_pins_catch_planted_mistakes`` rebuilds the oracle with
plausible mistakes planted in its source and checks that the battery rejects
every one of them.

Sources: "DeltaTTT: Layerwise Optimization for Nonlinear Recurrent Memory",
§2 Background (delta rule = serial gradient descent on a linear memory; fixed-
base evaluation = additive linear attention; the update is affine in the
preceding memory, hence chunkwise evaluation) and §4.1 (a gradient step on a
linear-regression objective is a delta-rule update); "Delta-Rule Linear
Attention" topic page, FG^2-GDN card (KDA: channel-wise decay); Gated
DeltaNet-2 abstract on page 2607.07953 (GDN-2 reduces to KDA, KDA to GDN).
"""
import os
import re
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from oracle import chunkwise_ref, gdr_fwd

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "delta_rule_hand_examples.txt")


# ----------------------------------------------------------------- helpers
def _rand_case(rng, B=2, T=11, H=2, dk=3, dv=4, gate="scalar", s0=True,
               decay=(0.05, 0.6)):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    la = None
    if gate == "scalar":
        la = -rng.uniform(*decay, size=(B, T, H))
    elif gate == "channel":
        la = -rng.uniform(*decay, size=(B, T, H, dk))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None
    return dict(q=q, k=k, v=v, beta=beta, log_alpha=la, gate=gate,
                initial_state=S0)


def _parse_golden(path=GOLDEN):
    blocks, cur = {}, None
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        m = re.match(r"\[(\w+)\]", line)
        if m:
            cur = blocks.setdefault(m.group(1), {})
            continue
        key, val = [s.strip() for s in line.split("=", 1)]
        if key == "gate":
            cur[key] = val
        else:
            cur[key] = np.array([[float(x) for x in row.split()]
                                 for row in val.split(";")])
    return blocks


def _decay_mats(la, gate, dk):
    if gate == "none":
        return np.eye(dk)
    if gate == "scalar":
        return np.exp(la) * np.eye(dk)
    return np.diag(np.exp(la))


# ------------------------------------------------ the battery (any library)
def pin_golden(lib):
    for name, b in _parse_golden().items():
        T = b["k"].shape[0]
        shp = lambda x: x.reshape(1, T, 1, -1)  # noqa: E731
        la = None
        if b["gate"] == "scalar":
            la = np.log(b["alpha"]).reshape(1, T, 1)
        elif b["gate"] == "channel":
            la = np.log(b["alpha"]).reshape(1, T, 1, -1)
        out, sT, _ = gdr_fwd(shp(b["q"]), shp(b["k"]), shp(b["v"]),
                             b["beta"].reshape(1, T, 1), la, gate=b["gate"],
                             initial_state=b["S0"][None, None], lib=lib)
        if not (np.allclose(out[0, :, 0, :], b["out"], atol=1e-12)
                and np.allclose(sT[0, 0], b["S_final"], atol=1e-12)):
            return f"golden example {name}"
    return None


def pin_gradient_step(lib, rng=None):
    """One token with alpha=1 is one gradient step of 1/2||S^T k - v||^2 with
    learning rate beta; with a decay the step is taken at D S0.  The gradient
    is found by central differences (exact for a quadratic up to rounding)."""
    rng = rng or np.random.default_rng(1)
    dk, dv = 3, 5
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=1, T=1, H=1, dk=dk, dv=dv, gate=gate)
        k, v = c["k"][0, 0, 0], c["v"][0, 0, 0]
        b = c["beta"][0, 0, 0]
        la = None if gate == "none" else c["log_alpha"][0, 0, 0]
        S = _decay_mats(la, gate, dk) @ c["initial_state"][0, 0]

        def loss(M):
            r = M.T @ k - v
            return 0.5 * float(r @ r)
        grad = np.zeros_like(S)
        h = 1e-3
        for i in range(dk):
            for j in range(dv):
                E = np.zeros_like(S)
                E[i, j] = h
                grad[i, j] = (loss(S + E) - loss(S - E)) / (2 * h)
        expect = S - b * grad
        out, sT, _ = gdr_fwd(**c, lib=lib)
        if not np.allclose(sT[0, 0], expect, atol=1e-9):
            return f"gradient step ({gate})"
        if not np.allclose(out[0, 0, 0], expect.T @ c["q"][0, 0, 0],
                           atol=1e-9):
            return f"gradient step read-out ({gate})"
    return None


def pin_beta_zero(lib, rng=None):
    """beta = 0: S_T = Gamma_T S0 and o_t = (Gamma_t S0)^T q_t."""
    rng = rng or np.random.default_rng(2)
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=1, T=9, H=2, dk=4, dv=3, gate=gate)
        c["beta"] = np.zeros_like(c["beta"])
        out, sT, _ = gdr_fwd(**c, lib=lib)
        for h in range(2):
            G = np.zeros(4) if gate == "none" else None
            for t in range(9):
                if gate == "scalar":
                    G = np.full(4, c["log_alpha"][0, :t + 1, h].sum())
                elif gate == "channel":
                    G = c["log_alpha"][0, :t + 1, h].sum(axis=0)
                St = np.exp(G)[:, None] * c["initial_state"][0, h]
                if not np.allclose(out[0, t, h], St.T @ c["q"][0, t, h],
                                   atol=1e-12):
                    return f"beta=0 output ({gate})"
            if not np.allclose(sT[0, h], St, atol=1e-12):
                return f"beta=0 final state ({gate})"
    return None


def pin_orthonormal_recall(lib, rng=None):
    """alpha = beta = 1 on orthonormal keys: after writing all of them,
    querying k_i returns v_i, from any initial state."""
    rng = rng or np.random.default_rng(3)
    dk, dv = 6, 5
    for n in (1, 4, 6):
        Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
        k = Qm[:, :n].T.reshape(1, n, 1, dk)
        v = rng.standard_normal((1, n, 1, dv))
        S0 = rng.standard_normal((1, 1, dk, dv))
        _, sT, _ = gdr_fwd(k, k, v, np.ones((1, n, 1)), None, gate="none",
                           initial_state=S0, lib=lib)
        if not np.allclose(sT[0, 0].T @ k[0, :, 0].T, v[0, :, 0].T,
                           atol=1e-12):
            return f"orthonormal recall (n={n})"
    return None


def pin_linear_attention(lib, rng=None):
    """Fixed-base variant (erase term dropped), alpha = 1, S0 = 0:
    o_t = sum_{i<=t} beta_i (k_i . q_t) v_i, the causal linear attention sum."""
    rng = rng or np.random.default_rng(4)
    c = _rand_case(rng, B=1, T=13, H=1, dk=4, dv=3, gate="none", s0=False)
    out, _, _ = gdr_fwd(**c, fixed_base=True, lib=lib)
    q, k, v, b = c["q"][0, :, 0], c["k"][0, :, 0], c["v"][0, :, 0], \
        c["beta"][0, :, 0]
    for t in range(13):
        o = sum(b[i] * (k[i] @ q[t]) * v[i] for i in range(t + 1))
        if not np.allclose(out[0, t, 0], o, atol=1e-12):
            return "fixed base = causal linear attention"
    return None


def pin_transition_products(lib, rng=None):
    """Brute force on tiny inputs: with transition matrices
    M_t = (I - beta_t k_t k_t^T) D_t (dk x dk), the state after t tokens is
    M_t..M_1 S0 + sum_{i<=t} M_t..M_{i+1} beta_i k_i v_i^T.  dk != dv so a
    transposed operand cannot pass."""
    rng = rng or np.random.default_rng(5)
    dk, dv, T = 3, 4, 7
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=1, T=T, H=1, dk=dk, dv=dv, gate=gate)
        out, sT, _ = gdr_fwd(**c, lib=lib)
        k, v, q = c["k"][0, :, 0], c["v"][0, :, 0], c["q"][0, :, 0]
        b = c["beta"][0, :, 0]
        M = []
        for t in range(T):
            la = None if gate == "none" else c["log_alpha"][0, t, 0]
            M.append((np.eye(dk) - b[t] * np.outer(k[t], k[t]))
                     @ _decay_mats(la, gate, dk))

        def prod(lo, hi):  # M_hi ... M_lo (1-based, inclusive); I if empty
            P = np.eye(dk)
            for s in range(lo, hi + 1):
                P = M[s - 1] @ P
            return P
        for t in range(1, T + 1):
            St = prod(1, t) @ c["initial_state"][0, 0]
            for i in range(1, t + 1):
                St = St + prod(i + 1, t) @ (b[i - 1] * np.outer(k[i - 1],
                                                               v[i - 1]))
            if not np.allclose(out[0, t - 1, 0], St.T @ q[t - 1], atol=1e-12):
                return f"transition products, output ({gate})"
        if not np.allclose(sT[0, 0], St, atol=1e-12):
            return f"transition products, state ({gate})"
    return None


def pin_chunkwise(lib, rng=None):
    """The independent chunkwise solve equals the token loop for several chunk
    sizes, ragged tails included."""
    rng = rng or np.random.default_rng(6)
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=2, T=19, H=2, dk=5, dv=3, gate=gate)
        out, sT, _ = gdr_fwd(**c, lib=lib)
        for C in (1, 2, 4, 16):
            o2, s2 = chunkwise_ref(**c, chunk=C)
            scale = max(np.abs(out).max(), 1.0)
            if not (np.abs(o2 - out).max() <= 1e-10 * scale
                    and np.abs(s2 - sT).max() <= 1e-10 * max(
                        np.abs(sT).max(), 1.0)):
                return f"chunkwise (gate={gate}, C={C})"
    return None


BATTERY = [pin_golden, pin_gradient_step, pin_beta_zero,
           pin_orthonormal_recall, pin_linear_attention,
           pin_transition_products, pin_chunkwise]


def run_battery(lib):
    return [f for f in (p(lib) for p in BATTERY) if f]


# ---------------------------------------------------------------- the tests
@pytest.mark.parametrize("pin", BATTERY, ids=lambda p: p.__name__)
def test_pin(oracle_lib, pin):
    assert pin(oracle_lib) is None


def test_gate_reductions(oracle_lib):
    """KDA with equal channels = GDN; GDN with log alpha = 0 = DeltaNet."""
    rng = np.random.default_rng(7)
    c = _rand_case(rng, B=2, T=17, H=3, dk=4, dv=5, gate="scalar")
    o_s, s_s, _ = gdr_fwd(**c)
    cc = dict(c, gate="channel",
              log_alpha=np.repeat(c["log_alpha"][..., None], 4, axis=-1))
    o_c, s_c, _ = gdr_fwd(**cc)
    assert np.allclose(o_s, o_c, atol=1e-13) and np.allclose(s_s, s_c,
                                                             atol=1e-13)
    cz = dict(c, log_alpha=np.zeros_like(c["log_alpha"]))
    o_z, s_z, _ = gdr_fwd(**cz)
    o_n, s_n, _ = gdr_fwd(**dict(c, gate="none", log_alpha=None))
    assert np.array_equal(o_z, o_n) and np.array_equal(s_z, s_n)


def test_state_carry_split(oracle_lib):
    """Two calls chained through final_state -> initial_state = one call."""
    rng = np.random.default_rng(8)
    c = _rand_case(rng, B=2, T=20, H=2, dk=4, dv=4, gate="channel")
    o, s, _ = gdr_fwd(**c)
    cut = 7
    a = {x: (c[x][:, :cut] if x in ("q", "k", "v", "beta", "log_alpha")
             else c[x]) for x in c}
    o1, s1, _ = gdr_fwd(**a)
    b = {x: (c[x][:, cut:] if x in ("q", "k", "v", "beta", "log_alpha")
             else c[x]) for x in c}
    b["initial_state"] = s1
    o2, s2, _ = gdr_fwd(**b)
    assert np.allclose(np.concatenate([o1, o2], axis=1), o, atol=1e-13)
    assert np.allclose(s2, s, atol=1e-13)


def test_varlen_equals_separate(oracle_lib):
    rng = np.random.default_rng(9)
    lens = [5, 1, 12, 0, 9]
    H, dk, dv = 2, 3, 4
    cases = [_rand_case(rng, B=1, T=L, H=H, dk=dk, dv=dv, gate="scalar")
             for L in lens]
    cat = lambda x: np.concatenate([c[x] for c in cases], axis=1)  # noqa
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0 = np.concatenate([c["initial_state"] for c in cases], axis=0)
    o, s, _ = gdr_fwd(cat("q"), cat("k"), cat("v"), cat("beta"),
                      cat("log_alpha"), gate="scalar", initial_state=S0,
                      cu_seqlens=cu)
    for n, c in enumerate(cases):
        on, sn, _ = gdr_fwd(**c)
        assert np.array_equal(o[:, cu[n]:cu[n + 1]], on)
        assert np.array_equal(s[n], sn[0])
    # chunkwise reformulation handles the same packing
    o2, s2 = chunkwise_ref(cat("q"), cat("k"), cat("v"), cat("beta"),
                           cat("log_alpha"), gate="scalar", initial_state=S0,
                           cu_seqlens=cu, chunk=4)
    assert np.allclose(o2, o, atol=1e-11) and np.allclose(s2, s, atol=1e-11)


def test_decode_step_chains_to_the_sequence(oracle_lib):
    """One-token steps, each handing its state to the next, reproduce the
    token loop over the whole sequence: outputs and final state (this is what
    the decode wrapper's reshaping and state handling must preserve)."""
    rng = np.random.default_rng(11)
    for gate in ("none", "scalar", "channel"):
        case = _rand_case(rng, B=3, T=6, H=2, dk=4, dv=3, gate=gate)
        out, sT, _ = gdr_fwd(**case, lib=oracle_lib)
        S = case["initial_state"]
        for t in range(case["q"].shape[1]):
            la = None if case["log_alpha"] is None else case["log_alpha"][:, t]
            o, S = oracle.decode_step(case["q"][:, t], case["k"][:, t],
                                      case["v"][:, t], case["beta"][:, t], la,
                                      gate=gate, state=S, lib=oracle_lib)
            np.testing.assert_allclose(o, out[:, t], rtol=0, atol=1e-13)
        np.testing.assert_allclose(S, sT, rtol=0, atol=1e-13)


def test_decode_step_special_cases(oracle_lib):
    """beta = 0: the step only decays the state, S' = D S and o = (D S)^T q.
    alpha = beta = 1 from a zero state: one write of (k, v) with a unit key
    stores v, so reading with q = k returns v exactly (DeltaTTT page, §2: the
    delta rule corrects the memory's read of the current key to its value)."""
    rng = np.random.default_rng(12)
    N, H, dk, dv = 3, 2, 5, 4
    for gate in ("none", "scalar", "channel"):
        q = rng.standard_normal((N, H, dk))
        k = rng.standard_normal((N, H, dk))
        v = rng.standard_normal((N, H, dv))
        S = rng.standard_normal((N, H, dk, dv))
        la = None if gate == "none" else -rng.uniform(
            0.1, 1.0, size=(N, H) if gate == "scalar" else (N, H, dk))
        o, S1 = oracle.decode_step(q, k, v, np.zeros((N, H)), la, gate=gate,
                                   state=S, lib=oracle_lib)
        for n in range(N):
            for h in range(H):
                if gate == "none":
                    D = np.eye(dk)
                elif gate == "scalar":
                    D = np.exp(la[n, h]) * np.eye(dk)
                else:
                    D = np.diag(np.exp(la[n, h]))
                np.testing.assert_allclose(S1[n, h], D @ S[n, h], atol=1e-13)
                np.testing.assert_allclose(o[n, h], (D @ S[n, h]).T @ q[n, h],
                                           atol=1e-12)
    kk = rng.standard_normal((N, H, dk))
    kk /= np.linalg.norm(kk, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, dv))
    o, _ = oracle.decode_step(kk, kk, v, np.ones((N, H)), None, gate="none",
                              state=None, lib=oracle_lib)
    np.testing.assert_allclose(o, v, atol=1e-13)


def _efla_step_size(k, beta):
    lam = np.sum(np.asarray(k) ** 2, axis=-1)
    return np.where(lam > 0, -np.expm1(-beta * lam) / np.where(lam > 0, lam, 1),
                    beta)


def _efla_flow(fn, lib=None):
    """The exact flow, integrated by a matrix exponential, equals the delta
    rule run with beta' = (1 - e^{-beta |k|^2}) / |k|^2 -- the closed form the
    library's gdr_efla_beta computes -- for every gate, with unnormalised keys
    too."""
    rng = np.random.default_rng(21)
    ok = True
    for gate in ("none", "scalar", "channel"):
        case = _rand_case(rng, B=2, T=7, H=2, dk=4, dv=3, gate=gate)
        case["k"] = case["k"] * rng.uniform(0.3, 2.0, size=case["k"].shape[:-1]
                                            + (1,))
        case["beta"] = case["beta"] * 3.0
        ro, rs = fn(**case)
        bp = _efla_step_size(case["k"], case["beta"])
        o, sT, _ = gdr_fwd(**{**case, "beta": bp}, lib=lib)
        ok &= np.allclose(o, ro, rtol=0, atol=1e-10)
        ok &= np.allclose(sT, rs, rtol=0, atol=1e-10)
    return ok


def _efla_limits(fn):
    """Small steps: the exact flow and one Euler step (the delta rule) agree
    to first order in beta.  Long flow with a unit key: the memory converges
    to the least-squares solution, so reading the key returns the value."""
    rng = np.random.default_rng(22)
    dk, dv = 5, 3
    k = rng.standard_normal((1, 1, 1, dk))
    k /= np.linalg.norm(k)
    v = rng.standard_normal((1, 1, 1, dv))
    S0 = rng.standard_normal((1, 1, dk, dv))
    ok = True
    for b in (1e-3, 1e-4):
        _, se = fn(k, k, v, np.full((1, 1, 1), b), gate="none",
                   initial_state=S0)
        euler = S0[0, 0] - b * np.outer(k[0, 0, 0], S0[0, 0].T @ k[0, 0, 0]
                                        - v[0, 0, 0])
        ok &= bool(np.max(np.abs(se[0, 0] - euler)) < 5 * b * b * (
            1 + np.max(np.abs(S0))))
    _, se = fn(k, k, v, np.full((1, 1, 1), 60.0), gate="none",
               initial_state=S0)
    return ok and np.allclose(se[0, 0].T @ k[0, 0, 0], v[0, 0, 0], rtol=0,
                              atol=1e-12)


def test_efla_flow_is_the_delta_rule_with_a_new_step_size(oracle_lib):
    assert _efla_flow(oracle.efla_fwd, oracle_lib)


def test_efla_limits():
    assert _efla_limits(oracle.efla_fwd)


# plausible mistakes in the EFLA flow integration, as (text, mutant)
EFLA_MUTANTS = {
    "flow_sign": ("M[:dk, :dk] = -np.outer(kt, kt)",
                  "M[:dk, :dk] = np.outer(kt, kt)"),
    "forcing_sign": ("M[:dk, dk:] = np.outer(kt, vt)",
                     "M[:dk, dk:] = -np.outer(kt, vt)"),
    "forcing_dropped": ("S = E[:dk, :dk] @ S + E[:dk, dk:]",
                        "S = E[:dk, :dk] @ S"),
    "step_length_ignored": ("E = expm(beta[b, t, h] * M)", "E = expm(M)"),
    "read_before_update": (
        "S = E[:dk, :dk] @ S + E[:dk, dk:]\n"
        "                out[b, t, h] = S.T @ q[b, t, h]",
        "out[b, t, h] = S.T @ q[b, t, h]\n"
        "                S = E[:dk, :dk] @ S + E[:dk, dk:]"),
    "scalar_decay_sign": ("S = np.exp(log_alpha[b, t, h]) * S",
                          "S = np.exp(-log_alpha[b, t, h]) * S"),
    "channel_decay_dropped": (
        "S = np.exp(np.asarray(log_alpha[b, t, h]))[:, None] * S", "S = S"),
}


def test_efla_pins_catch_planted_mistakes(oracle_lib):
    """Each plausible mistake, planted in a copy of the EFLA loop, fails at
    least one of its pins."""
    src = open(os.path.join(os.path.dirname(oracle.__file__),
                            "efla_ref.py")).read()
    for name, (text, mutant) in EFLA_MUTANTS.items():
        assert src.count(text) == 1, name
        ns = {"__name__": f"efla_mutant_{name}"}
        exec(compile(src.replace(text, mutant), name, "exec"), ns)
        fn = ns["efla_fwd"]
        fails = []
        for pin, call in (("flow", lambda: _efla_flow(fn, oracle_lib)),
                          ("limits", lambda: _efla_limits(fn))):
            try:
                ok = call()
            except Exception:  # noqa: BLE001  (a crash is a failed pin)
                ok = False
            if not ok:
                fails.append(pin)
        assert fails, f"planted mistake '{name}' passed every pin"


def _gdn2_reduction(fn, gate):
    """Erase and write gates equal to beta_t on every channel give the delta
    rule: the Gated DeltaNet-2 loop matches the C oracle."""
    rng = np.random.default_rng(31)
    c = _rand_case(rng, B=2, T=13, H=2, dk=4, dv=3, gate=gate)
    o, s, _ = gdr_fwd(**c)
    b = c["beta"]
    go, gs = fn(c["q"], c["k"], c["v"], np.repeat(b[..., None], 4, axis=-1),
                np.repeat(b[..., None], 3, axis=-1), c["log_alpha"], gate,
                c["initial_state"])
    return np.allclose(go, o, atol=1e-13) and np.allclose(gs, s, atol=1e-13)


def _gdn2_no_erase(fn):
    """b = 0: nothing is erased, so S_t = sum_{s<=t} (prod_{s<tau<=t} D_tau)
    k_s (w_s . v_s)^T (+ the decayed initial state), summed directly."""
    rng = np.random.default_rng(32)
    c = _rand_case(rng, B=1, T=9, H=1, dk=3, dv=2, gate="channel")
    w = rng.uniform(0.1, 1.0, size=(1, 9, 1, 2))
    go, gs = fn(c["q"], c["k"], c["v"], np.zeros((1, 9, 1, 3)), w,
                c["log_alpha"], "channel", c["initial_state"])
    la = c["log_alpha"][0, :, 0]
    ok = True
    for t in range(9):
        S = np.exp(la[:t + 1].sum(axis=0))[:, None] * c["initial_state"][0, 0]
        for s_ in range(t + 1):
            dec = np.exp(la[s_ + 1:t + 1].sum(axis=0))
            S = S + np.outer(dec * c["k"][0, s_, 0],
                             w[0, s_, 0] * c["v"][0, s_, 0])
        ok &= np.allclose(go[0, t, 0], S.T @ c["q"][0, t, 0], atol=1e-13)
    return ok and np.allclose(gs[0, 0], S, atol=1e-13)


def _gdn2_one_hot(fn):
    """With k_t = e_c, only row c of S changes, and it follows
    S_c <- (1 - b_t[c]) a_t[c] S_c + w_t . v_t (a = the decay of row c)."""
    rng = np.random.default_rng(33)
    T, dk, dv = 10, 3, 4
    cs = rng.integers(0, dk, size=T)
    k = np.zeros((1, T, 1, dk))
    k[0, np.arange(T), 0, cs] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    b = rng.uniform(0, 1, size=(1, T, 1, dk))
    w = rng.uniform(0, 1, size=(1, T, 1, dv))
    la = -rng.uniform(0.05, 0.5, size=(1, T, 1, dk))
    S0 = rng.standard_normal((1, 1, dk, dv))
    go, gs = fn(q, k, v, b, w, la, "channel", S0)
    S = S0[0, 0].copy()
    ok = True
    for t in range(T):
        S = np.exp(la[0, t, 0])[:, None] * S
        c = cs[t]
        S[c] = (1 - b[0, t, 0, c]) * S[c] + w[0, t, 0] * v[0, t, 0]
        ok &= np.allclose(go[0, t, 0], S.T @ q[0, t, 0], atol=1e-13)
    return ok and np.allclose(gs[0, 0], S, atol=1e-13)


def _gdn2_battery(fn):
    """Names of the Gated DeltaNet-2 pins that `fn` fails (an exception
    counts as a failure)."""
    pins = {f"reduction_{g}": (lambda g=g: _gdn2_reduction(fn, g))
            for g in ("none", "scalar", "channel")}
    pins["no_erase"] = lambda: _gdn2_no_erase(fn)
    pins["one_hot"] = lambda: _gdn2_one_hot(fn)
    fails = []
    for name, pin in pins.items():
        try:
            ok = pin()
        except Exception:  # noqa: BLE001  (a crash is a failed pin)
            ok = False
        if not ok:
            fails.append(name)
    return fails


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
def test_gdn2_reduces_to_the_delta_rule(oracle_lib, gate):
    assert _gdn2_reduction(oracle.gdn2_fwd, gate)


def test_gdn2_without_erase_is_decayed_linear_attention(oracle_lib):
    assert _gdn2_no_erase(oracle.gdn2_fwd)


def test_gdn2_one_hot_keys_update_rows_independently(oracle_lib):
    assert _gdn2_one_hot(oracle.gdn2_fwd)


# plausible mistakes in the Gated DeltaNet-2 token loop, as (text, mutant)
GDN2_MUTANTS = {
    "erase_gate_dropped": (
        "r = S.T @ (erase[b, t, h] * k[b, t, h])", "r = S.T @ k[b, t, h]"),
    "write_gate_dropped": (
        "u = write[b, t, h] * v[b, t, h] - r", "u = v[b, t, h] - r"),
    "write_gate_on_the_residual": (
        "u = write[b, t, h] * v[b, t, h] - r",
        "u = write[b, t, h] * (v[b, t, h] - r)"),
    "written_along_the_read_key": (
        "S = S + np.outer(k[b, t, h], u)",
        "S = S + np.outer(erase[b, t, h] * k[b, t, h], u)"),
    "residual_sign": (
        "u = write[b, t, h] * v[b, t, h] - r",
        "u = write[b, t, h] * v[b, t, h] + r"),
    "scalar_decay_sign": (
        "S = np.exp(la[b, t, h]) * S", "S = np.exp(-la[b, t, h]) * S"),
    "channel_decay_dropped": (
        "S = np.exp(la[b, t, h])[:, None] * S", "S = S"),
    "read_before_write": (
        "out[b, t, h] = S.T @ q[b, t, h]",
        "out[b, t, h] = (S - np.outer(k[b, t, h], u)).T @ q[b, t, h]"),
    "initial_state_ignored": (
        "else np.array(initial_state[n, h], np.float64))",
        "else np.zeros((dk, dv)))"),
}


def test_gdn2_pins_catch_planted_mistakes(oracle_lib):
    """Each plausible mistake, planted in a copy of the Gated DeltaNet-2 loop,
    fails at least one of its pins; the loop as written fails none."""
    assert _gdn2_battery(oracle.gdn2_fwd) == []
    src = open(os.path.join(os.path.dirname(oracle.__file__),
                            "gdn2_ref.py")).read()
    for name, (text, mutant) in GDN2_MUTANTS.items():
        assert src.count(text) == 1, name
        ns = {"__name__": f"gdn2_mutant_{name}"}
        exec(compile(src.replace(text, mutant), name, "exec"), ns)
        assert _gdn2_battery(ns["gdn2_fwd"]), (
            f"planted mistake '{name}' passed every pin")


def _fg2_case(rng, B=1, T=7, H=1, dk=3, dv=4, gate="channel"):
    c = _rand_case(rng, B=B, T=T, H=H, dk=dk, dv=dv, gate=gate)
    c["beta_k"] = rng.uniform(0.05, 1.0, size=(B, T, H, dk))
    c["beta_v"] = rng.uniform(0.1, 1.5, size=(B, T, H, dv))
    return c


def _fg2_reduction(fn, gate):
    """A key-side rate equal to beta_t on every channel (no value scaling,
    or a value scaling of ones) gives the delta rule: the loop matches the
    C oracle."""
    rng = np.random.default_rng(41)
    c = _rand_case(rng, B=2, T=13, H=2, dk=4, dv=3, gate=gate)
    o, s, _ = gdr_fwd(**c)
    bk = np.repeat(c["beta"][..., None], 4, axis=-1)
    ok = True
    for bv in (None, np.ones_like(c["v"])):
        fo, fs = fn(c["q"], c["k"], c["v"], bk, bv, c["log_alpha"], gate,
                    c["initial_state"])
        ok &= np.allclose(fo, o, atol=1e-13) and np.allclose(fs, s, atol=1e-13)
    return ok


def _fd_grad(loss, S, h=1e-3):
    """Central differences of loss at S, entry by entry (exact up to rounding
    for a quadratic loss)."""
    G = np.zeros_like(S)
    for idx in np.ndindex(*S.shape):
        E = np.zeros_like(S)
        E[idx] = h
        G[idx] = (loss(S + E) - loss(S - E)) / (2 * h)
    return G


def _fg2_gradient_step(fn, value_scale=True):
    """Token by token, the state is the decayed state minus diag(beta_k)
    times the gradient of L(S) = 1/2 ||S^T k - c . v||^2, the gradient taken
    by central differences of L around the decayed state; the output reads
    the state after the token's write."""
    rng = np.random.default_rng(42)
    T, dk, dv = 6, 3, 4
    c = _fg2_case(rng, T=T, dk=dk, dv=dv, gate="channel")
    bv = c["beta_v"] if value_scale else None
    fo, fs = fn(c["q"], c["k"], c["v"], c["beta_k"], bv, c["log_alpha"],
                "channel", c["initial_state"])
    S = c["initial_state"][0, 0].copy()
    ok = True
    for t in range(T):
        S = np.exp(c["log_alpha"][0, t, 0])[:, None] * S
        k = c["k"][0, t, 0]
        tgt = (bv[0, t, 0] if value_scale else 1.0) * c["v"][0, t, 0]
        G = _fd_grad(lambda X: 0.5 * np.sum((X.T @ k - tgt) ** 2), S)
        S = S - c["beta_k"][0, t, 0][:, None] * G
        ok &= np.allclose(fo[0, t, 0], S.T @ c["q"][0, t, 0], atol=1e-8)
    return ok and np.allclose(fs[0, 0], S, atol=1e-8)


def _fg2_one_hot(fn):
    """With k_t = e_c only row c of the state changes, and it moves a
    fraction beta_k[c] of the way to the scaled target:
    S_c <- (1 - beta_k[c]) a_t[c] S_c + beta_k[c] (c_t . v_t)."""
    rng = np.random.default_rng(43)
    T, dk, dv = 10, 3, 4
    cs = rng.integers(0, dk, size=T)
    k = np.zeros((1, T, 1, dk))
    k[0, np.arange(T), 0, cs] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    bk = rng.uniform(0, 1, size=(1, T, 1, dk))
    bv = rng.uniform(0, 2, size=(1, T, 1, dv))
    la = -rng.uniform(0.05, 0.5, size=(1, T, 1, dk))
    S0 = rng.standard_normal((1, 1, dk, dv))
    fo, fs = fn(q, k, v, bk, bv, la, "channel", S0)
    S = S0[0, 0].copy()
    ok = True
    for t in range(T):
        S = np.exp(la[0, t, 0])[:, None] * S
        r = cs[t]
        S[r] = (1 - bk[0, t, 0, r]) * S[r] + bk[0, t, 0, r] * bv[0, t, 0] * v[0, t, 0]
        ok &= np.allclose(fo[0, t, 0], S.T @ q[0, t, 0], atol=1e-13)
    return ok and np.allclose(fs[0, 0], S, atol=1e-13)


def _fg2_scalar_gate(fn):
    """The scalar decay alpha_t scales the whole state: it equals the channel
    gate with the same log-decay on every channel."""
    rng = np.random.default_rng(44)
    c = _fg2_case(rng, B=2, T=9, H=2, dk=3, dv=2, gate="scalar")
    la_c = np.repeat(c["log_alpha"][..., None], 3, axis=-1)
    a = fn(c["q"], c["k"], c["v"], c["beta_k"], c["beta_v"], c["log_alpha"],
           "scalar", c["initial_state"])
    b = fn(c["q"], c["k"], c["v"], c["beta_k"], c["beta_v"], la_c,
           "channel", c["initial_state"])
    return all(np.allclose(x, y, atol=1e-13) for x, y in zip(a, b))


def _fg2_battery(fn):
    """Names of the FG^2-GDN pins that `fn` fails (an exception counts as a
    failure)."""
    pins = {f"reduction_{g}": (lambda g=g: _fg2_reduction(fn, g))
            for g in ("none", "scalar", "channel")}
    pins["gradient_step"] = lambda: _fg2_gradient_step(fn)
    pins["gradient_step_no_value_scale"] = (
        lambda: _fg2_gradient_step(fn, value_scale=False))
    pins["one_hot"] = lambda: _fg2_one_hot(fn)
    pins["scalar_gate"] = lambda: _fg2_scalar_gate(fn)
    fails = []
    for name, pin in pins.items():
        try:
            ok = pin()
        except Exception:  # noqa: BLE001  (a crash is a failed pin)
            ok = False
        if not ok:
            fails.append(name)
    return fails


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
def test_fg2_reduces_to_the_delta_rule(oracle_lib, gate):
    assert _fg2_reduction(oracle.fg2_fwd, gate)


@pytest.mark.parametrize("value_scale", [False, True])
def test_fg2_is_a_per_key_channel_gradient_step(value_scale):
    assert _fg2_gradient_step(oracle.fg2_fwd, value_scale)


def test_fg2_one_hot_keys_move_one_row_toward_the_target():
    assert _fg2_one_hot(oracle.fg2_fwd)


def test_fg2_packed_sequences_equal_separate_calls():
    rng = np.random.default_rng(45)
    lens = [5, 1, 8]
    cu = np.concatenate([[0], np.cumsum(lens)])
    c = _fg2_case(rng, B=1, T=int(cu[-1]), H=2, dk=3, dv=2)
    S0 = rng.standard_normal((3, 2, 3, 2))
    po, ps = oracle.fg2_fwd(c["q"], c["k"], c["v"], c["beta_k"], c["beta_v"],
                            c["log_alpha"], "channel", S0, cu_seqlens=cu)
    for n in range(3):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        o, s = oracle.fg2_fwd(c["q"][:, sl], c["k"][:, sl], c["v"][:, sl],
                              c["beta_k"][:, sl], c["beta_v"][:, sl],
                              c["log_alpha"][:, sl], "channel", S0[n:n + 1])
        assert np.array_equal(po[:, sl], o) and np.array_equal(ps[n], s[0])


# plausible mistakes in the FG^2-GDN token loop, as (text, mutant)
_FG2_U = "u = bv[b, t, h] * v[b, t, h] - S.T @ k[b, t, h]"
_FG2_W = "S = S + np.outer(bk[b, t, h] * k[b, t, h], u)"
FG2_MUTANTS = {
    "key_rate_dropped": (_FG2_W, "S = S + np.outer(k[b, t, h], u)"),
    "key_rate_on_the_read_key_too": (
        _FG2_U, "u = bv[b, t, h] * v[b, t, h] - S.T @ (bk[b, t, h] * k[b, t, h])"),
    "key_rate_on_the_read_key_only": (
        _FG2_U + "\n                " + _FG2_W,
        "u = bv[b, t, h] * v[b, t, h] - S.T @ (bk[b, t, h] * k[b, t, h])"
        "\n                S = S + np.outer(k[b, t, h], u)"),
    "value_scale_dropped": (_FG2_U, "u = v[b, t, h] - S.T @ k[b, t, h]"),
    "value_scale_on_the_residual": (
        _FG2_U, "u = bv[b, t, h] * (v[b, t, h] - S.T @ k[b, t, h])"),
    "residual_sign": (_FG2_U, "u = bv[b, t, h] * v[b, t, h] + S.T @ k[b, t, h]"),
    "scalar_decay_sign": (
        "S = np.exp(la[b, t, h]) * S", "S = np.exp(-la[b, t, h]) * S"),
    "channel_decay_dropped": (
        "S = np.exp(la[b, t, h])[:, None] * S", "S = S"),
    "channel_decay_on_value_channels": (
        "S = np.exp(la[b, t, h])[:, None] * S",
        "S = S * np.exp(la[b, t, h])[:S.shape[1]][None, :]"),
    "read_before_write": (
        "out[b, t, h] = S.T @ q[b, t, h]",
        "out[b, t, h] = (S - np.outer(bk[b, t, h] * k[b, t, h], u)).T @ q[b, t, h]"),
    "initial_state_ignored": (
        "else np.array(initial_state[n, h], np.float64))",
        "else np.zeros((dk, dv)))"),
}


def test_fg2_pins_catch_planted_mistakes(oracle_lib):
    """Each plausible mistake, planted in a copy of the FG^2-GDN loop, fails
    at least one of its pins; the loop as written fails none."""
    assert _fg2_battery(oracle.fg2_fwd) == []
    src = open(os.path.join(os.path.dirname(oracle.__file__),
                            "fg2_ref.py")).read()
    for name, (text, mutant) in FG2_MUTANTS.items():
        assert src.count(text) == 1, name
        ns = {"__name__": f"fg2_mutant_{name}"}
        exec(compile(src.replace(text, mutant), name, "exec"), ns)
        assert _fg2_battery(ns["fg2_fwd"]), (
            f"planted mistake '{name}' passed every pin")


def test_gradients_match_finite_differences(oracle_lib):
    """The autograd gradients (oracle.gdr_grads, on a PyTorch token loop) agree
    with central differences of the C token loop's loss, element by element,
    for every input and every gate: the two share no code."""
    rng = np.random.default_rng(31)
    for gate in ("none", "scalar", "channel"):
        case = _rand_case(rng, B=2, T=5, H=1, dk=3, dv=2, gate=gate)
        dO = rng.standard_normal(case["v"].shape)
        dS = rng.standard_normal((2, 1, 3, 2))
        g = oracle.gdr_grads(**case, d_out=dO, d_final_state=dS)

        def loss(c):
            o, sT, _ = gdr_fwd(**c, lib=oracle_lib)
            return float((o * dO).sum() + (sT * dS).sum())

        names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"),
                 ("initial_state", "dinitial_state")]
        if gate != "none":
            names.append(("log_alpha", "dlog_alpha"))
        eps = 1e-6
        for key, gk in names:
            x = case[key]
            fd = np.zeros_like(x)
            for i in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[i] += eps
                xm[i] -= eps
                fd[i] = (loss({**case, key: xp}) - loss({**case, key: xm})) / (
                    2 * eps)
            np.testing.assert_allclose(g[gk], fd, atol=2e-7, rtol=1e-6,
                                       err_msg=f"{gate} {key}")
        o, sT, _ = gdr_fwd(**case, lib=oracle_lib)
        np.testing.assert_allclose(g["out"], o, atol=1e-13)
        np.testing.assert_allclose(g["final_state"], sT, atol=1e-13)


def test_gdn2_gradients_match_finite_differences():
    """The Gated DeltaNet-2 autograd gradients (oracle.gdn2_grads, a PyTorch
    token loop) agree with central differences of the numpy loop's loss
    (oracle.gdn2_fwd), element by element, for every input -- the erase and
    write gates included -- and every gate kind."""
    rng = np.random.default_rng(41)
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=1, T=5, H=1, dk=3, dv=2, gate=gate)
        case = dict(q=c["q"], k=c["k"], v=c["v"],
                    erase=rng.uniform(0.1, 0.9, size=(1, 5, 1, 3)),
                    write=rng.uniform(0.1, 0.9, size=(1, 5, 1, 2)),
                    log_alpha=c["log_alpha"], initial_state=c["initial_state"])
        dO = rng.standard_normal(c["v"].shape)
        dS = rng.standard_normal((1, 1, 3, 2))
        g = oracle.gdn2_grads(**case, gate=gate, d_out=dO, d_final_state=dS)

        def loss(x):
            o, sT = oracle.gdn2_fwd(x["q"], x["k"], x["v"], x["erase"],
                                    x["write"], x["log_alpha"], gate,
                                    x["initial_state"])
            return float((o * dO).sum() + (sT * dS).sum())

        names = ["q", "k", "v", "erase", "write", "initial_state"]
        if gate != "none":
            names.append("log_alpha")
        eps = 1e-6
        for key in names:
            x = case[key]
            fd = np.zeros_like(x)
            for i in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[i] += eps
                xm[i] -= eps
                fd[i] = (loss({**case, key: xp}) - loss({**case, key: xm})) / (
                    2 * eps)
            np.testing.assert_allclose(g["d" + key], fd, atol=2e-7, rtol=1e-6,
                                       err_msg=f"{gate} {key}")
        assert g["dbeta"] is None
        o, sT = oracle.gdn2_fwd(case["q"], case["k"], case["v"],
                                case["erase"], case["write"],
                                case["log_alpha"], gate,
                                case["initial_state"])
        np.testing.assert_allclose(g["out"], o, atol=1e-13)
        np.testing.assert_allclose(g["final_state"], sT, atol=1e-13)


@pytest.mark.parametrize("plus", [False, True])
def test_fg2_gradients_match_finite_differences(plus):
    """The FG^2-GDN autograd gradients (oracle.fg2_grads, a PyTorch token
    loop) agree with central differences of the numpy loop's loss
    (oracle.fg2_fwd), element by element, for every input -- the key-side
    rate and, for FG^2-GDN+, the value scaling included -- and every gate
    kind."""
    rng = np.random.default_rng(51 + plus)
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=1, T=5, H=1, dk=3, dv=2, gate=gate)
        case = dict(q=c["q"], k=c["k"], v=c["v"],
                    beta_k=rng.uniform(0.1, 0.9, size=(1, 5, 1, 3)),
                    beta_v=(rng.uniform(0.1, 1.5, size=(1, 5, 1, 2))
                            if plus else None),
                    log_alpha=c["log_alpha"], initial_state=c["initial_state"])
        dO = rng.standard_normal(c["v"].shape)
        dS = rng.standard_normal((1, 1, 3, 2))
        g = oracle.fg2_grads(**case, gate=gate, d_out=dO, d_final_state=dS)

        def loss(x):
            o, sT = oracle.fg2_fwd(x["q"], x["k"], x["v"], x["beta_k"],
                                   x["beta_v"], x["log_alpha"], gate,
                                   x["initial_state"])
            return float((o * dO).sum() + (sT * dS).sum())

        names = ["q", "k", "v", "beta_k", "initial_state"]
        if plus:
            names.append("beta_v")
        if gate != "none":
            names.append("log_alpha")
        eps = 1e-6
        for key in names:
            x = case[key]
            fd = np.zeros_like(x)
            for i in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[i] += eps
                xm[i] -= eps
                fd[i] = (loss({**case, key: xp}) - loss({**case, key: xm})) / (
                    2 * eps)
            np.testing.assert_allclose(g["d" + key], fd, atol=2e-7, rtol=1e-6,
                                       err_msg=f"{gate} {key}")
        if not plus:
            assert g["dbeta_v"] is None
        o, sT = oracle.fg2_fwd(case["q"], case["k"], case["v"],
                               case["beta_k"], case["beta_v"],
                               case["log_alpha"], gate, case["initial_state"])
        np.testing.assert_allclose(g["out"], o, atol=1e-13)
        np.testing.assert_allclose(g["final_state"], sT, atol=1e-13)


def test_fg2_gradients_reduce_to_the_delta_rule():
    """A key-side rate of beta on every channel (no value scaling) is the
    delta rule: the gradients equal oracle.gdr_grads', with dbeta the rate's
    gradient summed over its channels."""
    rng = np.random.default_rng(53)
    c = _rand_case(rng, B=1, T=6, H=2, dk=3, dv=2, gate="channel")
    dO = rng.standard_normal(c["v"].shape)
    g1 = oracle.gdr_grads(c["q"], c["k"], c["v"], c["beta"], c["log_alpha"],
                          gate="channel", initial_state=c["initial_state"],
                          d_out=dO)
    bk = np.repeat(c["beta"][..., None], 3, axis=-1)
    g2 = oracle.fg2_grads(c["q"], c["k"], c["v"], bk, None, c["log_alpha"],
                          gate="channel", initial_state=c["initial_state"],
                          d_out=dO)
    for key in ("dq", "dk", "dv", "dlog_alpha", "dinitial_state"):
        np.testing.assert_allclose(g2[key], g1[key], atol=1e-12)
    np.testing.assert_allclose(g2["dbeta_k"].sum(-1), g1["dbeta"], atol=1e-12)


def test_efla_gradients_match_finite_differences():
    """The EFLA autograd gradients (oracle.efla_grads) agree with central
    differences of the EFLA matrix-exponential flow's loss (oracle.efla_fwd),
    element by element, for every input and gate -- unnormalised keys, so
    the step size's dependence on |k| is exercised."""
    rng = np.random.default_rng(61)
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=1, T=4, H=1, dk=3, dv=2, gate=gate)
        case = dict(q=c["q"], k=c["k"] * rng.uniform(0.5, 2.0, (1, 4, 1, 1)),
                    v=c["v"], beta=c["beta"], log_alpha=c["log_alpha"],
                    initial_state=c["initial_state"])
        dO = rng.standard_normal(c["v"].shape)
        dS = rng.standard_normal((1, 1, 3, 2))
        g = oracle.efla_grads(**case, gate=gate, d_out=dO, d_final_state=dS)

        def loss(x):
            o, sT = oracle.efla_fwd(x["q"], x["k"], x["v"], x["beta"],
                                    x["log_alpha"], gate, x["initial_state"])
            return float((o * dO).sum() + (sT * dS).sum())

        names = ["q", "k", "v", "beta", "initial_state"]
        if gate != "none":
            names.append("log_alpha")
        eps = 1e-6
        for key in names:
            x = case[key]
            fd = np.zeros_like(x)
            for i in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[i] += eps
                xm[i] -= eps
                fd[i] = (loss({**case, key: xp}) - loss({**case, key: xm})) / (
                    2 * eps)
            np.testing.assert_allclose(g["d" + key], fd, atol=1e-6, rtol=1e-5,
                                       err_msg=f"{gate} {key}")


def test_gdn2_gradients_reduce_to_the_delta_rule():
    """Both gates equal to beta_t on every channel: the Gated DeltaNet-2
    gradients of q, k, v, log-alpha and the initial state are the delta
    rule's, and the delta rule's d beta_t is the sum of the two gates'
    gradients over their channels (chain rule through b = w = beta 1)."""
    rng = np.random.default_rng(42)
    for gate in ("none", "scalar", "channel"):
        c = _rand_case(rng, B=2, T=6, H=2, dk=4, dv=3, gate=gate)
        dO = rng.standard_normal(c["v"].shape)
        dS = rng.standard_normal((2, 2, 4, 3))
        g1 = oracle.gdr_grads(**c, d_out=dO, d_final_state=dS)
        b = c["beta"]
        g2 = oracle.gdn2_grads(c["q"], c["k"], c["v"],
                               np.repeat(b[..., None], 4, axis=-1),
                               np.repeat(b[..., None], 3, axis=-1),
                               c["log_alpha"], gate, c["initial_state"],
                               d_out=dO, d_final_state=dS)
        for key in ("dq", "dk", "dv", "dlog_alpha", "dinitial_state"):
            if g1[key] is None:
                assert g2[key] is None
            else:
                np.testing.assert_allclose(g2[key], g1[key], atol=1e-12,
                                           err_msg=f"{gate} {key}")
        np.testing.assert_allclose(
            g2["derase"].sum(-1) + g2["dwrite"].sum(-1), g1["dbeta"],
            atol=1e-12, err_msg=gate)


def test_thread_count_does_not_change_bits(oracle_lib):
    rng = np.random.default_rng(10)
    c = _rand_case(rng, B=3, T=15, H=5, dk=4, dv=4, gate="channel")
    o1, s1, n1 = gdr_fwd(**c, nthreads=1)
    o8, s8, n8 = gdr_fwd(**c, nthreads=8)
    assert n1 == 1 and n8 >= 1
    assert np.array_equal(o1, o8) and np.array_equal(s1, s8)


def test_zero_length_and_zero_state(oracle_lib):
    rng = np.random.default_rng(11)
    c = _rand_case(rng, B=1, T=6, H=1, dk=2, dv=2, gate="none", s0=False)
    cu = np.array([0, 0, 6, 6])
    o, s, _ = gdr_fwd(c["q"], c["k"], c["v"], c["beta"], None, gate="none",
                      cu_seqlens=cu)
    assert np.all(s[0] == 0) and np.all(s[2] == 0)
    on, sn, _ = gdr_fwd(**c)
    assert np.array_equal(o, on) and np.array_equal(s[1], sn[0])


def test_bad_arguments_rejected(oracle_lib):
    rng = np.random.default_rng(12)
    c = _rand_case(rng, B=1, T=4, H=1, dk=2, dv=2, gate="none", s0=False)
    with pytest.raises(ValueError):
        gdr_fwd(c["q"], c["k"], c["v"], c["beta"], None, gate="scalar")
    with pytest.raises(ValueError):
        gdr_fwd(c["q"], c["k"], c["v"], c["beta"], None, gate="none",
                cu_seqlens=[0, 3, 2])


# ------------------------------------------- planted mistakes (mutation test)
_MUTANTS = {
    # sign of the residual
    "residual_sign": ("bt * (vt[j] - acc)", "bt * (vt[j] + acc)"),
    # beta applied to v only
    "beta_on_v_only": ("bt * (vt[j] - acc)", "(bt * vt[j] - acc)"),
    # write with q instead of k
    "write_with_q": ("S[c * dv + j] += kt[c] * r[j];",
                     "S[c * dv + j] += qt[c] * r[j];"),
    # read out with k instead of q
    "readout_with_k": ("acc += S[c * dv + j] * qt[c];",
                       "acc += S[c * dv + j] * kt[c];"),
    # decay with the wrong sign of the log
    "decay_sign": ("a[c] = exp(J->log_alpha[(size_t)t * H + h]);",
                   "a[c] = exp(-J->log_alpha[(size_t)t * H + h]);"),
    # channel-wise decay with reversed channel index
    "decay_channel_index": (
        "a[c] = exp(J->log_alpha[((size_t)t * H + h) * dk + c]);",
        "a[c] = exp(J->log_alpha[((size_t)t * H + h) * dk + (dk - 1 - c)]);"),
    # the decay dropped entirely
    "no_decay": ("S[c * dv + j] *= a[c];", "S[c * dv + j] *= 1.0;"),
    # the initial state ignored
    "ignore_s0": ("if (J->s0)\n", "if (0)\n"),
}


def _mutant_sources():
    src = open(oracle._SRC).read()
    out = {name: src.replace(a, b, 1) for name, (a, b) in _MUTANTS.items()}
    # read-out before the write of the current token: move the output loop
    # above the write loop
    w0 = src.index("    /* write S += k u^T */")
    o0 = src.index("    /* output o = S^T q */")
    o1 = src.index("  }\n  if (J->sT)")
    out["read_before_write"] = src[:w0] + src[o0:o1] + src[w0:o0] + src[o1:]
    # decay applied after the erase and the write
    d0 = src.index("    for (int c = 0; c < dk; ++c)\n      for (int j = 0; "
                   "j < dv; ++j) S[c * dv + j] *= a[c];\n")
    d1 = d0 + len("    for (int c = 0; c < dk; ++c)\n      for (int j = 0; "
                  "j < dv; ++j) S[c * dv + j] *= a[c];\n")
    moved = src[:d0] + src[d1:]
    o0m = moved.index("    /* output o = S^T q */")
    out["decay_after_write"] = moved[:o0m] + src[d0:d1] + moved[o0m:]
    for name, s in out.items():
        assert s != src, name
    return out


def test_pins_catch_planted_mistakes(oracle_lib):
    assert run_battery(oracle_lib) == []
    tmp = tempfile.mkdtemp(prefix="oracle_mutants_")
    try:
        for name, s in _mutant_sources().items():
            c_path = os.path.join(tmp, f"{name}.c")
            so_path = os.path.join(tmp, f"{name}.so")
            open(c_path, "w").write(s)
            oracle.build(force=True, src=c_path, out=so_path)
            fails = run_battery(oracle.load(so_path))
            assert fails, f"planted mistake '{name}' passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def test_oracle_builds_with_warnings_clean():
    r = subprocess.run(["gcc", "-O2", "-Wall", "-Wextra", "-fsyntax-only",
                        "-std=c11", oracle._SRC], capture_output=True,
                       text=True)
    assert r.returncode == 0 and "warning" not in r.stderr, r.stderr
