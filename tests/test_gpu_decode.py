"""GPU parity of the single-token decode step (gdr_decode_step, through the C
ABI) against the fp64 CPU oracle's one-token step.

Tolerance: the decode kernel computes in fp32 with no operand rounding, so the
error is that of fp32 dot products of length dk, well under 1e-5 of the RMS;
the bar is max |gpu - oracle| / RMS(oracle) <= 1e-4 for the state and for the
output, whose half-ulp rounding to its storage dtype is discounted first
(``out_err``), as for the chunked forward pass.
"""
import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
import oracle
from chunkwise_recurrence_b200.inputs import (WORKLOADS, Workload, generate,
                                              out_err, rel_err)

pytestmark = pytest.mark.gpu

TOL = 1e-4


def decode_inputs(N, H, dk, dv, dtype, gate, seed=0, init_state=True):
    """One token per sequence, drawn like the chunked workloads' tokens."""
    w = Workload("decode", B=N, T=1, H=H, dk=dk, dv=dv, chunk=16, dtype=dtype,
                 gate=gate, decay_lo=0.01, decay_hi=0.1, init_state=init_state)
    inp = generate(w, seed=seed)
    sq = lambda t: None if t is None else t[:, 0].contiguous()  # noqa: E731
    return dict(q=sq(inp.q), k=sq(inp.k), v=sq(inp.v), beta=sq(inp.beta),
                log_alpha=sq(inp.log_alpha), state=inp.s0)


def run_gpu(d, in_place=True):
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    state = c(d["state"])
    out, s1 = gdr.decode_step(c(d["q"]), c(d["k"]), c(d["v"]), c(d["beta"]),
                              c(d["log_alpha"]), state,
                              state_out=None if in_place else torch.empty(
                                  d["q"].shape[0], d["q"].shape[1],
                                  d["q"].shape[2], d["v"].shape[2],
                                  device="cuda"))
    torch.cuda.synchronize()
    if in_place and state is not None:
        assert s1.data_ptr() == state.data_ptr()
    return out.float().cpu().numpy(), s1.cpu().numpy()


def run_oracle(d, gate):
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    return oracle.decode_step(f(d["q"]), f(d["k"]), f(d["v"]), f(d["beta"]),
                              f(d["log_alpha"]), gate=gate,
                              state=f(d["state"]))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 128), (128, 64),
                                   (128, 128)])
def test_decode_matches_oracle(dtype, gate, dk, dv):
    d = decode_inputs(3, 5, dk, dv, dtype, gate)
    o, s = run_gpu(d)
    ro, rs = run_oracle(d, gate)
    assert out_err(o, ro, dtype) <= TOL
    assert rel_err(s, rs) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_decode_zero_state_and_out_of_place(gate):
    d = decode_inputs(4, 3, 128, 128, "bf16", gate, init_state=False)
    o, s = run_gpu(d, in_place=False)
    ro, rs = run_oracle(d, gate)
    assert out_err(o, ro, "bf16") <= TOL and rel_err(s, rs) <= TOL
    # in place and out of place give the same bits
    d = decode_inputs(4, 3, 128, 128, "bf16", gate)
    o1, s1 = run_gpu(d, in_place=True)
    o2, s2 = run_gpu(d, in_place=False)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


@pytest.mark.parametrize("name", ["gdn_b8_h16_t4096_d128_bf16",
                                  "kda_b4_h16_t4096_d128_bf16",
                                  "deltanet_b1_h1_t256_d16_fp32"])
def test_decode_steps_continue_a_sequence(name):
    """Prefill with the chunked forward pass, then decode token by token:
    every decoded output and the final state match the oracle's token loop
    over the whole sequence (the decode step continues the recurrence)."""
    w = WORKLOADS[name]
    T, Td = 96, 24
    w = w.with_(B=min(w.B, 2), T=T + Td, H=min(w.H, 3))
    inp = generate(w, seed=3)
    ro, rs, _ = oracle.gdr_fwd(**inp.f64())
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    pre = lambda t: None if t is None else t[:, :T].contiguous()  # noqa: E731
    _, state = gdr.chunk_fwd(c(pre(inp.q)), c(pre(inp.k)), c(pre(inp.v)),
                             c(pre(inp.beta)), c(pre(inp.log_alpha)),
                             c(inp.s0), chunk=w.chunk, gate=w.gate)
    outs = []
    for t in range(T, T + Td):
        tok = lambda x: None if x is None else x[:, t].contiguous()  # noqa
        o, state = gdr.decode_step(c(tok(inp.q)), c(tok(inp.k)),
                                   c(tok(inp.v)), c(tok(inp.beta)),
                                   c(tok(inp.log_alpha)), state, gate=w.gate)
        outs.append(o.float().cpu().numpy())
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    tol = 1e-4 if w.dtype == "fp32" else 2e-2
    o = np.stack(outs, axis=1)
    assert out_err(o, ro[:, T:], w.dtype) <= tol
    assert rel_err(state.cpu().numpy(), rs) <= tol


def test_decode_full_size_sampled():
    """The decode benchmark's shape (256 sequences x 16 heads, d = 128, bf16,
    scalar gate, state N(0, 0.02^2)), run in full on the GPU; sequences 0..7
    (all heads) are compared with the oracle -- every (sequence, head) step is
    an independent sub-problem."""
    d = decode_inputs(256, 16, 128, 128, "bf16", "scalar")
    o, s = run_gpu(d)
    sub = {k: (None if v is None else v[:8]) for k, v in d.items()}
    ro, rs = run_oracle(sub, "scalar")
    assert out_err(o[:8], ro, "bf16") <= TOL
    assert rel_err(s[:8], rs) <= TOL
    assert np.isfinite(o).all() and np.isfinite(s).all()


def test_decode_wait_timeout_is_reported_and_recovers(monkeypatch):
    """Failure detection on the GPU without a fault: with the injection hook
    set, the decode kernel never issues its state copy, so each CTA's bounded
    wait runs out (after about 10^6 cycles); the CTA skips its step and the
    host reads GDR_ERR_TIMEOUT.  The state is left untouched, the context
    stays usable, and the next call is correct."""
    d = decode_inputs(4, 2, 128, 128, "bf16", "scalar")
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    state = c(d["state"])
    before = state.clone()
    monkeypatch.setenv("GDR_FAULT_INJECT_DECODE_TIMEOUT", "1")
    gdr.decode_step(c(d["q"]), c(d["k"]), c(d["v"]), c(d["beta"]),
                    c(d["log_alpha"]), state)
    assert gdr.device_error(clear=True) == 5          # GDR_ERR_TIMEOUT
    assert torch.equal(state, before)
    assert gdr.device_error() == 0                    # cleared
    monkeypatch.delenv("GDR_FAULT_INJECT_DECODE_TIMEOUT")
    o, s = run_gpu(d)
    assert gdr.device_error() == 0
    ro, rs = run_oracle(d, "scalar")
    assert out_err(o, ro, "bf16") <= TOL and rel_err(s, rs) <= TOL
