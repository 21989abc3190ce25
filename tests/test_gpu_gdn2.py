"""GPU parity of the Gated DeltaNet-2 gates (gdr_chunk_fwd_gdn2 on the staged
path and gdr_decode_step_gdn2, through the C ABI) against the fp64 token loop
of oracle.gdn2_fwd.

Tolerance: the bars of the forward pass, max |gpu - oracle| / RMS(oracle)
<= 1e-4 for fp32 inputs and <= 2e-2 for bf16 inputs (with the output's own
half-ulp rounding discounted, out_err), for out and final_state; the staged
path computes in fp32, so both sit far below them."""
import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
import oracle
from chunkwise_recurrence_b200.inputs import (WORKLOADS, gdn2_gates, generate,
                                              out_err, rel_err)

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _dev(t):
    return None if t is None else t.cuda()


def run_both(inp, erase, write):
    w = inp.w
    o, s = gdr.chunk_fwd_gdn2(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                              _dev(erase), _dev(write), _dev(inp.log_alpha),
                              _dev(inp.s0), chunk=w.chunk, gate=w.gate,
                              cu_seqlens=_dev(inp.cu_seqlens))
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    ro, rs = oracle.gdn2_fwd(f(inp.q), f(inp.k), f(inp.v), f(erase), f(write),
                             f(inp.log_alpha), w.gate, f(inp.s0),
                             None if inp.cu_seqlens is None
                             else inp.cu_seqlens.numpy())
    return o.float().cpu().numpy(), s.cpu().numpy(), ro, rs


@pytest.mark.parametrize("name,shape", [
    ("kda_b4_h16_t4096_d128_bf16", dict(B=2, T=2 * 64 + 37, H=2)),
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=2, T=64 + 11, H=2, init_state=True)),
    ("deltanet_b1_h1_t256_d16_fp32", dict(B=2, T=70, H=2)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=90, H=2, dk=64, dv=32,
                                        dtype="fp32", init_state=True)),
])
def test_gdn2_matches_oracle(name, shape):
    w = WORKLOADS[name].with_(**shape)
    inp = generate(w, seed=41)
    erase, write = gdn2_gates(inp, seed=41)
    o, s, ro, rs = run_both(inp, erase, write)
    assert out_err(o, ro, w.dtype) <= TOL[w.dtype]
    assert rel_err(s, rs) <= TOL[w.dtype]


def test_gdn2_varlen():
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        H=2, varlen_nseq=4, varlen_lo=1, varlen_hi=150, gate="channel")
    inp = generate(w, seed=42)
    erase, write = gdn2_gates(inp, seed=42)
    o, s, ro, rs = run_both(inp, erase, write)
    assert out_err(o, ro, "bf16") <= TOL["bf16"]
    assert rel_err(s, rs) <= TOL["bf16"]


def test_gdn2_with_gates_equal_to_beta_is_the_delta_rule():
    """b_t = w_t = beta_t on every channel: the same recurrence as
    gdr_chunk_fwd, so the two staged runs agree to fp32 rounding (fp32
    inputs and outputs, so that no output rounding step can separate them)."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=100, H=2,
                                                       dtype="fp32")
    inp = generate(w, seed=43)
    erase = inp.beta[..., None].expand(inp.k.shape).contiguous()
    write = inp.beta[..., None].expand(inp.v.shape).contiguous()
    o2, s2 = gdr.chunk_fwd_gdn2(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                                _dev(erase), _dev(write), _dev(inp.log_alpha),
                                _dev(inp.s0), gate=w.gate)
    o1, s1 = gdr.chunk_fwd(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                           _dev(inp.beta), _dev(inp.log_alpha), _dev(inp.s0),
                           gate=w.gate, algo="staged")
    torch.cuda.synchronize()
    assert rel_err(s2.cpu().numpy(), s1.cpu().numpy()) <= 1e-5
    assert rel_err(o2.cpu().numpy(), o1.cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("gate", ["scalar", "none"])
def test_gdn2_fused_with_a_scalar_or_no_decay(gate):
    """The fused kernel takes the gates with a scalar or absent decay as the
    channel-wise decay with every channel equal."""
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=2, T=2 * 64 + 19, H=2,
                                                       gate=gate)
    inp = generate(w, seed=44)
    erase, write = gdn2_gates(inp, seed=44)
    o, s = gdr.chunk_fwd_gdn2(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                              _dev(erase), _dev(write), _dev(inp.log_alpha),
                              _dev(inp.s0), algo="fused_tc", gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    ro, rs = oracle.gdn2_fwd(f(inp.q), f(inp.k), f(inp.v), f(erase), f(write),
                             f(inp.log_alpha), gate, f(inp.s0))
    assert out_err(o.float().cpu().numpy(), ro, "bf16") <= TOL["bf16"]
    assert rel_err(s.cpu().numpy(), rs) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# gdr_decode_step_gdn2: one token per (sequence, head).  The kernel is the
# decode step's (fp32 arithmetic, no operand rounding), so the bar is that of
# the decode tests: 1e-4 of the RMS for the state and for the output (its
# storage rounding discounted).

DECODE_TOL = 1e-4


def decode_gdn2_inputs(N, H, dk, dv, dtype, gate, seed, init_state=True):
    from chunkwise_recurrence_b200.inputs import Workload
    w = Workload("decode", B=N, T=1, H=H, dk=dk, dv=dv, chunk=16, dtype=dtype,
                 gate=gate, decay_lo=0.01, decay_hi=0.1, init_state=init_state)
    inp = generate(w, seed=seed)
    erase, write = gdn2_gates(inp, seed=seed)
    return inp, erase, write


def decode_gdn2_gpu(inp, erase, write, state=None):
    sq = lambda t: None if t is None else t[:, 0].contiguous().cuda()  # noqa
    st = None if state is None else state.clone().cuda()
    out, s1 = gdr.decode_step_gdn2(sq(inp.q), sq(inp.k), sq(inp.v), sq(erase),
                                   sq(write), sq(inp.log_alpha), st,
                                   gate=inp.w.gate)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    return out.float().cpu().numpy(), s1.cpu().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("dk,dv", [(16, 32), (64, 128), (128, 128)])
def test_decode_gdn2_matches_oracle(dtype, gate, dk, dv):
    inp, erase, write = decode_gdn2_inputs(3, 5, dk, dv, dtype, gate, seed=45)
    o, s = decode_gdn2_gpu(inp, erase, write, inp.s0)
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    ro, rs = oracle.gdn2_fwd(f(inp.q), f(inp.k), f(inp.v), f(erase), f(write),
                             f(inp.log_alpha), gate, f(inp.s0))
    assert out_err(o, ro[:, 0], dtype) <= DECODE_TOL
    assert rel_err(s, rs) <= DECODE_TOL


def test_decode_gdn2_zero_state():
    inp, erase, write = decode_gdn2_inputs(4, 3, 128, 128, "bf16", "channel",
                                           seed=46, init_state=False)
    o, s = decode_gdn2_gpu(inp, erase, write, None)
    f = lambda t: t.double().numpy()  # noqa: E731
    ro, rs = oracle.gdn2_fwd(f(inp.q), f(inp.k), f(inp.v), f(erase), f(write),
                             f(inp.log_alpha), "channel")
    assert out_err(o, ro[:, 0], "bf16") <= DECODE_TOL
    assert rel_err(s, rs) <= DECODE_TOL


def test_prefill_then_decode_gdn2_continues_the_sequence():
    """A prompt through gdr_chunk_fwd_gdn2, then its last tokens one at a
    time through gdr_decode_step_gdn2 on the resulting state, matches the
    oracle's token loop over the whole sequence."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=64 + 23 + 3, H=2)
    inp = generate(w, seed=47)
    erase, write = gdn2_gates(inp, seed=47)
    P = 64 + 23
    c = lambda t: None if t is None else t[:, :P].contiguous().cuda()  # noqa
    _, state = gdr.chunk_fwd_gdn2(c(inp.q), c(inp.k), c(inp.v), c(erase),
                                  c(write), c(inp.log_alpha), gate=w.gate)
    outs = []
    for t in range(P, w.T):
        s1 = lambda x: x[:, t].contiguous().cuda()  # noqa: E731
        o, state = gdr.decode_step_gdn2(s1(inp.q), s1(inp.k), s1(inp.v),
                                        s1(erase), s1(write),
                                        s1(inp.log_alpha), state, gate=w.gate)
        outs.append(o.float().cpu().numpy())
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    ro, rs = oracle.gdn2_fwd(f(inp.q), f(inp.k), f(inp.v), f(erase), f(write),
                             f(inp.log_alpha), w.gate)
    assert out_err(np.stack(outs, 1), ro[:, P:], "bf16") <= TOL["bf16"]
    assert rel_err(state.cpu().numpy(), rs) <= TOL["bf16"]


def test_decode_gdn2_with_gates_equal_to_beta_is_the_decode_step():
    inp, _, _ = decode_gdn2_inputs(3, 4, 128, 64, "fp32", "scalar", seed=48)
    erase = inp.beta[..., None].expand(inp.k.shape).contiguous()
    write = inp.beta[..., None].expand(inp.v.shape).contiguous()
    o2, s2 = decode_gdn2_gpu(inp, erase, write, inp.s0)
    sq = lambda t: t[:, 0].contiguous().cuda()  # noqa: E731
    o1, s1 = gdr.decode_step(sq(inp.q), sq(inp.k), sq(inp.v), sq(inp.beta),
                             sq(inp.log_alpha), inp.s0.clone().cuda())
    torch.cuda.synchronize()
    assert rel_err(s2, s1.cpu().numpy()) <= 1e-5
    assert rel_err(o2, o1.float().cpu().numpy()) <= 1e-5
