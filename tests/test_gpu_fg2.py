"""GPU parity of FG^2-GDN's channel-wise learning rate (gdr_chunk_fwd_fg2 on
the staged path and gdr_decode_step_fg2, through the C ABI) against the fp64
token loop of oracle.fg2_fwd, for FG^2-GDN (no value scaling) and FG^2-GDN+
(a per-value-channel target scaling).

Tolerance: the bars of the forward pass, max |gpu - oracle| / RMS(oracle)
<= 1e-4 for fp32 inputs and <= 2e-2 for bf16 inputs (with the output's own
half-ulp rounding discounted, out_err), for out and final_state; the staged
path computes in fp32, so both sit far below them.  The decode step is fp32
throughout and is held to 1e-4."""
import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
import oracle
from chunkwise_recurrence_b200.inputs import (WORKLOADS, Workload, fg2_gates,
                                              generate, out_err, rel_err)

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}
DECODE_TOL = 1e-4


def _dev(t):
    return None if t is None else t.cuda()


def _f(t):
    return None if t is None else t.double().numpy()


def run_both(inp, beta_k, beta_v):
    w = inp.w
    o, s = gdr.chunk_fwd_fg2(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                             _dev(beta_k), _dev(beta_v), _dev(inp.log_alpha),
                             _dev(inp.s0), chunk=w.chunk, gate=w.gate,
                             cu_seqlens=_dev(inp.cu_seqlens))
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    ro, rs = oracle.fg2_fwd(_f(inp.q), _f(inp.k), _f(inp.v), _f(beta_k),
                            _f(beta_v), _f(inp.log_alpha), w.gate, _f(inp.s0),
                            None if inp.cu_seqlens is None
                            else inp.cu_seqlens.numpy())
    return o.float().cpu().numpy(), s.cpu().numpy(), ro, rs


@pytest.mark.parametrize("plus", [False, True])
@pytest.mark.parametrize("name,shape", [
    ("kda_b4_h16_t4096_d128_bf16", dict(B=2, T=2 * 64 + 37, H=2)),
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=2, T=64 + 11, H=2, init_state=True)),
    ("deltanet_b1_h1_t256_d16_fp32", dict(B=2, T=70, H=2)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=90, H=2, dk=64, dv=32,
                                        dtype="fp32", init_state=True)),
])
def test_fg2_matches_oracle(name, shape, plus):
    w = WORKLOADS[name].with_(**shape)
    inp = generate(w, seed=51)
    beta_k, beta_v = fg2_gates(inp, seed=51)
    o, s, ro, rs = run_both(inp, beta_k, beta_v if plus else None)
    assert out_err(o, ro, w.dtype) <= TOL[w.dtype]
    assert rel_err(s, rs) <= TOL[w.dtype]


def test_fg2_varlen():
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        H=2, varlen_nseq=4, varlen_lo=1, varlen_hi=150, gate="channel")
    inp = generate(w, seed=52)
    beta_k, beta_v = fg2_gates(inp, seed=52)
    o, s, ro, rs = run_both(inp, beta_k, beta_v)
    assert out_err(o, ro, "bf16") <= TOL["bf16"]
    assert rel_err(s, rs) <= TOL["bf16"]


def test_fg2_headline_shape_sampled_heads():
    """One full-length sequence of the headline shape (T = 4096, d = 128,
    bf16) on two heads: 64 chunks of state passing under the channel-wise
    rate."""
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, H=2)
    inp = generate(w, seed=53)
    beta_k, beta_v = fg2_gates(inp, seed=53)
    o, s, ro, rs = run_both(inp, beta_k, beta_v)
    assert out_err(o, ro, "bf16") <= TOL["bf16"]
    assert rel_err(s, rs) <= TOL["bf16"]


def test_fg2_with_a_uniform_rate_is_the_delta_rule():
    """beta_k = beta_t on every channel, no value scaling: the same
    recurrence as gdr_chunk_fwd, so the two staged runs agree to fp32
    rounding (fp32 inputs and outputs)."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=100, H=2,
                                                       dtype="fp32")
    inp = generate(w, seed=54)
    beta_k = inp.beta[..., None].expand(inp.k.shape).contiguous()
    o2, s2 = gdr.chunk_fwd_fg2(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                               _dev(beta_k), None, _dev(inp.log_alpha),
                               _dev(inp.s0), gate=w.gate)
    o1, s1 = gdr.chunk_fwd(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                           _dev(inp.beta), _dev(inp.log_alpha), _dev(inp.s0),
                           gate=w.gate, algo="staged")
    torch.cuda.synchronize()
    assert rel_err(s2.cpu().numpy(), s1.cpu().numpy()) <= 1e-5
    assert rel_err(o2.cpu().numpy(), o1.cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("gate", ["scalar", "none"])
def test_fg2_fused_with_a_scalar_or_no_decay(gate):
    """The fused kernel takes the rate with a scalar or absent decay as the
    channel-wise decay with every channel equal."""
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=2, T=2 * 64 + 19, H=2,
                                                       gate=gate)
    inp = generate(w, seed=55)
    beta_k, beta_v = fg2_gates(inp, seed=55)
    o, s = gdr.chunk_fwd_fg2(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                             _dev(beta_k), _dev(beta_v), _dev(inp.log_alpha),
                             _dev(inp.s0), algo="fused_tc", gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    ro, rs = oracle.fg2_fwd(_f(inp.q), _f(inp.k), _f(inp.v), _f(beta_k),
                            _f(beta_v), _f(inp.log_alpha), gate, _f(inp.s0))
    assert out_err(o.float().cpu().numpy(), ro, "bf16") <= TOL["bf16"]
    assert rel_err(s.cpu().numpy(), rs) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# gdr_decode_step_fg2: one token per (sequence, head).

def decode_fg2_inputs(N, H, dk, dv, dtype, gate, seed, init_state=True):
    w = Workload("decode", B=N, T=1, H=H, dk=dk, dv=dv, chunk=16, dtype=dtype,
                 gate=gate, decay_lo=0.01, decay_hi=0.1, init_state=init_state)
    inp = generate(w, seed=seed)
    beta_k, beta_v = fg2_gates(inp, seed=seed)
    return inp, beta_k, beta_v


def decode_fg2_gpu(inp, beta_k, beta_v, state=None):
    sq = lambda t: None if t is None else t[:, 0].contiguous().cuda()  # noqa
    st = None if state is None else state.clone().cuda()
    out, s1 = gdr.decode_step_fg2(sq(inp.q), sq(inp.k), sq(inp.v), sq(beta_k),
                                  sq(beta_v), sq(inp.log_alpha), st,
                                  gate=inp.w.gate)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    return out.float().cpu().numpy(), s1.cpu().numpy()


@pytest.mark.parametrize("plus", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("dk,dv", [(16, 32), (128, 128)])
def test_decode_fg2_matches_oracle(dtype, gate, dk, dv, plus):
    inp, beta_k, beta_v = decode_fg2_inputs(3, 5, dk, dv, dtype, gate,
                                            seed=56)
    bv = beta_v if plus else None
    o, s = decode_fg2_gpu(inp, beta_k, bv, inp.s0)
    ro, rs = oracle.fg2_fwd(_f(inp.q), _f(inp.k), _f(inp.v), _f(beta_k),
                            _f(bv), _f(inp.log_alpha), gate, _f(inp.s0))
    assert out_err(o, ro[:, 0], dtype) <= DECODE_TOL
    assert rel_err(s, rs) <= DECODE_TOL


def test_prefill_then_decode_fg2_continues_the_sequence():
    """A prompt through gdr_chunk_fwd_fg2, then its last tokens one at a time
    through gdr_decode_step_fg2 on the resulting state, matches the oracle's
    token loop over the whole sequence."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=64 + 23 + 3, H=2)
    inp = generate(w, seed=57)
    beta_k, beta_v = fg2_gates(inp, seed=57)
    P = 64 + 23
    c = lambda t: None if t is None else t[:, :P].contiguous().cuda()  # noqa
    _, state = gdr.chunk_fwd_fg2(c(inp.q), c(inp.k), c(inp.v), c(beta_k),
                                 c(beta_v), c(inp.log_alpha), None,
                                 gate=w.gate)
    outs = []
    for t in range(P, w.T):
        s = lambda x: x[:, t].contiguous().cuda()  # noqa: E731
        o, state = gdr.decode_step_fg2(s(inp.q), s(inp.k), s(inp.v),
                                       s(beta_k), s(beta_v),
                                       s(inp.log_alpha), state, gate=w.gate)
        outs.append(o.float().cpu().numpy())
    torch.cuda.synchronize()
    ro, rs = oracle.fg2_fwd(_f(inp.q), _f(inp.k), _f(inp.v), _f(beta_k),
                            _f(beta_v), _f(inp.log_alpha), w.gate)
    o = np.stack(outs, axis=1)
    assert out_err(o, ro[:, P:], "bf16") <= TOL["bf16"]
    assert rel_err(state.cpu().numpy(), rs) <= TOL["bf16"]
