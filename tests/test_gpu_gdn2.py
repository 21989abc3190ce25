"""GPU parity of the Gated DeltaNet-2 gates (gdr_chunk_fwd_gdn2, through the
C ABI, staged path) against the fp64 token loop of oracle.gdn2_fwd.

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


def test_gdn2_fused_algo_is_unsupported():
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=1, T=64, H=1)
    inp = generate(w, seed=44)
    erase, write = gdn2_gates(inp, seed=44)
    with pytest.raises(gdr.GdrError):
        gdr.chunk_fwd_gdn2(_dev(inp.q), _dev(inp.k), _dev(inp.v), _dev(erase),
                           _dev(write), _dev(inp.log_alpha), algo="fused_tc",
                           gate=w.gate)
