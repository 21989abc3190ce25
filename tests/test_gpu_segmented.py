"""GPU parity of the context-parallel forward pass (gdr_chunk_fwd_segmented,
through the C ABI) against the fp64 token-loop oracle: every sequence cut
into pieces whose state maps (M, N) are computed in parallel, combined in
order, then re-run from their true initial states.

Tolerance as for gdr_chunk_fwd: max |gpu - oracle| / RMS(oracle) <= 1e-4 for
fp32 inputs, <= 2e-2 for bf16 inputs (out after the half-ulp discount)."""
import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
from chunkwise_recurrence_b200.inputs import (WORKLOADS, generate, head_slice,
                                              out_err, rel_err)
from oracle import gdr_fwd

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _run(inp, segments, chunk=None, final=True):
    w = inp.w
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    out, sT = gdr.chunk_fwd_segmented(
        c(inp.q), c(inp.k), c(inp.v), c(inp.beta), c(inp.log_alpha),
        c(inp.s0), segments=segments, chunk=chunk or w.chunk, gate=w.gate,
        cu_seqlens=c(inp.cu_seqlens), output_final_state=final)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    return out.float().cpu().numpy(), (None if sT is None else
                                       sT.cpu().numpy())


def _check(inp, segments, chunk=None):
    o, s = _run(inp, segments, chunk)
    ro, rs, _ = gdr_fwd(**inp.f64())
    tol = TOL[inp.w.dtype]
    eo, es = out_err(o, ro, inp.w.dtype), rel_err(s, rs)
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


@pytest.mark.parametrize("segments", [1, 3, 8])
def test_segmented_gdn_fused(segments):
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=1000, H=2)
    _check(generate(w, seed=1), segments)


def test_segmented_kda_fused():
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=500, H=2)
    _check(generate(w, seed=2), 4)


@pytest.mark.parametrize("segments", [2, 5])
def test_segmented_fp32_staged(segments):
    w = WORKLOADS["deltanet_b1_h1_t256_d16_fp32"].with_(B=2, T=300, H=2)
    _check(generate(w, seed=3), segments)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 32)])
def test_segmented_rectangular_state(dk, dv):
    w = WORKLOADS["gdn_b4_h8_t2048_d128_bf16"].with_(B=2, T=333, H=2, dk=dk,
                                                     dv=dv, init_state=True)
    _check(generate(w, seed=4), 3)


def test_segmented_varlen_with_empty_and_short_sequences():
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        varlen_nseq=5, varlen_lo=0, varlen_hi=400, H=2)
    inp = generate(w, seed=7)
    # force an empty and a very short sequence into the batch
    lengths = [0, 37, 300, 5, 129]
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    tot = int(cu[-1])
    cut = lambda t: None if t is None else t[:, :tot].contiguous()  # noqa
    inp = type(inp)(w=w, q=cut(inp.q), k=cut(inp.k), v=cut(inp.v),
                    beta=cut(inp.beta), log_alpha=cut(inp.log_alpha),
                    s0=inp.s0, cu_seqlens=cu, lengths=lengths)
    _check(inp, 3)


def test_segmented_without_final_state_and_equal_to_sequential():
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=640, H=2)
    inp = generate(w, seed=8)
    o_seg, s_none = _run(inp, 4, final=False)
    assert s_none is None
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    o_seq, _ = gdr.chunk_fwd(c(inp.q), c(inp.k), c(inp.v), c(inp.beta),
                             c(inp.log_alpha), c(inp.s0), chunk=w.chunk,
                             gate=w.gate)
    # both match the oracle; against each other they differ only by the
    # rounding of the segment maps
    ro, _, _ = gdr_fwd(**inp.f64())
    assert out_err(o_seg, ro, "bf16") <= 2e-2
    assert rel_err(o_seg, o_seq.float().cpu().numpy()) <= 4e-2


def test_segmented_long_context_sampled_heads():
    """One 16 K-token sequence x 16 heads, cut into 8 pieces (the case the
    entry exists for: fewer chains than SMs); heads 0 and 15 are compared with
    the oracle in full."""
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=16384)
    inp = generate(w, seed=9)
    o, s = _run(inp, 8)
    sub = head_slice(inp, [0, 15])
    ro, rs, _ = gdr_fwd(**sub.f64())
    assert out_err(o[:, :, [0, 15]], ro, "bf16") <= 2e-2
    assert rel_err(s[:, [0, 15]], rs) <= 2e-2
