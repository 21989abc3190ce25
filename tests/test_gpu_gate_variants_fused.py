"""GPU parity of the per-channel gate variants on the fused tensor-core path
(bf16, d = 128, C = 64; a scalar or absent decay runs as the channel-wise
one with every channel equal): Gated DeltaNet-2's erase and
write gates (gdr_chunk_fwd_gdn2) and FG^2-GDN's key-side rate with and
without FG^2-GDN+'s value scaling (gdr_chunk_fwd_fg2), against the fp64
token loops oracle.gdn2_fwd and oracle.fg2_fwd.

Tolerance: the bf16 bar of the forward pass, max |gpu - oracle| / RMS(oracle)
<= 2e-2 for out (its own half-ulp rounding discounted, out_err) and for the
final state, element by element, at sizes spanning several chunks and a
ragged tail, and on sampled heads of the full KDA workload."""
import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
import oracle
from chunkwise_recurrence_b200.inputs import (WORKLOADS, fg2_gates,
                                              gdn2_gates, generate, half_ulp,
                                              head_slice, out_err, rel_err)

pytestmark = pytest.mark.gpu

TOL = 2e-2
VARIANTS = ["gdn2", "fg2", "fg2plus"]


def _dev(t):
    return None if t is None else t.cuda()


def _f(t):
    return None if t is None else t.double().numpy()


def _gates(kind, inp, seed):
    if kind == "gdn2":
        return gdn2_gates(inp, seed=seed)
    bk, bv = fg2_gates(inp, seed=seed)
    return bk, (bv if kind == "fg2plus" else None)


def _run_gpu(kind, inp, gk, gv, algo):
    w = inp.w
    fn = gdr.chunk_fwd_gdn2 if kind == "gdn2" else gdr.chunk_fwd_fg2
    o, s = fn(_dev(inp.q), _dev(inp.k), _dev(inp.v), _dev(gk), _dev(gv),
              _dev(inp.log_alpha), _dev(inp.s0), chunk=w.chunk, gate=w.gate,
              cu_seqlens=_dev(inp.cu_seqlens), algo=algo)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    return o.float().cpu().numpy(), s.cpu().numpy()


def _run_oracle(kind, inp, gk, gv):
    fn = oracle.gdn2_fwd if kind == "gdn2" else oracle.fg2_fwd
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    return fn(_f(inp.q), _f(inp.k), _f(inp.v), _f(gk), _f(gv),
              _f(inp.log_alpha), inp.w.gate, _f(inp.s0), cu)


@pytest.mark.parametrize("kind", VARIANTS)
@pytest.mark.parametrize("name,shape", [
    ("kda_b4_h16_t4096_d128_bf16", dict(B=2, T=3 * 64 + 37, H=2)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=64, H=3, init_state=True)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=3, T=5, H=1)),
])
def test_fused_gate_variants_match_oracle(kind, name, shape):
    w = WORKLOADS[name].with_(**shape)
    inp = generate(w, seed=61)
    gk, gv = _gates(kind, inp, 61)
    o, s = _run_gpu(kind, inp, gk, gv, "fused_tc")
    ro, rs = _run_oracle(kind, inp, gk, gv)
    assert out_err(o, ro, "bf16") <= TOL
    assert rel_err(s, rs) <= TOL


@pytest.mark.parametrize("kind", VARIANTS)
def test_fused_gate_variants_varlen(kind):
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        H=2, varlen_nseq=5, varlen_lo=1, varlen_hi=200, gate="channel")
    inp = generate(w, seed=62)
    gk, gv = _gates(kind, inp, 62)
    o, s = _run_gpu(kind, inp, gk, gv, "fused_tc")
    ro, rs = _run_oracle(kind, inp, gk, gv)
    assert out_err(o, ro, "bf16") <= TOL
    assert rel_err(s, rs) <= TOL


@pytest.mark.parametrize("kind", VARIANTS)
def test_fused_gate_variants_full_kda_workload_sampled_heads(kind):
    """The whole KDA workload (B4 H16 T4096) through the fused kernel; two
    heads of every sequence checked against the oracle element by element."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"]
    inp = generate(w, seed=0)
    gk, gv = _gates(kind, inp, 0)
    o, s = _run_gpu(kind, inp, gk, gv, "fused_tc")
    heads = [3, 12]
    sub = head_slice(inp, heads)
    hs = torch.tensor(heads)
    pick = lambda t: None if t is None else t.index_select(2, hs)  # noqa
    ro, rs = _run_oracle(kind, sub, pick(gk), pick(gv))
    assert out_err(o[:, :, heads], ro, "bf16") <= TOL
    assert rel_err(s[:, heads], rs) <= TOL


@pytest.mark.parametrize("gate", ["channel", "scalar", "none"])
@pytest.mark.parametrize("kind", VARIANTS)
def test_auto_takes_the_fused_path(kind, gate):
    """AUTO gives the fused kernel's bits for bf16, d = 128, C = 64 with every
    decay form (a scalar or absent decay as the channel-wise one with all
    channels equal), within the bar of the oracle."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=100, H=2,
                                                       gate=gate)
    inp = generate(w, seed=63)
    gk, gv = _gates(kind, inp, 63)
    oa, sa = _run_gpu(kind, inp, gk, gv, "auto")
    of, sf = _run_gpu(kind, inp, gk, gv, "fused_tc")
    os_, ss = _run_gpu(kind, inp, gk, gv, "staged")
    assert np.array_equal(oa, of) and np.array_equal(sa, sf)
    assert not np.array_equal(sa, ss)
    ro, rs = _run_oracle(kind, inp, gk, gv)
    assert out_err(oa, ro, "bf16") <= TOL
    assert rel_err(sa, rs) <= TOL


def test_fused_gdn2_with_gates_equal_to_beta_is_the_fused_kda_pass():
    """b_t = w_t = beta_t on every channel: Gated DeltaNet-2 is KDA, and the
    two fused runs agree to the fused path's own accuracy."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=150, H=2)
    inp = generate(w, seed=64)
    erase = inp.beta[..., None].expand(inp.k.shape).contiguous()
    write = inp.beta[..., None].expand(inp.v.shape).contiguous()
    o2, s2 = _run_gpu("gdn2", inp, erase, write, "fused_tc")
    o1, s1 = gdr.chunk_fwd(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                           _dev(inp.beta), _dev(inp.log_alpha), _dev(inp.s0),
                           gate=w.gate, algo="fused_tc")
    torch.cuda.synchronize()
    assert rel_err(s2, s1.cpu().numpy()) <= 5e-3
    # both outputs are rounded to bf16, each by up to half an ulp: the two
    # roundings are discounted before the difference is measured
    o1 = o1.float().cpu().numpy()
    u = half_ulp(np.maximum(np.abs(o1), np.abs(o2)), "bf16")
    d = np.maximum(np.abs(o2 - o1) - 2 * u, 0.0)
    assert d.max() / np.sqrt(np.mean(o1.astype(np.float64) ** 2)) <= 5e-3
