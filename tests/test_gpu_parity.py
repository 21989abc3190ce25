"""GPU parity: libgdr (through its C ABI) against the fp64 CPU oracle.

Tolerance (the parity bar): max |gpu - oracle| / RMS(oracle) over the whole
tensor, for `out` and `final_state` separately: <= 1e-4 for fp32 inputs,
<= 2e-2 for bf16 inputs.  The oracle runs on the device-rounded inputs, so
only the GPU's arithmetic is measured.  `out` is written in the input dtype and
must be rounded to it: for bf16 that rounding alone is up to 2^-8 max|o|, above
2e-2 RMS once max|o| > 5.1 RMS (the 1.3B-layer workload has max|o| = 7.6 RMS).
So the metric of `out` discounts, per element, half an ulp of the output dtype
(`out_err`); `final_state` is fp32 and uses the plain metric.

Small cases span several chunks and a ragged tail and are compared element by
element; the full-size workloads run on the GPU in full and are compared on
sampled heads (every (sequence, head) chain is independent, so a sampled head
is an exact sub-problem for the oracle).
"""
import dataclasses

import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
from chunkwise_recurrence_b200.inputs import (WORKLOADS, generate, head_slice,
                                              out_err, rel_err)
from oracle import gdr_fwd

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _dev(t):
    return None if t is None else t.cuda()


def run_gpu(inp, algo="auto", chunk=None):
    w = inp.w
    out, sT = gdr.chunk_fwd(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                            _dev(inp.beta), _dev(inp.log_alpha),
                            _dev(inp.s0), chunk=chunk or w.chunk, gate=w.gate,
                            cu_seqlens=_dev(inp.cu_seqlens), algo=algo)
    assert gdr.device_error() == 0
    return out.float().cpu().numpy(), sT.cpu().numpy()


def run_oracle(inp):
    out, sT, _ = gdr_fwd(**inp.f64())
    return out, sT


def check(inp, algo="auto", chunk=None):
    o, s = run_gpu(inp, algo, chunk)
    ro, rs = run_oracle(inp)
    tol = TOL[inp.w.dtype]
    eo, es = out_err(o, ro, inp.w.dtype), rel_err(s, rs)
    assert np.isfinite(o).all() and np.isfinite(s).all()
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


def algos_for(w):
    """Every kernel path that serves this workload's dtype, gate and shape."""
    return [a for a in ("staged", "fused_tc")
            if gdr.algo_applies(a, w.dtype, w.gate, w.dk, w.dv, w.chunk)]


# ---- small versions of every workload (same distributions), several chunks
# ---- plus a ragged tail
SMALL = {
    "deltanet_b1_h1_t256_d16_fp32": dict(),                    # full size
    "gdn_b4_h8_t2048_d128_bf16": dict(B=2, T=3 * 64 + 37, H=3),
    "gdn_b8_h16_t4096_d128_bf16": dict(B=2, T=5 * 64 + 1, H=2),
    "kda_b4_h16_t4096_d128_bf16": dict(B=2, T=4 * 64 + 63, H=2),
    "gdn_varlen8_h16_d128_bf16": dict(H=2, varlen_nseq=5, varlen_lo=1,
                                      varlen_hi=300),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_workloads(name):
    w = WORKLOADS[name].with_(**SMALL[name])
    inp = generate(w, seed=0)
    for algo in algos_for(w):
        check(inp, algo)


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_shapes_and_gates(gate, dtype, d):
    chunk = 16 if d == 16 else 64
    w = WORKLOADS["gdn_b4_h8_t2048_d128_bf16"].with_(
        B=1, T=2 * chunk + 5, H=2, dk=d, dv=d, chunk=chunk, dtype=dtype,
        gate=gate, decay_lo=0.005, decay_hi=0.05, init_state=True)
    for algo in algos_for(w):
        check(generate(w, seed=1), algo)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 32), (16, 64)])
def test_rectangular_state(dk, dv):
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=1, T=150, H=2, dk=dk, dv=dv, init_state=True)
    check(generate(w, seed=2), "staged")


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_chunk_size_does_not_change_the_result(chunk):
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=200, H=2,
                                                       chunk=chunk)
    check(generate(w, seed=3), "staged", chunk=chunk)


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 128])
def test_short_and_boundary_lengths(T):
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=2, T=T, H=2)
    inp = generate(w, seed=4)
    for algo in algos_for(w):
        check(inp, algo)


def time_slice(inp, a, b):
    """Tokens [a, b) of a fixed-length batch, same heads and initial state."""
    cut = lambda t: None if t is None else t[:, a:b].contiguous()  # noqa
    return dataclasses.replace(inp, w=inp.w.with_(T=b - a), q=cut(inp.q),
                               k=cut(inp.k), v=cut(inp.v),
                               beta=cut(inp.beta),
                               log_alpha=cut(inp.log_alpha),
                               lengths=[b - a] * len(inp.lengths))


def test_zero_length_sequences_pass_state_through():
    lens = [0, 70, 0, 1, 130, 0]
    ntok = sum(lens)
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        B=1, T=ntok, H=2, varlen_nseq=0, init_state=False)
    inp = generate(w, seed=5)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0).to(torch.int32)
    g = torch.Generator().manual_seed(6)
    inp = dataclasses.replace(
        inp, w=inp.w.with_(varlen_nseq=len(lens)), cu_seqlens=cu,
        lengths=lens,
        s0=torch.randn(len(lens), 2, 128, 128, generator=g) * 0.02)
    for algo in algos_for(inp.w):
        o, s = run_gpu(inp, algo)
        ro, rs = run_oracle(inp)
        assert out_err(o, ro, "bf16") <= 2e-2 and rel_err(s, rs) <= 2e-2
        # an empty sequence returns its initial state unchanged
        for n in (0, 2, 5):
            assert np.array_equal(s[n], inp.s0[n].numpy())


def test_state_carry_across_calls():
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=2, T=300, H=2)
    inp = generate(w, seed=8)
    cut = 130          # not a chunk multiple
    for algo in algos_for(w):
        o, s = run_gpu(inp, algo)
        o1, s1 = run_gpu(time_slice(inp, 0, cut), algo)
        second = dataclasses.replace(time_slice(inp, cut, 300),
                                     s0=torch.from_numpy(s1))
        o2, s2 = run_gpu(second, algo)
        oo = np.concatenate([o1, o2], axis=1)
        assert out_err(oo, o, "bf16") <= 2e-2 and rel_err(s2, s) <= 2e-2


def test_final_state_optional_and_no_out_of_bounds_writes():
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=2, T=77, H=2)
    inp = generate(w, seed=9)
    for algo in algos_for(w):
        guard = 4096
        buf = torch.full((2 * 77 * 2 * 128 + 2 * guard,), 7.0,
                         dtype=torch.bfloat16, device="cuda")
        out = buf[guard:guard + 2 * 77 * 2 * 128].view(2, 77, 2, 128)
        gdr.chunk_fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(),
                      inp.beta.cuda(), inp.log_alpha.cuda(), inp.s0.cuda(),
                      out=out, output_final_state=False, algo=algo)
        torch.cuda.synchronize()
        assert torch.all(buf[:guard] == 7.0) and torch.all(
            buf[-guard:] == 7.0)
        ro, _ = run_oracle(inp)
        assert out_err(out.float().cpu().numpy(), ro, "bf16") <= 2e-2


def test_host_entry_matches_device_entry():
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=150, H=2,
                                                       init_state=True)
    inp = generate(w, seed=10)
    for algo in algos_for(w):
        o, s = run_gpu(inp, algo)
        pin = lambda t: None if t is None else t.pin_memory()  # noqa: E731
        out = torch.empty_like(inp.v).pin_memory()
        sT = torch.empty(2, 2, 128, 128).pin_memory()
        gdr.chunk_fwd_host(pin(inp.q), pin(inp.k), pin(inp.v), pin(inp.beta),
                           pin(inp.log_alpha), pin(inp.s0), out=out,
                           final_state=sT, algo=algo)
        torch.cuda.synchronize()
        assert np.array_equal(out.float().numpy(), o)
        assert np.array_equal(sT.numpy(), s)


def run_host(inp, algo, final_state=True):
    """The host-buffer entry on pinned copies of the inputs."""
    pin = lambda t: None if t is None else t.pin_memory()  # noqa: E731
    out = torch.empty_like(inp.v).pin_memory()
    sT = (torch.full((inp.nseq, inp.w.H, inp.w.dk, inp.w.dv), 7.0).pin_memory()
          if final_state else None)
    gdr.chunk_fwd_host(pin(inp.q), pin(inp.k), pin(inp.v), pin(inp.beta),
                       pin(inp.log_alpha), pin(inp.s0), out=out,
                       final_state=sT, chunk=inp.w.chunk, gate=inp.w.gate,
                       cu_seqlens=pin(inp.cu_seqlens), algo=algo)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    return out.float().numpy(), None if sT is None else sT.numpy()


def test_host_entry_pieces_varlen():
    # 11 sequences, four of them empty: the host entry cuts them into 8
    # pieces of uneven size, each computed as its own sub-problem; the result
    # is the device entry's, bit for bit
    lens = [0, 70, 0, 1, 130, 0, 64, 200, 5, 0, 90]
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        B=1, T=sum(lens), H=2, varlen_nseq=0, init_state=False)
    inp = generate(w, seed=21)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0).to(torch.int32)
    g = torch.Generator().manual_seed(22)
    inp = dataclasses.replace(
        inp, w=inp.w.with_(varlen_nseq=len(lens)), cu_seqlens=cu,
        lengths=lens,
        s0=torch.randn(len(lens), 2, 128, 128, generator=g) * 0.02)
    for algo in algos_for(inp.w):
        o, s = run_gpu(inp, algo)
        ho, hs = run_host(inp, algo)
        assert np.array_equal(ho, o) and np.array_equal(hs, s)


def test_host_entry_pieces_fixed_length():
    # fixed length is cut by time at chunk boundaries: T = 100 -> pieces of
    # 64 and 36 tokens, the second starting from the first's state on the
    # device; no initial state, and no final state requested
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=10, T=100, H=3)
    inp = generate(w, seed=23)
    for algo in algos_for(w):
        o, _ = run_gpu(inp, algo)
        ho, hs = run_host(inp, algo, final_state=False)
        assert hs is None and np.array_equal(ho, o)
        ro, _ = run_oracle(inp)
        assert out_err(ho, ro, "bf16") <= 2e-2


@pytest.mark.parametrize("name,shape", [
    # 9 chunks -> 8 time pieces of 1 or 2 chunks and a ragged last chunk
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=3, T=8 * 64 + 37, H=2)),
    # fp32 staged path, chunk 16: 16 chunks -> 8 pieces of 2
    ("deltanet_b1_h1_t256_d16_fp32", dict(B=2, H=2)),
])
def test_host_entry_time_pieces_match_device_entry(name, shape):
    # the state passes from piece to piece in fp32, as from chunk to chunk:
    # the host entry's results are the device entry's, bit for bit, for every
    # path, with and without an initial state
    for init in (True, False):
        w = WORKLOADS[name].with_(**shape, init_state=init)
        inp = generate(w, seed=24)
        for algo in algos_for(w):
            o, s = run_gpu(inp, algo)
            ho, hs = run_host(inp, algo)
            assert np.array_equal(ho, o) and np.array_equal(hs, s)


def test_deterministic():
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=2, T=200, H=2)
    inp = generate(w, seed=11)
    for algo in algos_for(w):
        o1, s1 = run_gpu(inp, algo)
        o2, s2 = run_gpu(inp, algo)
        assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


# ---- full-size workloads, sampled heads
FULL_SAMPLE_HEADS = {
    "deltanet_b1_h1_t256_d16_fp32": [0],
    "gdn_b4_h8_t2048_d128_bf16": [0, 5],
    "gdn_b8_h16_t4096_d128_bf16": [3, 12],
    "kda_b4_h16_t4096_d128_bf16": [7],
    "gdn_varlen8_h16_d128_bf16": [1, 14],
}


@pytest.mark.parametrize("name", list(FULL_SAMPLE_HEADS))
def test_full_size_workloads_sampled_heads(name):
    w = WORKLOADS[name]
    inp = generate(w, seed=0)
    heads = FULL_SAMPLE_HEADS[name]
    sub = head_slice(inp, heads)
    ro, rs = run_oracle(sub)
    for algo in ["auto"] + algos_for(w):
        o, s = run_gpu(inp, algo)
        o, s = o[:, :, heads], s[:, heads]
        tol = TOL[w.dtype]
        assert out_err(o, ro, w.dtype) <= tol and rel_err(s, rs) <= tol, algo


def test_fused_reports_out_of_range_inputs():
    """The fused kernel's fp16 operands cannot hold |q| > 65504: the call
    must report GDR_ERR_RANGE through gdr_device_error, not pass silently."""
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=70, H=1)
    if "fused_tc" not in algos_for(w):
        pytest.skip("fused path not built")
    inp = generate(w, seed=12)
    q = inp.q.clone()
    q[0, 5, 0, 7] = 1.0e5
    gdr.chunk_fwd(q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.beta.cuda(),
                  inp.log_alpha.cuda(), inp.s0.cuda(), algo="fused_tc")
    assert gdr.device_error(clear=True) == 6          # GDR_ERR_RANGE
    assert gdr.device_error(clear=True) == 0          # cleared
    # the staged path computes the same call in fp32 without complaint
    o, s = gdr.chunk_fwd(q.cuda(), inp.k.cuda(), inp.v.cuda(),
                         inp.beta.cuda(), inp.log_alpha.cuda(),
                         inp.s0.cuda(), algo="staged")
    assert gdr.device_error() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(s).all()


@pytest.mark.parametrize("decay", [1.0, 2.0])
def test_strong_decays_scalar_gate(decay):
    # log-decays of about -0.8 and -1.6 per token on average: a chunk spans a
    # decay range above 80, so the fused kernel takes its per-element
    # exponential path instead of the factored one; every path meets the bar
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(
        B=2, T=3 * 64 + 17, H=2, decay_lo=decay, decay_hi=decay)
    inp = generate(w, seed=31)
    for algo in algos_for(w):
        check(inp, algo)


# Channel gate, fused path: the per-channel decay sits inside the contraction,
# so K K^T, Q K^T and U, W read operands rescaled by e^{+-(g - g_m)}: fp16
# while a chunk's decay stays within the fp16 window (about 3e-3 of the RMS at
# the KDA workload's decays); a chunk beyond it is computed on bf16 operands
# and the call reports GDR_ERR_RANGE.  So every fused result either meets the
# bar or is reported; the fp32 staged path meets the bar at any decay.
def fused_meets_bar_or_reports(inp):
    w = inp.w
    o, s = gdr.chunk_fwd(_dev(inp.q), _dev(inp.k), _dev(inp.v),
                         _dev(inp.beta), _dev(inp.log_alpha), _dev(inp.s0),
                         chunk=w.chunk, gate=w.gate, algo="fused_tc")
    err = gdr.device_error(clear=True)
    assert err in (0, 6)                       # OK or GDR_ERR_RANGE
    if err == 0:
        ro, rs = run_oracle(inp)
        o, s = o.float().cpu().numpy(), s.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(s).all()
        assert out_err(o, ro, w.dtype) <= TOL[w.dtype]
        assert rel_err(s, rs) <= TOL[w.dtype]
    return err


@pytest.mark.parametrize("decay", [1.0, 2.0])
def test_strong_decays_channel_gate(decay):
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=2, T=3 * 64 + 17, H=2, decay_lo=decay, decay_hi=decay)
    inp = generate(w, seed=31)
    check(inp, "staged")
    if "fused_tc" in algos_for(w):
        fused_meets_bar_or_reports(inp)


def test_channel_gate_reports_decays_beyond_its_window():
    """Log-decays of about -4 per token and channel: every chunk leaves the
    fused channel gate's fp16 window, so the call must report GDR_ERR_RANGE;
    at the KDA workload's own decays it reports nothing and meets the bar."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=1, T=2 * 64 + 9, H=2, decay_lo=5.0, decay_hi=5.0)
    if "fused_tc" not in algos_for(w):
        pytest.skip("fused path not built")
    inp = generate(w, seed=32)
    assert fused_meets_bar_or_reports(inp) == 6
    check(inp, "staged")                       # any decay in fp32
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=1, T=2 * 64 + 9, H=2)
    assert fused_meets_bar_or_reports(generate(w, seed=32)) == 0
