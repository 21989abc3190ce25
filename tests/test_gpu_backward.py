"""GPU parity of the backward pass (gdr_backward, through the C ABI) against
fp64 autograd gradients of the token loop (oracle.gdr_grads, itself pinned by
finite differences of the C oracle), for both algorithms: the chunked
backward (AUTO, STAGED) and the reverse token recurrence (RECURRENT).

Tolerance: both compute in fp32 (the chunked one's tensor-core products on
operands split into a tf32 part and its remainder); every gradient tensor
must satisfy max |gpu - oracle| / RMS(oracle) <= 1e-3 (fp32 accumulation over
a few hundred dependent steps stays two orders of magnitude below that)."""
import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
import oracle
from chunkwise_recurrence_b200.inputs import WORKLOADS, generate, rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _check(w, seed=0, with_final=True, with_s0_grad=True, algo="auto"):
    inp = generate(w, seed=seed)
    g = torch.Generator().manual_seed(seed + 100)
    dO = torch.randn(inp.v.shape, generator=g).to(inp.v.dtype)
    nseq = inp.nseq
    dS = (torch.randn(nseq, w.H, w.dk, w.dv, generator=g) * 0.1
          if with_final else None)
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    res = gdr.backward(c(inp.q), c(inp.k), c(inp.v), c(inp.beta),
                       c(inp.log_alpha), c(inp.s0), c(dO), c(dS), gate=w.gate,
                       cu_seqlens=c(inp.cu_seqlens),
                       need_initial_state_grad=with_s0_grad, algo=algo)
    torch.cuda.synchronize()
    f = inp.f64()
    ref = oracle.gdr_grads(f["q"], f["k"], f["v"], f["beta"], f["log_alpha"],
                           gate=w.gate, initial_state=f["initial_state"],
                           d_out=dO.double().numpy(),
                           d_final_state=None if dS is None else dS.numpy(),
                           cu_seqlens=f["cu_seqlens"])
    errs = {}
    for key in ("dq", "dk", "dv", "dbeta", "dlog_alpha"):
        if ref[key] is None:
            assert res[key] is None
            continue
        errs[key] = rel_err(res[key].cpu().numpy(), ref[key])
    if with_s0_grad:
        # without an initial state the gradient of a zero state is still
        # defined: it is the gradient with respect to S_0
        if ref["dinitial_state"] is not None:
            errs["ds0"] = rel_err(res["dinitial_state"].cpu().numpy(),
                                  ref["dinitial_state"])
    for key, e in errs.items():
        assert e <= TOL, (key, e, errs)
    return errs


@pytest.mark.parametrize("name,shape", [
    ("deltanet_b1_h1_t256_d16_fp32", dict(T=70)),
    ("gdn_b4_h8_t2048_d128_bf16", dict(B=2, T=37, H=2, dk=32, dv=16)),
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=2, T=48, H=2)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=33, H=2, dk=64, dv=128)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=2, T=16, H=1, dk=16, dv=32,
                                        dtype="fp32")),
    # column-split kernel: two column groups, fp32, channel gate, ragged
    # last window; no gate with four groups
    ("kda_b4_h16_t4096_d128_bf16", dict(B=2, T=19, H=2, dk=128, dv=64,
                                        dtype="fp32")),
    ("deltanet_b1_h1_t256_d16_fp32", dict(T=45, H=3, dk=32, dv=128)),
])
@pytest.mark.parametrize("algo", ["auto", "recurrent"])
def test_backward_matches_autograd(name, shape, algo):
    _check(WORKLOADS[name].with_(**shape), algo=algo)


@pytest.mark.parametrize("algo", ["staged", "recurrent"])
def test_backward_varlen_and_optional_gradients(algo):
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        varlen_nseq=3, varlen_lo=5, varlen_hi=40, H=2, dk=32, dv=32)
    _check(w, with_final=False, with_s0_grad=True, algo=algo)
    w2 = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=20, H=1)
    _check(w2, with_final=True, with_s0_grad=False, algo=algo)


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("fp32", 64, 32),
                                         ("bf16", 16, 64)])
def test_chunked_backward_several_chunks(gate, dtype, dk, dv):
    """Several 64-token chunks and a ragged last one: the chunk-boundary
    scans carry the state forward and its gradient backward."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=2, T=3 * 64 + 17, H=2, dk=dk, dv=dv, dtype=dtype, gate=gate,
        init_state=True)
    _check(w, seed=3, algo="staged")


def test_chunked_backward_varlen_many_sequences():
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        varlen_nseq=5, varlen_lo=1, varlen_hi=300, H=2, gate="channel")
    _check(w, seed=4, algo="staged")


@pytest.mark.parametrize("decay", [0.3, 3.0])
def test_chunked_backward_strong_channel_decay(decay):
    """Mean log-decays of -0.3 and -3 per token and channel: the second puts
    a chunk's spread beyond the factored range, so the gradient kernel takes
    its one-exponential-per-element path (and P too)."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=1, T=2 * 64 + 9, H=2, decay_lo=decay, decay_hi=decay)
    _check(w, seed=5, algo="staged")


def test_backward_headline_shape_sampled():
    """The 1.3B-layer Gated DeltaNet shape with the full sequence length
    (T = 4096, d = 128) on one sequence and two heads: 4096 dependent reverse
    steps, compared with autograd in full."""
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, H=2)
    for algo in ("staged", "recurrent"):
        errs = _check(w, algo=algo)
        assert max(errs.values()) <= TOL


# ---------------------------------------------------------------------------
# gdr_backward_gdn2: the gate-aware backward of the Gated DeltaNet-2 forward,
# against fp64 autograd through oracle.gdn2_fwd's token loop
# (oracle.gdn2_grads, pinned by central differences).

def _check_gdn2(w, seed=0, with_final=True):
    from chunkwise_recurrence_b200.inputs import gdn2_gates
    inp = generate(w, seed=seed)
    erase, write = gdn2_gates(inp, seed=seed)
    g = torch.Generator().manual_seed(seed + 200)
    dO = torch.randn(inp.v.shape, generator=g).to(inp.v.dtype)
    dS = (torch.randn(inp.nseq, w.H, w.dk, w.dv, generator=g) * 0.1
          if with_final else None)
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    res = gdr.backward_gdn2(c(inp.q), c(inp.k), c(inp.v), c(erase),
                            c(write), c(inp.log_alpha), c(inp.s0), c(dO),
                            c(dS), gate=w.gate, cu_seqlens=c(inp.cu_seqlens))
    torch.cuda.synchronize()
    f = inp.f64()
    ref = oracle.gdn2_grads(f["q"], f["k"], f["v"], erase.double().numpy(),
                            write.double().numpy(), f["log_alpha"],
                            gate=w.gate, initial_state=f["initial_state"],
                            d_out=dO.double().numpy(),
                            d_final_state=None if dS is None else dS.numpy(),
                            cu_seqlens=f["cu_seqlens"])
    errs = {}
    for key in ("dq", "dk", "dv", "derase", "dwrite", "dlog_alpha"):
        if ref[key] is None:
            continue
        errs[key] = rel_err(res[key].cpu().numpy(), ref[key])
    if ref["dinitial_state"] is not None:
        errs["ds0"] = rel_err(res["dinitial_state"].cpu().numpy(),
                              ref["dinitial_state"])
    for key, e in errs.items():
        assert e <= TOL, (key, e, errs)
    return errs


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("fp32", 32, 64)])
def test_backward_gdn2_matches_autograd(gate, dtype, dk, dv):
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=2, T=2 * 64 + 29, H=2, dk=dk, dv=dv, dtype=dtype, gate=gate,
        init_state=True)
    _check_gdn2(w, seed=7)


def test_backward_gdn2_varlen_and_strong_decay():
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        varlen_nseq=4, varlen_lo=1, varlen_hi=200, H=2, gate="channel")
    _check_gdn2(w, seed=8, with_final=False)
    w2 = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=1, T=64 + 40, H=1, decay_lo=3.0, decay_hi=3.0)
    _check_gdn2(w2, seed=9)


def test_backward_gdn2_with_gates_equal_to_beta_is_the_delta_rule():
    """b = w = beta on every channel: the Gated DeltaNet-2 gradients are the
    delta rule's, with dbeta the sum of the two gates' gradients over their
    channels."""
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(B=2, T=100, H=2,
                                                       dtype="fp32")
    inp = generate(w, seed=10)
    erase = inp.beta[..., None].expand(inp.k.shape).contiguous()
    write = inp.beta[..., None].expand(inp.v.shape).contiguous()
    g = torch.Generator().manual_seed(11)
    dO = torch.randn(inp.v.shape, generator=g)
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    r2 = gdr.backward_gdn2(c(inp.q), c(inp.k), c(inp.v), c(erase), c(write),
                           c(inp.log_alpha), c(inp.s0), c(dO), gate=w.gate)
    r1 = gdr.backward(c(inp.q), c(inp.k), c(inp.v), c(inp.beta),
                      c(inp.log_alpha), c(inp.s0), c(dO), gate=w.gate)
    torch.cuda.synchronize()
    for key in ("dq", "dk", "dv", "dlog_alpha", "dinitial_state"):
        assert rel_err(r2[key].cpu().numpy(), r1[key].cpu().numpy()) <= 1e-4
    db = (r2["derase"].sum(-1) + r2["dwrite"].sum(-1)).cpu().numpy()
    assert rel_err(db, r1["dbeta"].cpu().numpy()) <= 1e-4


# ---------------------------------------------------------------------------
# gdr_backward_fg2: FG^2-GDN's rate (and FG^2-GDN+'s value scaling) through
# the chunked backward, against fp64 autograd through oracle.fg2_fwd's token
# loop (oracle.fg2_grads, pinned by central differences).

def _check_fg2(w, seed=0, plus=True, with_final=True):
    from chunkwise_recurrence_b200.inputs import fg2_gates
    inp = generate(w, seed=seed)
    bk, bv = fg2_gates(inp, seed=seed)
    if not plus:
        bv = None
    g = torch.Generator().manual_seed(seed + 300)
    dO = torch.randn(inp.v.shape, generator=g).to(inp.v.dtype)
    dS = (torch.randn(inp.nseq, w.H, w.dk, w.dv, generator=g) * 0.1
          if with_final else None)
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    res = gdr.backward_fg2(c(inp.q), c(inp.k), c(inp.v), c(bk), c(bv),
                           c(inp.log_alpha), c(inp.s0), c(dO), c(dS),
                           gate=w.gate, cu_seqlens=c(inp.cu_seqlens))
    torch.cuda.synchronize()
    f = inp.f64()
    ref = oracle.fg2_grads(f["q"], f["k"], f["v"], bk.double().numpy(),
                           None if bv is None else bv.double().numpy(),
                           f["log_alpha"], gate=w.gate,
                           initial_state=f["initial_state"],
                           d_out=dO.double().numpy(),
                           d_final_state=None if dS is None else dS.numpy(),
                           cu_seqlens=f["cu_seqlens"])
    errs = {}
    for key in ("dq", "dk", "dv", "dbeta_k", "dbeta_v", "dlog_alpha"):
        if ref[key] is None:
            assert res[key] is None or key == "dlog_alpha"
            continue
        errs[key] = rel_err(res[key].cpu().numpy(), ref[key])
    if ref["dinitial_state"] is not None:
        errs["ds0"] = rel_err(res["dinitial_state"].cpu().numpy(),
                              ref["dinitial_state"])
    for key, e in errs.items():
        assert e <= TOL, (key, e, errs)
    return errs


@pytest.mark.parametrize("plus", [False, True])
@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
def test_backward_fg2_matches_autograd(gate, plus):
    w = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=2, T=2 * 64 + 29, H=2, gate=gate, init_state=True)
    _check_fg2(w, seed=12, plus=plus)


def test_backward_fg2_varlen_fp32_and_strong_decay():
    w = WORKLOADS["gdn_varlen8_h16_d128_bf16"].with_(
        varlen_nseq=4, varlen_lo=1, varlen_hi=200, H=2, gate="channel",
        dtype="fp32", dk=64, dv=32)
    _check_fg2(w, seed=13, with_final=False)
    w2 = WORKLOADS["kda_b4_h16_t4096_d128_bf16"].with_(
        B=1, T=64 + 40, H=1, decay_lo=3.0, decay_hi=3.0)
    _check_fg2(w2, seed=14)
