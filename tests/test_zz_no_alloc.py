"""gdr_chunk_fwd_noalloc: the entry point for callers that cannot allocate
device memory at call time (for example a process whose device memory is
already reserved by another allocator, so any new cudaMalloc would fail).

It must give the fp64 oracle's result within the parity bar, and the
allocating entry point's, call after call, even though every call reuses
one static scratch array; it must still run when every allocation fails;
and it takes exactly the problems whose scratch fits its array.  This file
is collected last on purpose, and passes alone in a fresh process as well
as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
from chunkwise_recurrence_b200.inputs import (WORKLOADS, generate, out_err,
                                              rel_err)
from oracle import gdr_fwd

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _dev(t):
    return None if t is None else t.cuda()


def _noalloc(inp, w):
    q, k, v = _dev(inp.q), _dev(inp.k), _dev(inp.v)
    out = torch.full_like(inp.v, float("nan"), device="cuda")
    sT = torch.full((inp.nseq, w.H, w.dk, w.dv), float("nan"), device="cuda")
    gdr.chunk_fwd_noalloc(q, k, v, _dev(inp.beta), _dev(inp.log_alpha),
                          _dev(inp.s0), out=out, final_state=sT,
                          chunk=w.chunk, gate=w.gate,
                          cu_seqlens=_dev(inp.cu_seqlens))
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), sT.cpu().numpy()


def _check_oracle(inp, w, o, s):
    ro, rs, _ = gdr_fwd(**inp.f64())
    assert np.isfinite(o).all() and np.isfinite(s).all()
    assert out_err(o, ro, w.dtype) <= TOL[w.dtype]
    assert rel_err(s, rs) <= TOL[w.dtype]


@pytest.mark.gpu
@pytest.mark.parametrize("name,shape", [
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=2, T=5 * 64 + 7, H=2)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=150, H=3)),
    ("deltanet_b1_h1_t256_d16_fp32", dict()),
    ("gdn_varlen8_h16_d128_bf16", dict(H=2, varlen_nseq=4, varlen_lo=1,
                                       varlen_hi=200)),
])
def test_noalloc_matches_oracle_and_allocating_entry_two_calls_in_a_row(
        name, shape):
    w = WORKLOADS[name].with_(**shape)
    inp = generate(w, seed=21)
    ref_o, ref_s = gdr.chunk_fwd(
        _dev(inp.q), _dev(inp.k), _dev(inp.v), _dev(inp.beta),
        _dev(inp.log_alpha), _dev(inp.s0), chunk=w.chunk, gate=w.gate,
        cu_seqlens=_dev(inp.cu_seqlens), algo="staged")
    torch.cuda.synchronize()
    ref_o = ref_o.float().cpu().numpy()
    ref_s = ref_s.cpu().numpy()
    for _ in range(2):
        o, s = _noalloc(inp, w)
        _check_oracle(inp, w, o, s)
        assert rel_err(o, ref_o) <= TOL[w.dtype]
        assert rel_err(s, ref_s) <= TOL[w.dtype]


@pytest.mark.gpu
def test_noalloc_runs_when_every_allocation_fails(monkeypatch):
    # the library's allocation hook makes every scratch allocation fail: the
    # allocating entry reports it, the no-allocation entry runs as before
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=2, T=3 * 64 + 9, H=2)
    inp = generate(w, seed=22)
    monkeypatch.setenv("GDR_FAULT_INJECT_ALLOC", "1")
    with pytest.raises(gdr.GdrError) as e:
        gdr.chunk_fwd(_dev(inp.q), _dev(inp.k), _dev(inp.v), _dev(inp.beta),
                      _dev(inp.log_alpha), _dev(inp.s0), chunk=w.chunk,
                      gate=w.gate, algo="staged")
    assert e.value.code == 4          # GDR_ERR_OUT_OF_MEMORY
    for _ in range(2):
        o, s = _noalloc(inp, w)
        _check_oracle(inp, w, o, s)


def _staged_scratch_bytes(B, T, H, dk, dv, C, gdim):
    # the staged path's scratch: the chunk table and sequence offsets, the
    # fp32 log-decay cumsum, W, U and V_new per token-head, and the fp32
    # state of every chunk-head, each region rounded up to 256 bytes
    a = lambda x: (x + 255) & ~255  # noqa: E731
    th, nch = B * T * H, B * ((T + C - 1) // C)
    return (a(16 * nch) + a(4 * (B + 1)) + a(4 * th * gdim) + a(4 * th * dk)
            + 2 * a(4 * th * dv) + a(4 * nch * H * dk * dv))


@pytest.mark.gpu
def test_noalloc_takes_a_problem_just_under_its_scratch():
    limit = 64 << 20                   # GDR_NOALLOC_SCRATCH_BYTES
    T = 26167
    assert _staged_scratch_bytes(1, T, 1, 128, 128, 64, 1) <= limit
    assert _staged_scratch_bytes(1, T + 1, 1, 128, 128, 64, 1) > limit
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=T, H=1)
    inp = generate(w, seed=23)
    o, s = _noalloc(inp, w)
    _check_oracle(inp, w, o, s)
    # one token more no longer fits: rejected before any CUDA call
    w2 = w.with_(T=T + 1)
    inp2 = generate(w2, seed=23)
    with pytest.raises(gdr.GdrError) as e:
        _noalloc(inp2, w2)
    assert e.value.code == 2          # GDR_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = gdr.load_library()
    A = 0x10000   # aligned fake address: the size check precedes any CUDA call
    opts = gdr._Opts(0, 1, None, 0, 0)
    rc = lib.gdr_chunk_fwd_noalloc(A, A, A, A, A, None, A, None, 8, 4096, 16,
                                   128, 128, 64, None, ctypes.byref(opts))
    assert rc == 2      # GDR_ERR_UNSUPPORTED
    opts = gdr._Opts(0, 1, None, 0, 2)   # the fused path has no such variant
    rc = lib.gdr_chunk_fwd_noalloc(A, A, A, A, A, None, A, None, 1, 64, 1,
                                   128, 128, 64, None, ctypes.byref(opts))
    assert rc == 2
