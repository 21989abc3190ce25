"""gdr_chunk_fwd_noalloc: the entry point for callers that cannot allocate
device memory at call time (for example a process whose device memory is
already reserved by another allocator, so any new cudaMalloc would fail).

It must give the same result as the allocating entry point, call after call,
even though every call reuses one static scratch array.  This file is
collected last on purpose, and passes alone in a fresh process as well as
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
from chunkwise_recurrence_b200.inputs import WORKLOADS, generate, rel_err

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _dev(t):
    return None if t is None else t.cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("name,shape", [
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=2, T=5 * 64 + 7, H=2)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=150, H=3)),
    ("deltanet_b1_h1_t256_d16_fp32", dict()),
    ("gdn_varlen8_h16_d128_bf16", dict(H=2, varlen_nseq=4, varlen_lo=1,
                                       varlen_hi=200)),
])
def test_noalloc_matches_allocating_entry_two_calls_in_a_row(name, shape):
    w = WORKLOADS[name].with_(**shape)
    inp = generate(w, seed=21)
    q, k, v = _dev(inp.q), _dev(inp.k), _dev(inp.v)
    beta, la, s0 = _dev(inp.beta), _dev(inp.log_alpha), _dev(inp.s0)
    cu = _dev(inp.cu_seqlens)
    ref_o, ref_s = gdr.chunk_fwd(q, k, v, beta, la, s0, chunk=w.chunk,
                                 gate=w.gate, cu_seqlens=cu, algo="staged")
    torch.cuda.synchronize()
    ref_o = ref_o.float().cpu().numpy()
    ref_s = ref_s.cpu().numpy()
    for _ in range(2):
        out = torch.full_like(inp.v, float("nan"), device="cuda")
        sT = torch.full((inp.nseq, w.H, w.dk, w.dv), float("nan"),
                        device="cuda")
        gdr.chunk_fwd_noalloc(q, k, v, beta, la, s0, out=out, final_state=sT,
                              chunk=w.chunk, gate=w.gate, cu_seqlens=cu)
        torch.cuda.synchronize()
        o, s = out.float().cpu().numpy(), sT.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(s).all()
        assert rel_err(o, ref_o) <= TOL[w.dtype]
        assert rel_err(s, ref_s) <= TOL[w.dtype]


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
