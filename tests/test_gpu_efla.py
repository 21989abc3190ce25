"""GPU parity of the exact-flow (EFLA) variant: gdr_efla_beta turns beta into
the exact-flow step size, then the unchanged chunked forward pass (or decode
step) runs the recurrence; both are compared with oracle.efla_fwd, which
integrates each token's flow with a matrix exponential.

Tolerance as for the plain recurrence: max |gpu - oracle| / RMS(oracle) <=
1e-4 for fp32 inputs and <= 2e-2 for bf16 inputs (output after the half-ulp
discount of its storage dtype)."""
import numpy as np
import pytest
import torch

import chunkwise_recurrence_b200 as gdr
import oracle
from chunkwise_recurrence_b200.inputs import WORKLOADS, generate, out_err, rel_err

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _efla_case(name, **shape):
    w = WORKLOADS[name].with_(**shape)
    inp = generate(w, seed=5)
    # step sizes up to 3 and keys off the unit sphere, where the exact flow
    # and the Euler step differ most
    g = torch.Generator().manual_seed(9)
    scale = torch.rand(*inp.k.shape[:-1], 1, generator=g) * 1.5 + 0.5
    k = (inp.k.float() * scale).to(inp.k.dtype)
    beta = (inp.beta * 3.0).contiguous()
    return w, inp, k, beta


@pytest.mark.parametrize("name,shape", [
    ("deltanet_b1_h1_t256_d16_fp32", dict(T=80)),
    ("gdn_b4_h8_t2048_d128_bf16", dict(B=1, T=64 + 13, H=2, dk=16, dv=16,
                                       dtype="fp32", chunk=16)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=50, H=2, dk=32, dv=16,
                                        dtype="fp32", chunk=16)),
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=1, T=70, H=2)),
])
def test_efla_chunked_matches_exact_flow(name, shape):
    w, inp, k, beta = _efla_case(name, **shape)
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    bp = gdr.efla_beta(c(k), c(beta))
    out, sT = gdr.chunk_fwd(c(inp.q), c(k), c(inp.v), bp, c(inp.log_alpha),
                            c(inp.s0), chunk=w.chunk, gate=w.gate)
    torch.cuda.synchronize()
    assert gdr.device_error() == 0
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    ro, rs = oracle.efla_fwd(f(inp.q), f(k), f(inp.v), f(beta),
                             f(inp.log_alpha), gate=w.gate,
                             initial_state=f(inp.s0))
    assert out_err(out.float().cpu().numpy(), ro, w.dtype) <= TOL[w.dtype]
    assert rel_err(sT.cpu().numpy(), rs) <= TOL[w.dtype]


def test_efla_decode_step_matches_exact_flow():
    w, inp, k, beta = _efla_case("gdn_b8_h16_t4096_d128_bf16", B=3, T=1, H=4,
                                 dtype="fp32")
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    one = lambda t: None if t is None else t[:, 0].contiguous()  # noqa: E731
    bp = gdr.efla_beta(c(one(k)), c(one(beta)))
    state = c(inp.s0).clone()
    out, state = gdr.decode_step(c(one(inp.q)), c(one(k)), c(one(inp.v)), bp,
                                 c(one(inp.log_alpha)), state)
    torch.cuda.synchronize()
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    ro, rs = oracle.efla_fwd(f(inp.q), f(k), f(inp.v), f(beta),
                             f(inp.log_alpha), gate="scalar",
                             initial_state=f(inp.s0))
    assert rel_err(out.cpu().numpy(), ro[:, 0]) <= 1e-4
    assert rel_err(state.cpu().numpy(), rs) <= 1e-4


def test_efla_beta_in_place_and_zero_key():
    k = torch.zeros(3, 2, 64, device="cuda", dtype=torch.bfloat16)
    k[0] = 1.0 / 8.0                       # |k|^2 = 1 for the first token
    beta = torch.full((3, 2), 0.7, device="cuda")
    gdr.efla_beta(k, beta, out=beta)       # in place
    torch.cuda.synchronize()
    b = beta.cpu().numpy()
    assert np.allclose(b[0], 1 - np.exp(-0.7), rtol=1e-6)
    assert np.allclose(b[1:], 0.7)         # zero key: the limit beta


# ---------------------------------------------------------------------------
# The EFLA backward: gdr_backward with beta' gives d beta' and dk at fixed
# beta'; gdr_efla_beta_backward carries d beta' through beta' = f(beta, |k|^2)
# into d beta and dk.  Against fp64 autograd with beta' formed inside the
# graph (oracle.efla_grads, pinned by central differences of the
# matrix-exponential flow), 1e-3 of the RMS per gradient (the backward's
# fp32 bar).

@pytest.mark.parametrize("name,shape", [
    ("gdn_b8_h16_t4096_d128_bf16", dict(B=2, T=2 * 64 + 21, H=2)),
    ("kda_b4_h16_t4096_d128_bf16", dict(B=1, T=90, H=2, dk=32, dv=64,
                                        dtype="fp32")),
    ("deltanet_b1_h1_t256_d16_fp32", dict(T=70)),
])
def test_efla_backward_matches_autograd(name, shape):
    w, inp, k, beta = _efla_case(name, **shape)
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    g = torch.Generator().manual_seed(17)
    dO = torch.randn(inp.v.shape, generator=g).to(inp.v.dtype)
    dS = torch.randn(inp.nseq, w.H, w.dk, w.dv, generator=g) * 0.1
    kc, bc = c(k), c(beta)
    bp = gdr.efla_beta(kc, bc)
    res = gdr.backward(c(inp.q), kc, c(inp.v), bp, c(inp.log_alpha),
                       c(inp.s0), c(dO), c(dS), gate=w.gate)
    dbeta = gdr.efla_beta_backward(kc, bc, res["dbeta"], res["dk"])
    torch.cuda.synchronize()
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    ref = oracle.efla_grads(f(inp.q), f(k), f(inp.v), f(beta),
                            f(inp.log_alpha), gate=w.gate,
                            initial_state=f(inp.s0), d_out=f(dO),
                            d_final_state=f(dS))
    got = dict(res, dbeta=dbeta)
    for key in ("dq", "dk", "dv", "dbeta", "dlog_alpha"):
        if ref[key] is None:
            continue
        assert rel_err(got[key].cpu().numpy(), ref[key]) <= 1e-3, key
    if ref["dinitial_state"] is not None:
        assert rel_err(res["dinitial_state"].cpu().numpy(),
                       ref["dinitial_state"]) <= 1e-3


def test_efla_beta_backward_small_and_zero_keys():
    """The chain rule's small-|k| branch (Taylor series) and its limit at
    k = 0 (d beta = d beta', dk unchanged) against float64 formulas."""
    H, dk = 1, 16
    g = torch.Generator().manual_seed(19)
    k = torch.randn(6, H, dk, generator=g)
    k[0] = 0.0
    k[1] *= 1e-3
    k[2] *= 0.05
    beta = torch.tensor([[0.5], [0.9], [2.0], [0.3], [3.0], [1.0]])
    dbp = torch.randn(6, H, generator=g)
    dk0 = torch.randn(6, H, dk, generator=g)
    dkg = dk0.clone().cuda()
    db = gdr.efla_beta_backward(k.cuda(), beta.cuda(), dbp.cuda(), dkg)
    torch.cuda.synchronize()
    kd, bd, gd = k.double(), beta.double(), dbp.double()
    s = (kd * kd).sum(-1)
    x = bd * s
    db_ref = gd * torch.exp(-x)
    # d beta' / d s = beta^2 f(x) / x^2, f(x) = x e^-x + e^-x - 1 (-> -1/2)
    fx = torch.where(x > 1e-8, (x * torch.exp(-x) + torch.expm1(-x)) /
                     (x * x).clamp_min(1e-300), torch.full_like(x, -0.5))
    dk_ref = dk0.double() + (2 * gd * bd * bd * fx)[..., None] * kd
    assert torch.allclose(db.cpu().double(), db_ref, rtol=1e-5, atol=1e-7)
    assert torch.allclose(dkg.cpu().double(), dk_ref, rtol=1e-4, atol=1e-6)
