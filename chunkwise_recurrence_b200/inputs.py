"""Seeded synthetic workloads for the chunkwise gated delta rule.

This module holds input generation only -- none of the method's arithmetic --
so that the tests, the benchmark and the CPU oracle draw the very same inputs.

Value recipe (shapes follow the 340M-1.3B models the pages describe; no dataset
is involved):
  * q, k ~ N(0, 1), each token's q and k L2-normalised in fp32, then cast to the
    device dtype (the library takes keys as given and does not renormalise);
  * v ~ N(0, 1);
  * beta = sigmoid(N(0, 1));
  * scalar gate (Gated DeltaNet): log alpha = -softplus(N(0,1)) * U(lo, hi),
    one draw per (token, head);
  * channel gate (KDA): the same per (token, head, key channel);
  * initial state ~ N(0, 0.02^2) fp32 when the workload carries one;
  * varlen: sequence lengths drawn uniformly from [lo, hi] inclusive.
All draws come from one CPU ``torch.Generator`` seeded with ``seed`` in a fixed
order: lengths (varlen only), q, k, v, beta logit, alpha normal, alpha
uniform, initial state.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int            # per-sequence length (fixed) or 0 for varlen (drawn)
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str        # "fp32" or "bf16": dtype of q, k, v and out
    gate: str         # "none" | "scalar" | "channel"
    decay_lo: float = 0.0
    decay_hi: float = 0.0
    init_state: bool = False
    varlen_nseq: int = 0
    varlen_lo: int = 0
    varlen_hi: int = 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    w.name: w for w in [
        Workload("deltanet_b1_h1_t256_d16_fp32", B=1, T=256, H=1, dk=16,
                 dv=16, chunk=16, dtype="fp32", gate="none"),
        Workload("gdn_b4_h8_t2048_d128_bf16", B=4, T=2048, H=8, dk=128,
                 dv=128, chunk=64, dtype="bf16", gate="scalar",
                 decay_lo=0.01, decay_hi=0.1),
        Workload("gdn_b8_h16_t4096_d128_bf16", B=8, T=4096, H=16, dk=128,
                 dv=128, chunk=64, dtype="bf16", gate="scalar",
                 decay_lo=0.01, decay_hi=0.1, init_state=True),
        Workload("kda_b4_h16_t4096_d128_bf16", B=4, T=4096, H=16, dk=128,
                 dv=128, chunk=64, dtype="bf16", gate="channel",
                 decay_lo=0.005, decay_hi=0.05),
        Workload("gdn_varlen8_h16_d128_bf16", B=1, T=0, H=16, dk=128,
                 dv=128, chunk=64, dtype="bf16", gate="scalar",
                 decay_lo=0.01, decay_hi=0.1, init_state=True,
                 varlen_nseq=8, varlen_lo=2048, varlen_hi=16384),
        # long context, one sequence: fewer (sequence, head) chains than SMs
        # (the case for context-parallel state passing)
        Workload("gdn_longctx_b1_h16_t65536_d128_bf16", B=1, T=65536, H=16,
                 dk=128, dv=128, chunk=64, dtype="bf16", gate="scalar",
                 decay_lo=0.01, decay_hi=0.1, init_state=True),
    ]
}

# The headline workload: Gated DeltaNet, H=16, dk=dv=128, T=4096, bf16.
HEADLINE = "gdn_b8_h16_t4096_d128_bf16"

TORCH_DTYPE = {"fp32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class Inputs:
    w: Workload
    q: torch.Tensor            # [B, T, H, dk] in the device dtype (CPU)
    k: torch.Tensor
    v: torch.Tensor            # [B, T, H, dv]
    beta: torch.Tensor         # [B, T, H] fp32
    log_alpha: torch.Tensor | None   # [B, T, H] or [B, T, H, dk] fp32
    s0: torch.Tensor | None    # [N, H, dk, dv] fp32
    cu_seqlens: torch.Tensor | None  # [N+1] int32 (varlen only)
    lengths: list

    @property
    def nseq(self) -> int:
        return len(self.lengths)

    @property
    def ntok(self) -> int:
        return int(sum(self.lengths))

    def f64(self) -> dict:
        """fp64 numpy copies of the device-rounded values (oracle inputs)."""
        def c(t):
            return None if t is None else t.to(torch.float64).numpy()
        return dict(q=c(self.q), k=c(self.k), v=c(self.v), beta=c(self.beta),
                    log_alpha=c(self.log_alpha), initial_state=c(self.s0),
                    cu_seqlens=(None if self.cu_seqlens is None
                                else self.cu_seqlens.numpy().astype(np.int64)),
                    gate=self.w.gate)


def generate(w: Workload, seed: int = 0) -> Inputs:
    g = torch.Generator().manual_seed(seed)
    if w.varlen_nseq:
        lengths = torch.randint(w.varlen_lo, w.varlen_hi + 1,
                                (w.varlen_nseq,), generator=g).tolist()
        B, T = 1, int(sum(lengths))
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(
            torch.int32)
        nseq = len(lengths)
    else:
        B, T = w.B, w.T
        lengths = [T] * B
        cu = None
        nseq = B
    H, dk, dv = w.H, w.dk, w.dv
    q = torch.randn(B, T, H, dk, generator=g)
    k = torch.randn(B, T, H, dk, generator=g)
    v = torch.randn(B, T, H, dv, generator=g)
    beta_logit = torch.randn(B, T, H, generator=g)
    log_alpha = None
    if w.gate != "none":
        shp = (B, T, H) if w.gate == "scalar" else (B, T, H, dk)
        a_n = torch.randn(*shp, generator=g)
        a_u = torch.rand(*shp, generator=g) * (w.decay_hi - w.decay_lo) \
            + w.decay_lo
        log_alpha = (-F.softplus(a_n) * a_u).contiguous()
    s0 = None
    if w.init_state:
        s0 = (torch.randn(nseq, H, dk, dv, generator=g) * 0.02).contiguous()
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    dt = TORCH_DTYPE[w.dtype]
    return Inputs(w=w, q=q.to(dt).contiguous(), k=k.to(dt).contiguous(),
                  v=v.to(dt).contiguous(), beta=torch.sigmoid(beta_logit),
                  log_alpha=log_alpha, s0=s0, cu_seqlens=cu, lengths=lengths)


def gdn2_gates(inp: Inputs, seed: int = 0):
    """Gated DeltaNet-2 gates for a generated batch: an erase gate per key
    channel (the layout of k) and a write gate per value channel (the layout
    of v), both sigmoid(N(0, 1)) like beta, fp32, seeded."""
    g = torch.Generator().manual_seed(1_000_003 + seed)
    erase = torch.sigmoid(torch.randn(inp.k.shape, generator=g))
    write = torch.sigmoid(torch.randn(inp.v.shape, generator=g))
    return erase.float().contiguous(), write.float().contiguous()


def fg2_gates(inp: Inputs, seed: int = 0):
    """FG^2-GDN rates for a generated batch: a learning rate per key channel
    (the layout of k) and, for FG^2-GDN+, a target scaling per value channel
    (the layout of v), both sigmoid(N(0, 1)) like beta, fp32, seeded."""
    g = torch.Generator().manual_seed(2_000_003 + seed)
    beta_k = torch.sigmoid(torch.randn(inp.k.shape, generator=g))
    beta_v = torch.sigmoid(torch.randn(inp.v.shape, generator=g))
    return beta_k.float().contiguous(), beta_v.float().contiguous()


def head_slice(inp: Inputs, heads) -> Inputs:
    """The same inputs restricted to a subset of heads (chains are independent
    per head, so this is how large workloads are sampled for the oracle)."""
    hs = list(heads)

    def s(t, dim):
        return None if t is None else t.index_select(
            dim, torch.tensor(hs)).contiguous()
    return Inputs(w=inp.w.with_(H=len(hs)), q=s(inp.q, 2), k=s(inp.k, 2),
                  v=s(inp.v, 2), beta=s(inp.beta, 2),
                  log_alpha=s(inp.log_alpha, 2), s0=s(inp.s0, 1),
                  cu_seqlens=inp.cu_seqlens, lengths=inp.lengths)


def half_ulp(x, dtype: str):
    """Half a unit in the last place of |x| in `dtype` ("bf16": 8 significant
    bits, "fp32": 24): the rounding error of a correctly rounded result."""
    bits = {"bf16": 8, "fp32": 24}[dtype]
    _, e = np.frexp(np.abs(np.asarray(x, np.float64)))
    return np.ldexp(1.0, (e - 1 - bits).astype(np.int64))


def out_err(x, ref, dtype: str) -> float:
    """Parity metric of an output stored in `dtype`: max over elements of
    max(0, |x - ref| - u) / RMS(ref), u = half an ulp (in `dtype`) of the
    larger of |x| and |ref|.  The stored output must round its value; this
    discounts exactly that rounding, so the budget measures the arithmetic."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    if not x.size:
        return 0.0
    u = half_ulp(np.maximum(np.abs(x), np.abs(ref)), dtype)
    d = np.maximum(np.abs(x - ref) - u, 0.0)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(d.max()) / rms if rms else float(d.max())


def rel_err(x, ref) -> float:
    """max |x - ref| / RMS(ref) over the whole tensor (the parity metric)."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    if rms == 0.0:
        return float(np.max(np.abs(x - ref))) if x.size else 0.0
    return float(np.max(np.abs(x - ref))) / rms if x.size else 0.0
