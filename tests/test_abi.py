"""The C ABI without a GPU: the library loads, exports every declared symbol,
and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import chunkwise_recurrence_b200 as gdr
from chunkwise_recurrence_b200 import build as gdr_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, CUDA, OOM, TIMEOUT = range(6)


@pytest.fixture(scope="module")
def lib():
    gdr_build.build()
    return gdr.load_library()


def _declared_symbols():
    syms = []
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            text = open(os.path.join(ROOT, "include", name)).read()
            syms += re.findall(r"^GDR_API[^(]*?\b(\w+)\s*\(", text, re.M)
    return syms


def test_exports_every_declared_symbol(lib):
    syms = _declared_symbols()
    assert set(gdr.EXPORTED_SYMBOLS) <= set(syms)
    for s in syms:
        assert hasattr(lib, s), s


def test_status_strings(lib):
    for code, name in gdr.STATUS.items():
        assert gdr.status_string(code) == name
    assert gdr.status_string(99) == "GDR_ERR_UNKNOWN"


A = 0x10000       # a 16-byte-aligned fake device address (never dereferenced)


def call(lib, *, q=A, k=A, v=A, la=A, beta=A, s0=None, out=A, sT=None, B=1,
         T=64, H=1, dk=128, dv=128, chunk=64, dtype=0, gate=1, cu=None,
         nseq=0, algo=0, host=False):
    opts = gdr._Opts(dtype, gate, cu, nseq, algo)
    f = lib.gdr_chunk_fwd_host if host else lib.gdr_chunk_fwd
    return f(q, k, v, la, beta, s0, out, sT, B, T, H, dk, dv, chunk, None,
             ctypes.byref(opts))


@pytest.mark.parametrize("host", [False, True])
def test_rejects_bad_arguments(lib, host):
    c = lambda **kw: call(lib, host=host, **kw)  # noqa: E731
    assert c(q=None) == INVALID
    assert c(out=None) == INVALID
    assert c(beta=None) == INVALID
    assert c(k=A + 8) == INVALID                   # misaligned
    assert c(s0=A + 4) == INVALID
    assert c(la=None) == INVALID                   # scalar gate needs alpha
    assert c(gate=0) == INVALID                    # no gate forbids alpha
    assert c(gate=7) == INVALID
    assert c(dtype=5) == INVALID
    assert c(algo=9) == INVALID
    assert c(T=-1) == INVALID
    assert c(B=-2) == INVALID
    assert c(dk=48) == UNSUPPORTED
    assert c(dv=256) == UNSUPPORTED
    assert c(dk=8) == UNSUPPORTED
    assert c(chunk=128) == UNSUPPORTED
    assert c(chunk=8) == UNSUPPORTED
    assert c(chunk=48) == UNSUPPORTED
    assert c(B=2, cu=A, nseq=1) == INVALID         # varlen needs B == 1
    assert c(cu=A, nseq=-1) == INVALID
    assert c(nseq=3) == INVALID                    # num_seqs without cu
    assert c(B=1 << 20, T=1 << 12) == UNSUPPORTED  # too many tokens
    assert c(H=70000) == UNSUPPORTED


@pytest.mark.parametrize("cu", [[1, 10, 64], [0, 40, 30, 64], [0, 10, 63],
                                [0, 10, 65]])
def test_host_entry_checks_sequence_offsets(lib, cu):
    # the host entry reads cu_seqlens on the host: first 0, non-decreasing,
    # last T; the tensor pointers are never touched on rejection
    arr = np.zeros(len(cu) + 4, dtype=np.int32)
    base = (-arr.ctypes.data // 4) % 4          # a 16-byte-aligned start
    view = arr[base:base + len(cu)]
    view[:] = cu
    assert call(lib, host=True, cu=view.ctypes.data, nseq=len(cu) - 1,
                T=64) == INVALID


@pytest.mark.parametrize("host", [False, True])
def test_empty_batch_is_a_noop(lib, host):
    # no pointer is touched and no CUDA call is made
    assert call(lib, q=None, k=None, v=None, la=None, beta=None, out=None, gate=0,
                B=0, host=host) == OK
    assert call(lib, q=None, k=None, v=None, la=None, beta=None, out=None, gate=0,
                H=0, host=host) == OK
    assert call(lib, q=None, k=None, v=None, la=None, beta=None, out=None, gate=0,
                cu=A, nseq=0, host=host) == OK


@pytest.mark.parametrize("host", [False, True])
def test_scratch_allocation_failure_is_reported(lib, host, monkeypatch):
    monkeypatch.setenv("GDR_FAULT_INJECT_ALLOC", "1")
    assert call(lib, algo=1, host=host) == OOM


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        gdr.load_library(str(tmp_path / "libgdr.so"))


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "chunkwise_recurrence_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cuh", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text,
                                     re.M), f
                assert "gdr_oracle" not in text and "liboracle" not in text, f


def dcall(lib, *, q=A, k=A, v=A, la=A, beta=A, sin=None, sout=A, out=A, N=4,
          H=2, dk=128, dv=128, dtype=0, gate=1, cu=None, nseq=0, algo=0):
    opts = gdr._Opts(dtype, gate, cu, nseq, algo)
    return lib.gdr_decode_step(q, k, v, la, beta, sin, sout, out, N, H, dk, dv,
                               None, ctypes.byref(opts))


def test_decode_step_rejects_bad_arguments(lib):
    c = lambda **kw: dcall(lib, **kw)  # noqa: E731
    assert c(q=None) == INVALID
    assert c(sout=None) == INVALID                 # the state is written
    assert c(out=None) == INVALID
    assert c(v=A + 8) == INVALID                   # misaligned
    assert c(sin=A + 4) == INVALID
    assert c(la=None) == INVALID
    assert c(gate=0) == INVALID
    assert c(gate=3) == INVALID
    assert c(dtype=2) == INVALID
    assert c(N=-1) == INVALID
    assert c(cu=A) == INVALID                      # nothing to pack
    assert c(nseq=2) == INVALID
    assert c(algo=1) == UNSUPPORTED
    assert c(dk=48) == UNSUPPORTED
    assert c(dv=8) == UNSUPPORTED
    assert c(N=1 << 20, H=1 << 12) == UNSUPPORTED  # N * H >= 2^31
    # partially overlapping input and output states (4*2*128*128*4 bytes)
    assert c(sin=A, sout=A + 4096) == INVALID
    assert c(sin=A + 4096, sout=A) == INVALID
    # no pointer is touched and no CUDA call is made for an empty batch
    assert c(q=None, k=None, v=None, la=None, beta=None, sout=None, out=None,
             gate=0, N=0) == OK
    assert c(q=None, k=None, v=None, la=None, beta=None, sout=None, out=None,
             gate=0, H=0) == OK


def test_efla_beta_backward_rejects_bad_arguments(lib):
    f = lambda k=A, b=A, g=A + 4096, db=A + 8192, dk=A + 16384, ntok=8, H=2, \
        d=64, dt=0: lib.gdr_efla_beta_backward(k, b, g, db, dk, ntok, H, d,
                                                dt, None)  # noqa: E731
    assert f(k=None) == INVALID
    assert f(g=None) == INVALID
    assert f(dk=A + 4) == INVALID        # misaligned
    assert f(dt=3) == INVALID
    assert f(ntok=-1) == INVALID
    assert f(d=48) == UNSUPPORTED
    assert f(k=None, b=None, g=None, db=None, dk=None, ntok=0) == OK


def test_efla_beta_rejects_bad_arguments(lib):
    f = lambda k=A, b=A, o=A + 4096, ntok=8, H=2, dk=64, dt=0: \
        lib.gdr_efla_beta(k, b, o, ntok, H, dk, dt, None)  # noqa: E731
    assert f(k=None) == INVALID
    assert f(b=A + 4) == INVALID        # misaligned
    assert f(o=A + 16) == INVALID       # overlaps beta (8 x 2 floats)
    assert f(dt=3) == INVALID
    assert f(ntok=-1) == INVALID
    assert f(dk=48) == UNSUPPORTED
    assert f(k=None, b=None, o=None, ntok=0) == OK   # empty: no-op


def bcall(lib, *, q=A, k=A, v=A, la=A, beta=A, s0=None, dout=A, dsT=None,
          dq=A, dk=A, dv=A, dla=A, db=A, ds0=None, B=1, T=32, H=1, dk_=64,
          dv_=64, gate=1, dtype=0, algo=0, cu=None, nseq=0):
    opts = gdr._Opts(dtype, gate, cu, nseq, algo)
    return lib.gdr_backward(q, k, v, la, beta, s0, dout, dsT, dq, dk, dv, dla,
                            db, ds0, B, T, H, dk_, dv_, None,
                            ctypes.byref(opts))


def test_backward_rejects_bad_arguments(lib):
    c = lambda **kw: bcall(lib, **kw)  # noqa: E731
    assert c(dout=None) == INVALID       # the upstream output gradient
    assert c(dq=None) == INVALID
    assert c(db=None) == INVALID
    assert c(dla=None) == INVALID        # a gate needs its gradient
    assert c(gate=0, la=None) == INVALID  # ... and no gate forbids it
    assert c(dk=A + 4) == INVALID        # misaligned
    assert c(ds0=A + 8) == INVALID
    assert c(algo=2) == UNSUPPORTED      # no fused backward
    assert c(algo=4) == INVALID          # not an algorithm
    assert c(algo=3, dk_=48) == UNSUPPORTED
    assert c(dk_=48) == UNSUPPORTED
    assert c(T=-1) == INVALID
    assert c(q=None, k=None, v=None, la=None, beta=None, dout=None, dq=None,
             dk=None, dv=None, dla=None, db=None, gate=0, B=0) == OK


def test_backward_gdn2_rejects_bad_arguments(lib):
    def c(**kw):
        a = dict(q=A, k=A, v=A, la=A, er=A, wr=A, s0=None, dout=A, dsT=None,
                 dq=A, dk=A, dv=A, dla=A, de=A, dw=A, ds0=None, B=1, T=32,
                 H=1, dk_=64, dv_=64, gate=2, dtype=0, algo=0)
        a.update(kw)
        opts = gdr._Opts(a["dtype"], a["gate"], None, 0, a["algo"])
        return lib.gdr_backward_gdn2(
            a["q"], a["k"], a["v"], a["la"], a["er"], a["wr"], a["s0"],
            a["dout"], a["dsT"], a["dq"], a["dk"], a["dv"], a["dla"],
            a["de"], a["dw"], a["ds0"], a["B"], a["T"], a["H"], a["dk_"],
            a["dv_"], None, ctypes.byref(opts))
    # every case is rejected on the host, before any CUDA call
    assert c(er=None) == INVALID          # both gates are required
    assert c(wr=None) == INVALID
    assert c(de=None) == INVALID          # and both gate gradients
    assert c(dw=None) == INVALID
    assert c(dw=A + 4) == INVALID         # misaligned
    assert c(dout=None) == INVALID
    assert c(dla=None) == INVALID         # a decay gate needs its gradient
    assert c(algo=3) == UNSUPPORTED       # no token recurrence with gates
    assert c(algo=2) == UNSUPPORTED
    assert c(dk_=48) == UNSUPPORTED
    assert c(q=None, k=None, v=None, la=None, dout=None, dq=None, dk=None,
             dv=None, dla=None, gate=0, B=0) == OK


def test_backward_fg2_rejects_bad_arguments(lib):
    def c(**kw):
        a = dict(q=A, k=A, v=A, la=A, bk=A, bv=None, s0=None, dout=A,
                 dsT=None, dq=A, dk=A, dv=A, dla=A, dbk=A, dbv=None, ds0=None,
                 B=1, T=32, H=1, dk_=64, dv_=64, gate=2, dtype=0, algo=0)
        a.update(kw)
        opts = gdr._Opts(a["dtype"], a["gate"], None, 0, a["algo"])
        return lib.gdr_backward_fg2(
            a["q"], a["k"], a["v"], a["la"], a["bk"], a["bv"], a["s0"],
            a["dout"], a["dsT"], a["dq"], a["dk"], a["dv"], a["dla"],
            a["dbk"], a["dbv"], a["ds0"], a["B"], a["T"], a["H"], a["dk_"],
            a["dv_"], None, ctypes.byref(opts))
    # every case is rejected on the host, before any CUDA call
    assert c(bk=None) == INVALID          # the rate is required
    assert c(dbk=None) == INVALID         # and its gradient
    assert c(bv=A) == INVALID             # a value scaling needs its gradient
    assert c(dbv=A) == INVALID            # ... and its gradient needs it
    assert c(dbk=A + 4) == INVALID        # misaligned
    assert c(dla=None) == INVALID
    assert c(algo=3) == UNSUPPORTED       # no token recurrence with gates
    assert c(algo=2) == UNSUPPORTED
    assert c(dk_=48) == UNSUPPORTED
    assert c(q=None, k=None, v=None, la=None, dout=None, dq=None, dk=None,
             dv=None, dla=None, gate=0, B=0) == OK


def test_segmented_rejects_bad_arguments(lib):
    def c(segments=4, **kw):
        args = dict(q=A, k=A, v=A, la=A, beta=A, s0=None, out=A, sT=None, B=1,
                    T=64, H=1, dk=128, dv=128, chunk=64, dtype=0, gate=1,
                    cu=None, nseq=0, algo=0)
        args.update(kw)
        opts = gdr._Opts(args["dtype"], args["gate"], args["cu"], args["nseq"],
                         args["algo"])
        return lib.gdr_chunk_fwd_segmented(
            args["q"], args["k"], args["v"], args["la"], args["beta"],
            args["s0"], args["out"], args["sT"], args["B"], args["T"],
            args["H"], args["dk"], args["dv"], args["chunk"], segments, None,
            ctypes.byref(opts))
    assert c(segments=0) == INVALID
    assert c(segments=-3) == INVALID
    assert c(q=None) == INVALID
    assert c(dk=48) == UNSUPPORTED
    assert c(q=None, k=None, v=None, la=None, beta=None, out=None, gate=0,
             B=0) == OK


def test_gdn2_rejects_bad_arguments(lib):
    def c(**kw):
        args = dict(q=A, k=A, v=A, la=A, er=A, wr=A, s0=None, out=A, sT=None,
                    B=1, T=64, H=1, dk=128, dv=128, chunk=64, dtype=0, gate=2,
                    cu=None, nseq=0, algo=0)
        args.update(kw)
        opts = gdr._Opts(args["dtype"], args["gate"], args["cu"], args["nseq"],
                         args["algo"])
        return lib.gdr_chunk_fwd_gdn2(
            args["q"], args["k"], args["v"], args["la"], args["er"],
            args["wr"], args["s0"], args["out"], args["sT"], args["B"],
            args["T"], args["H"], args["dk"], args["dv"], args["chunk"], None,
            ctypes.byref(opts))
    assert c(er=None) == INVALID          # both gates are required
    assert c(wr=None) == INVALID
    assert c(wr=A + 4) == INVALID         # 16-byte alignment
    assert c(la=None) == INVALID          # a decay gate needs log_alpha
    # the fused path takes bf16 only (rejected before any CUDA call; the
    # cases it takes would launch, so they are not called with these
    # placeholder addresses)
    assert c(algo=2, dtype=1) == UNSUPPORTED
    assert c(dk=48) == UNSUPPORTED
    assert c(q=None, k=None, v=None, la=None, er=None, wr=None, out=None,
             gate=0, B=0) == OK


def test_fg2_rejects_bad_arguments(lib):
    def c(**kw):
        args = dict(q=A, k=A, v=A, la=A, bk=A, bv=None, s0=None, out=A,
                    sT=None, B=1, T=64, H=1, dk=128, dv=128, chunk=64,
                    dtype=0, gate=2, cu=None, nseq=0, algo=0)
        args.update(kw)
        opts = gdr._Opts(args["dtype"], args["gate"], args["cu"], args["nseq"],
                         args["algo"])
        return lib.gdr_chunk_fwd_fg2(
            args["q"], args["k"], args["v"], args["la"], args["bk"],
            args["bv"], args["s0"], args["out"], args["sT"], args["B"],
            args["T"], args["H"], args["dk"], args["dv"], args["chunk"], None,
            ctypes.byref(opts))
    assert c(bk=None) == INVALID          # the key-side rate is required
    assert c(bk=A + 4) == INVALID         # 16-byte alignment
    assert c(bv=A + 8) == INVALID
    assert c(la=None) == INVALID          # a decay gate needs log_alpha
    # the fused path takes bf16 only (rejected before any CUDA call)
    assert c(algo=2, dtype=1) == UNSUPPORTED
    assert c(algo=2, dtype=1, bv=A) == UNSUPPORTED
    assert c(dk=48) == UNSUPPORTED
    assert c(q=None, k=None, v=None, la=None, bk=None, out=None, gate=0,
             B=0) == OK


def test_decode_fg2_rejects_bad_arguments(lib):
    def c(**kw):
        args = dict(q=A, k=A, v=A, la=A, bk=A, bv=None, s0=None, s1=A, out=A,
                    N=1, H=1, dk=128, dv=128, dtype=0, gate=1, cu=None,
                    nseq=0, algo=0)
        args.update(kw)
        opts = gdr._Opts(args["dtype"], args["gate"], args["cu"], args["nseq"],
                         args["algo"])
        return lib.gdr_decode_step_fg2(
            args["q"], args["k"], args["v"], args["la"], args["bk"],
            args["bv"], args["s0"], args["s1"], args["out"], args["N"],
            args["H"], args["dk"], args["dv"], None, ctypes.byref(opts))
    assert c(bk=None) == INVALID          # the key-side rate is required
    assert c(bk=A + 4) == INVALID         # 16-byte alignment
    assert c(bv=A + 8) == INVALID
    assert c(la=None) == INVALID
    assert c(cu=A, nseq=1) == INVALID     # one token per sequence
    assert c(algo=2) == UNSUPPORTED
    assert c(dv=48) == UNSUPPORTED
    assert c(s0=A, s1=A + 64) == INVALID  # overlapping, not identical states
    assert c(q=None, k=None, v=None, la=None, s1=None, out=None, gate=0,
             N=0) == OK


def test_decode_gdn2_rejects_bad_arguments(lib):
    def c(**kw):
        args = dict(q=A, k=A, v=A, la=A, er=A, wr=A, s0=None, s1=A, out=A,
                    N=1, H=1, dk=128, dv=128, dtype=0, gate=1, cu=None,
                    nseq=0, algo=0)
        args.update(kw)
        opts = gdr._Opts(args["dtype"], args["gate"], args["cu"], args["nseq"],
                         args["algo"])
        return lib.gdr_decode_step_gdn2(
            args["q"], args["k"], args["v"], args["la"], args["er"],
            args["wr"], args["s0"], args["s1"], args["out"], args["N"],
            args["H"], args["dk"], args["dv"], None, ctypes.byref(opts))
    assert c(er=None) == INVALID          # both gates are required
    assert c(wr=None) == INVALID
    assert c(er=A + 4) == INVALID         # 16-byte alignment
    assert c(wr=A + 8) == INVALID
    assert c(la=None) == INVALID          # a decay gate needs log_alpha
    assert c(cu=A, nseq=1) == INVALID     # one token per sequence
    assert c(algo=2) == UNSUPPORTED
    assert c(dv=48) == UNSUPPORTED
    assert c(s0=A, s1=A + 64) == INVALID  # overlapping, not identical states
    assert c(q=None, k=None, v=None, la=None, s1=None, out=None, gate=0,
             N=0) == OK


def test_algo_applies(lib):
    assert gdr.algo_applies("staged", "fp32", "none", 16, 16, 16)
    assert gdr.algo_applies("auto", "bf16", "channel", 128, 64, 32)
    assert not gdr.algo_applies("staged", "bf16", "scalar", 48, 128, 64)
    assert not gdr.algo_applies("fused_tc", "fp32", "scalar", 128, 128, 64)
    assert not gdr.algo_applies("fused_tc", "bf16", "scalar", 64, 128, 64)
