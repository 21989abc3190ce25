"""Benchmark of libgdr's chunkwise gated-delta forward pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--algo auto|staged|fused_tc]
                    [--batch B] [--segments S] [--decode] [--backward]
                    [--gdn2 | --fg2]

One step = one gdr_chunk_fwd call over one batch of the workload (all four
stages: log-decay cumsum, WY/UT transform, state passing, output), inputs
resident in HBM.  Timing: W untimed warm-up steps, then K steps bracketed by a
barrier and a device synchronise, timed with CUDA events on the launching
stream; the max over ranks is reported.  The workload's inputs (>= 557 MB at
the headline size) exceed the 126 MB L2, so no flush is done between steps.

N > 1 (launched with torch.distributed.run): every rank runs its own full
workload on its own GPU (independent sequences, weak scaling); the only
collectives are the barrier and the max/gather of timings.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("tokens/s & TFLOP/s, chunked gated-delta fwd H16 d128 T4096 bf16; "
          "% roofline")
# nominal-figure fallback, used only without the measured file
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}


def flops_per_token_head(C, dk, dv):
    # six dense tile products per token-head: K K^T, T.K, Q K^T (2 C dk each),
    # T.V, P.V_new (2 C dv each), W.S, K^T.V_new, Q.S (2 dk dv each)
    return 6 * C * dk + 4 * C * dv + 6 * dk * dv


def algorithmic_bytes(w, ntok, nseq):
    """Bytes a step must move at least: q, k, v, out in the I/O dtype, beta
    and log-alpha in fp32, initial and final state in fp32."""
    esz = 4 if w.dtype == "fp32" else 2
    per_th = esz * (2 * w.dk + 2 * w.dv) + 4
    if w.gate == "scalar":
        per_th += 4
    elif w.gate == "channel":
        per_th += 4 * w.dk
    states = (2 if w.init_state else 1) * nseq * w.H * w.dk * w.dv * 4
    return ntok * w.H * per_th + states


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(algo):
    files = {"fused_tc": ["fused_tc.cu"],
             "staged": ["staged.cu"],
             "decode": ["decode.cu"]}.get(algo, [])
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "chunkwise_recurrence_b200", "csrc",
                                   f), "rb").read())
    return h.hexdigest()[:16]


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")
# the kernel whose DRAM traffic the roofline line reports, per path
TRAFFIC_KERNEL = {"fused_tc": "gdr_fused_tc_kernel",
                  "decode": "decode"}


def recorded_traffic(key, src_hash, path=TRAFFIC_JSON):
    """DRAM bytes per launch recorded for `key` ("<algo>:<workload>") from
    an ncu capture, if it was taken on the current kernel source (else
    None)."""
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(key)
    if not rec or rec.get("source_sha256_16") != src_hash:
        return None
    return float(rec["dram_bytes_per_launch"])


_BYTE_UNITS = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9,
               "Tbyte": 1e12, "KB": 1e3, "MB": 1e6, "GB": 1e9}


def traffic_from_ncu_csv(csv_path, kernel_regex):
    """Mean DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per
    captured launch of the kernels matching `kernel_regex`, from the output
    of `ncu --csv --metrics dram__bytes_read.sum,dram__bytes_write.sum`;
    and the number of launches."""
    import csv
    rows = list(csv.reader(l for l in open(csv_path) if l.startswith('"')))
    hdr = rows[0]
    per_launch = {}
    for r in rows[1:]:
        d = dict(zip(hdr, r))
        if not re.search(kernel_regex, d.get("Kernel Name", "")):
            continue
        if d.get("Metric Name") not in ("dram__bytes_read.sum",
                                        "dram__bytes_write.sum"):
            continue
        val = float(d["Metric Value"].replace(",", ""))
        val *= _BYTE_UNITS.get(d.get("Metric Unit", "byte"), 1.0)
        per_launch[d["ID"]] = per_launch.get(d["ID"], 0.0) + val
    if not per_launch:
        raise SystemExit(f"no dram__bytes rows for /{kernel_regex}/ in "
                         f"{csv_path}")
    return sum(per_launch.values()) / len(per_launch), len(per_launch)


def record_traffic(csv_path, algo, workload, command, path=TRAFFIC_JSON):
    """Writes the traffic of `algo` on `workload` from an ncu capture into
    the committed record, with the hash of the kernel source it was taken
    on (bench.py reports it only while that source is unchanged)."""
    by, n = traffic_from_ncu_csv(csv_path, TRAFFIC_KERNEL[algo])
    recs = json.load(open(path)) if os.path.exists(path) else {}
    recs[f"{algo}:{workload}"] = {
        "kernel": TRAFFIC_KERNEL[algo],
        "source_sha256_16": kernel_source_hash(algo),
        "dram_bytes_per_launch": by, "launches": n, "command": command}
    with open(path, "w") as f:
        json.dump(recs, f, indent=1, sort_keys=True)
        f.write("\n")
    return by


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "samples": 0}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]),
                             float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, x in enumerate(r[3])
                          if x.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def max_over_ranks(values, ws, device=None):
    """Element-wise max of a list of floats over all ranks (the timing
    reduction: a job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if ws > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(tokens_per_rank_step, ws, steps, max_ms):
    """Whole-job tokens/s: every rank processes its own batch each step."""
    return tokens_per_rank_step * ws * steps / (max_ms / 1e3)


def rank_seed(seed, rank):
    """Each rank draws its own independent batch."""
    return seed + rank


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def free_port():
    """A free TCP port on 127.0.0.1 for the ranks' rendezvous."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


def relaunch_command(argv, n, port):
    """This script as n ranks on one node (one process per GPU) under
    torch.distributed.run, rendezvous on 127.0.0.1."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
            "--master-port", str(port), os.path.abspath(__file__), *argv]


def launch_ranks(argv, n):
    """Runs the benchmark as n ranks and returns the launcher's exit code.
    A hard limit well above the ranks' own collective timeouts ends a run
    whose ranks wait on one another for good."""
    import subprocess
    env = dict(os.environ)
    env.setdefault("OMP_NUM_THREADS", "1")
    cmd = ["timeout", "-k", "60", "1800",
           *relaunch_command(argv, n, free_port())]
    return subprocess.run(cmd, env=env).returncode


def run_launch_check(args):
    """The multi-rank plumbing without a GPU: every rank joins a gloo group,
    the ranks' numbers go through the max-over-ranks reduction, and rank 0
    prints one JSON line with the world size it saw."""
    import torch.distributed as dist
    from datetime import timedelta
    ws, rank, _ = dist_env()
    if ws > 1:
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    ranks = max_over_ranks([float(r == rank) * (r + 1) for r in range(ws)],
                           ws)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"launch_check": True, "n_gpus": ws,
                          "ranks_seen": [int(x) - 1 for x in ranks]}),
              flush=True)
    return 0


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(inp, nseq_sample):
    """The first `nseq_sample` sequences of the workload (all heads), as
    oracle inputs, and their token count."""
    f = inp.f64()
    if f["cu_seqlens"] is None:
        for key in ("q", "k", "v", "beta", "log_alpha"):
            if f[key] is not None:
                f[key] = f[key][:nseq_sample]
        tokens = nseq_sample * inp.w.T
    else:
        tokens = int(f["cu_seqlens"][nseq_sample])
        for key in ("q", "k", "v", "beta", "log_alpha"):
            if f[key] is not None:
                f[key] = f[key][:, :tokens]
        f["cu_seqlens"] = f["cu_seqlens"][:nseq_sample + 1]
    if f["initial_state"] is not None:
        f["initial_state"] = f["initial_state"][:nseq_sample]
    return f, tokens


def time_oracle(inp, nseq_sample, nthreads=0):
    """The oracle on the first `nseq_sample` sequences (all heads), on
    `nthreads` host threads (0: all cores): tokens/s, threads, seconds,
    tokens."""
    import oracle
    f, tokens = oracle_sample(inp, nseq_sample)
    t0 = time.perf_counter()
    _, _, threads = oracle.gdr_fwd(**f, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return tokens / dt, threads, dt, tokens


def workload_config(w, inp):
    """The `config` object of a bench line: the workload and its sizes."""
    cfg = {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk,
           "dv": w.dv, "chunk": w.chunk, "gate": w.gate}
    if w.varlen_nseq:
        cfg.update(B=inp.nseq, T=None, total_tokens=inp.ntok,
                   lengths=list(inp.lengths))
    return cfg


def run_reference(args, w):
    """CPU oracle arm: rank 0 only, bounded sample per step."""
    from chunkwise_recurrence_b200.inputs import generate
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    inp = generate(w, seed=0)
    nsample = max(1, min(args.ref_seqs, len(inp.lengths)))
    for _ in range(args.warmup):
        time_oracle(inp, nsample)
    vals, total_tok, total_t, threads = [], 0, 0.0, 1
    for _ in range(args.steps):
        v, threads, dt, tok = time_oracle(inp, nsample)
        vals.append(v)
        total_tok += tok
        total_t += dt
    value = total_tok / total_t
    _, tok = oracle_sample(inp, nsample)
    sample = (f"sequences 0..{nsample - 1} of {len(inp.lengths)} "
              f"({tok} tokens x {w.H} heads) per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, inp),
        "cpu_baseline": {"value": value, "unit": "tokens/s",
                         "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def sampled_parity(inp, out, final_state, head=3):
    """The timed result against the fp64 oracle on one head of every
    sequence (the chains are independent, so a head is an exact
    sub-problem): max|gpu - oracle| / RMS(oracle) for out (less half an ulp
    of its storage dtype) and for the final state, beside the bar."""
    import oracle
    from chunkwise_recurrence_b200.inputs import head_slice, out_err, rel_err
    w = inp.w
    h = min(head, w.H - 1)
    ro, rs, _ = oracle.gdr_fwd(**head_slice(inp, [h]).f64())
    o = out.float().cpu().numpy()[:, :, [h]]
    st = final_state.cpu().numpy()[:, [h]]
    return {"head": h, "out_err": out_err(o, ro, w.dtype),
            "state_err": rel_err(st, rs),
            "bar": 1e-4 if w.dtype == "fp32" else 2e-2,
            "metric": "max |gpu - fp64 oracle| / RMS(oracle), all sequences "
                      "of one head; out less half an ulp of its dtype"}


def launches_per_step(algo_used, w, segments=0):
    one = 1 if algo_used == "fused_tc" else 4 + (0 if w.gate == "none" else 1)
    if segments:
        # three forward passes, the identity fill and the combine
        return 3 * one + 2
    return one


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import chunkwise_recurrence_b200 as gdr
    from chunkwise_recurrence_b200.inputs import generate

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    inp = generate(w, seed=rank_seed(args.seed, rank))
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    beta = inp.beta.to(dev)
    la = None if inp.log_alpha is None else inp.log_alpha.to(dev)
    s0 = None if inp.s0 is None else inp.s0.to(dev)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    out = torch.empty_like(v)
    sT = torch.empty(inp.nseq, w.H, w.dk, w.dv, dtype=torch.float32,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(s=stream):
        if args.segments:
            gdr.chunk_fwd_segmented(q, k, v, beta, la, s0,
                                    segments=args.segments, chunk=w.chunk,
                                    gate=w.gate, cu_seqlens=cu, out=out,
                                    final_state=sT, algo=args.algo,
                                    stream=s)
            return
        gdr.chunk_fwd(q, k, v, beta, la, s0, chunk=w.chunk, gate=w.gate,
                      cu_seqlens=cu, out=out, final_state=sT, algo=args.algo,
                      stream=s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdr.device_error() != 0:
        raise RuntimeError("device-side error during warm-up")
    # One step as a CUDA graph (the same launches, without the per-call host
    # work between steps); the context-parallel call reads the sequence
    # offsets on the host and runs directly.
    graph = None
    if not args.segments:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(torch.cuda.current_stream(dev))
            g.replay()
            torch.cuda.synchronize()
            if gdr.device_error() == 0:
                graph = g
        except RuntimeError:
            torch.cuda.synchronize()
            graph = None
    run_step = graph.replay if graph is not None else step
    algo_used = args.algo
    if algo_used == "auto":
        algo_used = ("fused_tc" if (w.dtype == "bf16" and w.dk == 128 and
                                    w.dv == 128 and w.chunk == 64 and
                                    gdr_fused_available())
                     else "staged")

    # ---- device-timed region (inputs resident in HBM)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_gpu_index(local)) as clocks:
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            run_step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    if gdr.device_error() != 0:
        raise RuntimeError("device-side error during timing")
    launch_mode = "cuda graph of one step" if graph is not None else "direct"
    del graph

    # ---- end to end through the host-buffer entry point
    pin = lambda t: None if t is None else t.pin_memory()  # noqa: E731
    hq, hk, hv, hb = pin(inp.q), pin(inp.k), pin(inp.v), pin(inp.beta)
    hla, hs0 = pin(inp.log_alpha), pin(inp.s0)
    hcu = pin(inp.cu_seqlens)
    hout = torch.empty_like(inp.v).pin_memory()
    hsT = torch.empty(inp.nseq, w.H, w.dk, w.dv).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in
              (hq, hk, hv, hb, hla, hs0, hcu) if t is not None)
    d2h = hout.numel() * hout.element_size() + hsT.numel() * 4

    def e2e_step():
        gdr.chunk_fwd_host(hq, hk, hv, hb, hla, hs0, out=hout,
                           final_state=hsT, chunk=w.chunk, gate=w.gate,
                           cu_seqlens=hcu, algo=args.algo, stream=stream)

    for _ in range(max(1, min(args.warmup, 3))):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(1, min(args.steps, 10))
    ea, eb = (torch.cuda.Event(enable_timing=True),
              torch.cuda.Event(enable_timing=True))
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ea.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ea.elapsed_time(eb)

    # ---- max over ranks
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], ws, device=dev)

    ntok = inp.ntok
    value = job_throughput(ntok, ws, args.steps, total_ms)
    e2e_value = job_throughput(ntok, ws, e2e_steps, e2e_ms)
    ms = total_ms / args.steps
    fl = flops_per_token_head(w.chunk, w.dk, w.dv) * ntok * w.H
    by = algorithmic_bytes(w, ntok, inp.nseq)
    peaks, peak_src = load_peaks()
    kernel_ms = statistics.mean(per_step)
    achieved_gbs = by / (kernel_ms / 1e3) / 1e9
    src_hash = kernel_source_hash(algo_used)
    traffic = recorded_traffic(f"{algo_used}:{w.name}", src_hash)
    roofline = {
        "bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
        "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
        "traffic": traffic,
        "peak_source": peak_src,
        "kernel": "gdr_fused_tc_kernel" if algo_used == "fused_tc"
        else "staged path (5 kernels, whole call)",
        "algorithmic_bytes_per_launch": by,
        "tflops": fl / (kernel_ms / 1e3) / 1e12,
        "tensor_frac": fl / (kernel_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
        "roofline_time_us": 1e6 * max(by / (peaks["hbm_gbs"] * 1e9),
                                      fl / (peaks["bf16_tflops"] * 1e12)),
    }
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic",
        "config": {**workload_config(w, inp),
                   "global_batch": inp.nseq * ws,
                   "seq_len": None if w.varlen_nseq else w.T,
                   "parallelism": f"dp{ws} (independent sequences)",
                   "algo": algo_used,
                   "segments": args.segments or None,
                   "l2": "inputs larger than L2 (no flush)",
                   "launch": launch_mode},
        "tflops": fl * ws / (ms / 1e3) / 1e12,
        "roofline": roofline,
        "clocks": clocks.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": h2d * ws, "d2h_bytes_per_step": d2h * ws,
                "entry": "gdr_chunk_fwd_host (pinned host buffers)"},
        "gpu_launches": launches_per_step(algo_used, w, args.segments) *
        args.steps,
        "ms_per_step_min": min(per_step), "ms_per_step_max": max(per_step),
        "ms_per_step_median": statistics.median(per_step),
    }
    if rank == 0:
        line["parity"] = sampled_parity(inp, out, sT)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        nsample = max(1, min(args.cpu_seqs, len(inp.lengths)))
        val, threads, dt, tok = time_oracle(inp, nsample)
        v1, _, dt1, tok1 = time_oracle(inp, 1, nthreads=1)
        line["cpu_baseline"] = {
            "value": val, "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": (f"sequences 0..{nsample - 1} of {len(inp.lengths)} "
                       f"({tok} tokens x {w.H} heads), {dt:.1f} s wall"),
            "single_core": {
                "value": v1, "unit": "tokens/s", "cores": 1,
                "sample": (f"sequence 0 of {len(inp.lengths)} ({tok1} tokens "
                           f"x {w.H} heads), {dt1:.1f} s wall")}}
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


DECODE_METRIC = ("tokens/s, single-token decode step (gdr_decode_step), GDN "
                 "H16 d128 bf16, state resident in HBM; % HBM roofline")
DECODE_GDN2_METRIC = ("tokens/s, single-token decode step with Gated "
                      "DeltaNet-2 gates (gdr_decode_step_gdn2), H16 d128 bf16, "
                      "state resident in HBM; % HBM roofline")


def decode_bytes(N, H, dk, dv, esz, gate, gdn2=False):
    """Bytes a decode step must move: the state read and written once (fp32),
    q, k, v, out in the I/O dtype, beta (or the erase and write gates) and
    log-alpha in fp32."""
    per = 2 * dk * dv * 4 + esz * (2 * dk + 2 * dv)
    per += 4 * (dk + dv) if gdn2 else 4
    per += {"none": 0, "scalar": 4, "channel": 4 * dk}[gate]
    return N * H * per


def run_decode(args):
    """One decode step per sequence per timed step: N sequences x H heads,
    the state updated in place in HBM (256 MiB at the default size, larger
    than L2, so no flush is needed)."""
    import torch

    import chunkwise_recurrence_b200 as gdr
    from chunkwise_recurrence_b200.inputs import Workload, generate

    ws, rank, local = dist_env()
    if ws > 1:
        raise SystemExit("--decode runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    N, H, d = args.decode_seqs, 16, 128
    g2 = args.gdn2
    w = Workload("gdn2_decode_h16_d128_bf16" if g2 else
                 "gdn_decode_h16_d128_bf16", B=N, T=1, H=H, dk=d, dv=d,
                 chunk=16, dtype="bf16", gate="scalar", decay_lo=0.01,
                 decay_hi=0.1, init_state=True)
    inp = generate(w, seed=args.seed)
    sq = lambda t: t[:, 0].contiguous()  # noqa: E731
    hq, hk, hv = sq(inp.q), sq(inp.k), sq(inp.v)
    hb, hla = sq(inp.beta), sq(inp.log_alpha)
    q, k, v, b, la = (t.to(dev) for t in (hq, hk, hv, hb, hla))
    if g2:
        from chunkwise_recurrence_b200.inputs import gdn2_gates
        her, hwr = (sq(t) for t in gdn2_gates(inp, seed=args.seed))
        er, wr = her.to(dev), hwr.to(dev)
    state = inp.s0.to(dev)
    out = torch.empty_like(v)
    stream = torch.cuda.current_stream(dev)

    def step():
        if g2:
            gdr.decode_step_gdn2(q, k, v, er, wr, la, state, out=out,
                                 stream=stream)
        else:
            gdr.decode_step(q, k, v, b, la, state, out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_gpu_index(local)) as clocks:
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    # end to end: the step's token inputs come from pinned host memory and
    # its outputs go back; the state stays resident on the device
    pin = lambda t: t.pin_memory()  # noqa: E731
    pairs = [(q, pin(hq)), (k, pin(hk)), (v, pin(hv)), (la, pin(hla))]
    pairs += ([(er, pin(her)), (wr, pin(hwr))] if g2 else [(b, pin(hb))])
    pout = torch.empty_like(hv).pin_memory()
    h2d = sum(t.numel() * t.element_size() for _, t in pairs)
    d2h = pout.numel() * pout.element_size()

    def e2e_step():
        for dst, src in pairs:
            dst.copy_(src, non_blocking=True)
        step()
        pout.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ea, eb = (torch.cuda.Event(enable_timing=True),
              torch.cuda.Event(enable_timing=True))
    ea.record(stream)
    for _ in range(args.steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ea.elapsed_time(eb)
    ms = total_ms / args.steps
    by = decode_bytes(N, H, d, d, 2, "scalar", gdn2=g2)
    peaks, peak_src = load_peaks()
    kernel_ms = statistics.mean(per_step)
    gbs = by / (kernel_ms / 1e3) / 1e9
    line = {
        "metric": DECODE_GDN2_METRIC if g2 else DECODE_METRIC,
        "value": N / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "sequences": N, "H": H, "dk": d,
                   "dv": d, "gate": "scalar",
                   "l2": f"state {N * H * d * d * 4 >> 20} MiB > L2 (no flush)"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "traffic": recorded_traffic(
                         f"decode:{w.name}", kernel_source_hash("decode")),
                     "peak_source": peak_src,
                     "kernel": "gdr_decode_kernel",
                     "algorithmic_bytes_per_launch": by},
        "clocks": clocks.summary(),
        "e2e": {"value": N * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "entry": ("gdr_decode_step_gdn2" if g2 else "gdr_decode_step")
                + ", token inputs from pinned host memory, state resident"},
        "gpu_launches": args.steps,
        "ms_per_step_min": min(per_step), "ms_per_step_max": max(per_step),
        "ms_per_step_median": statistics.median(per_step),
    }
    if not args.no_cpu_baseline:
        import oracle
        ns = min(N, 32)
        f = lambda t: t[:ns].double().numpy()  # noqa: E731
        t0 = time.perf_counter()
        if g2:
            u = lambda t: t[:ns, None].double().numpy()  # noqa: E731
            oracle.gdn2_fwd(u(hq), u(hk), u(hv), u(her), u(hwr), u(hla),
                            "scalar", f(inp.s0))
            cores = 1   # a numpy token loop on one thread
        else:
            oracle.decode_step(f(hq), f(hk), f(hv), f(hb), f(hla),
                               gate="scalar", state=f(inp.s0))
            cores = cpu_cores()
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {
            "value": ns / dt, "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"sequences 0..{ns - 1} of {N} (x {H} heads), one step"}
    print(json.dumps(line), flush=True)
    return 0


BACKWARD_METRIC = ("tokens/s, backward pass (gdr_backward) of the chunked "
                   "gated-delta fwd; % fp32 ALU roofline")
# reverse token recurrence: fp32 flops per state element, token and head over
# its three sweeps: forward and replay 5 each (decay, S~^T k, k u^T), reverse 19
BACKWARD_FLOPS_PER_ELEM = 29


def chunked_backward_flops_per_chunk(dk, dv, C=64):
    """fp32 flops of one (chunk, head) of the chunked backward, from its
    products (multiply-adds x 2): 9 C dk dv (W S and the state update in the
    forward scan; Kc Lambda, Qd^T dO, W^T dV_new in the reverse scan;
    (K e^g) S and the three slice products dO S^T, Z S^T, V_new Lambda^T in
    the gradient kernel), C^2 (7 dk + 4.5 dv) (A, W, U in the WY kernel; P;
    P^T dO; Z, dT, dP; M and the four key/query products of A and P) and
    2.17 C^3 (the inverse, T^T dT, dA)."""
    return 2 * (9 * C * dk * dv + C * C * (7 * dk + 4.5 * dv)
                + 2.17 * C ** 3)


def run_backward(args, w):
    """Backward pass of the workload: upstream gradients of out and of the
    final state in, gradients of every input out."""
    import torch

    import chunkwise_recurrence_b200 as gdr
    from chunkwise_recurrence_b200.inputs import generate

    ws, rank, local = dist_env()
    if ws > 1:
        raise SystemExit("--backward runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    inp = generate(w, seed=args.seed)
    g = torch.Generator().manual_seed(args.seed + 1)
    dO = torch.randn(inp.v.shape, generator=g).to(inp.v.dtype).to(dev)
    dS = (torch.randn(inp.nseq, w.H, w.dk, w.dv, generator=g) * 0.1).to(dev)
    c = lambda t: None if t is None else t.to(dev)  # noqa: E731
    q, k, v, b, la, s0, cu = (c(t) for t in (inp.q, inp.k, inp.v, inp.beta,
                                             inp.log_alpha, inp.s0,
                                             inp.cu_seqlens))
    stream = torch.cuda.current_stream(dev)

    # --algo auto / staged: the chunked backward (gdr_backward's AUTO);
    # recurrent: the reverse token recurrence.  --gdn2: gdr_backward_gdn2
    # with Gated DeltaNet-2's erase and write gates (chunked only)
    algo = "recurrent" if args.algo == "recurrent" else "auto"
    g2 = args.gdn2
    if g2:
        if algo == "recurrent":
            raise SystemExit("--gdn2 --backward runs the chunked backward")
        from chunkwise_recurrence_b200.inputs import gdn2_gates
        er, wr = (t.to(dev) for t in gdn2_gates(inp, seed=args.seed))

    def step():
        if g2:
            return gdr.backward_gdn2(q, k, v, er, wr, la, s0, dO, dS,
                                     gate=w.gate, cu_seqlens=cu,
                                     stream=stream)
        return gdr.backward(q, k, v, b, la, s0, dO, dS, gate=w.gate,
                            cu_seqlens=cu, stream=stream, algo=algo)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_gpu_index(local)) as clocks:
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    ms = ev[0].elapsed_time(ev[-1]) / args.steps
    ntok, H, dk, dv = inp.ntok, w.H, w.dk, w.dv
    esz = 4 if w.dtype == "fp32" else 2
    la_b = {"none": 0, "scalar": 4, "channel": 4 * dk}[w.gate]
    # inputs (q, k, v, d_out in the I/O dtype, beta, log-alpha) read once,
    # gradients (fp32) written once, states in and out
    by = ntok * H * (esz * (2 * dk + 2 * dv) + 4 + la_b +
                     4 * (2 * dk + dv) + 4 + la_b)
    if g2:   # the gates read and their gradients written, in place of beta's
        by += ntok * H * (2 * 4 * (dk + dv) - 8)
    by += inp.nseq * H * dk * dv * 4 * (2 + (1 if inp.s0 is not None else 0))
    gbs = by / (statistics.mean(per_step) / 1e3) / 1e9
    cols = dk >= 32 and dv >= 32   # the column-split kernel + its reduction
    clk = clocks.summary()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    max_mhz = clk.get("sm_max_mhz") or 1965.0
    # CUDA-core fp32 peak: SMs x 128 lanes x 2 flops (FMA) x max SM clock
    alu_peak = sms * 128 * 2 * max_mhz * 1e6 / 1e12
    if algo == "recurrent":
        flops = BACKWARD_FLOPS_PER_ELEM * dk * dv * ntok * H
        kernel = "gdr_bwd_cols_kernel" if cols else "gdr_bwd_kernel"
        launches = 2 if cols else 1
        algo_name = "reverse token recurrence"
    else:
        nchunks = sum((n + 63) // 64 for n in inp.lengths)
        flops = chunked_backward_flops_per_chunk(dk, dv) * nchunks * H
        kernel = ("chunked backward, whole call (WY, state maps, two "
                  "scans, V_new, gradient kernels)")
        # chunk table, cumsum (with a gate), WY, prep, two scans, V_new,
        # gradients
        launches = 7 + (0 if w.gate == "none" else 1)
        algo_name = "chunked (64-token chunks, fp32)" + (
            ", Gated DeltaNet-2 gates" if g2 else "")
    tflops = flops / (statistics.mean(per_step) / 1e3) / 1e12
    line = {
        "metric": BACKWARD_METRIC, "value": ntok / (ms / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {**workload_config(w, inp), "algo": algo_name,
                   "l2": "inputs larger than L2 (no flush)"},
        "roofline": {"bound": "alu", "achieved": tflops, "peak": alu_peak,
                     "unit": "TFLOP/s", "frac": tflops / alu_peak,
                     "traffic": None,
                     "peak_source": f"derived: {sms} SMs x 128 fp32 lanes x 2 "
                                    f"x {max_mhz:.0f} MHz",
                     "kernel": kernel,
                     "flops_per_step": flops,
                     "hbm_gbs_on_algorithmic_bytes": gbs,
                     "algorithmic_bytes_per_launch": by},
        "clocks": clk,
        "gpu_launches": args.steps * launches,
        "ms_per_step_min": min(per_step), "ms_per_step_max": max(per_step),
        "ms_per_step_median": statistics.median(per_step),
    }
    print(json.dumps(line), flush=True)
    return 0


GDN2_METRIC = ("tokens/s, chunked forward with Gated DeltaNet-2 erase and "
               "write gates (gdr_chunk_fwd_gdn2); % HBM roofline")
FG2_METRIC = ("tokens/s, chunked forward with FG^2-GDN+ per-key-channel rate "
              "and per-value-channel target scaling (gdr_chunk_fwd_fg2); "
              "% HBM roofline")

# per gate variant: metric, the gate generator's name in inputs, the binding,
# the C entry, the oracle's token loop, and what the two gate tensors are
TWO_GATES = {
    "gdn2": (GDN2_METRIC, "gdn2_gates", "chunk_fwd_gdn2",
             "gdr_chunk_fwd_gdn2", "gdn2_fwd",
             "erase [.., dk], write [.., dv], sigmoid(N(0,1))"),
    "fg2": (FG2_METRIC, "fg2_gates", "chunk_fwd_fg2", "gdr_chunk_fwd_fg2",
            "fg2_fwd",
            "key-side rate [.., dk], value-side scaling [.., dv], "
            "sigmoid(N(0,1))"),
}


def run_gdn2(args, w, kind="gdn2"):
    """The workload's forward pass with two per-channel gate tensors in place
    of beta: Gated DeltaNet-2's erase and write gates (kind "gdn2") or
    FG^2-GDN+'s key-side rate and value-side scaling (kind "fg2"); the fused
    kernel with the channel-wise decay, else the staged path."""
    import torch

    import chunkwise_recurrence_b200 as gdr
    from chunkwise_recurrence_b200 import inputs as inputs_mod
    from chunkwise_recurrence_b200.inputs import generate

    metric, gen_name, fn_name, entry, oracle_name, gate_desc = TWO_GATES[kind]
    ws, rank, local = dist_env()
    if ws > 1:
        raise SystemExit(f"--{kind} runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    inp = generate(w, seed=args.seed)
    her, hwr = getattr(inputs_mod, gen_name)(inp, seed=args.seed)
    fwd = getattr(gdr, fn_name)
    host = dict(q=inp.q, k=inp.k, v=inp.v, er=her, wr=hwr,
                la=inp.log_alpha, s0=inp.s0, cu=inp.cu_seqlens)
    d = {n: None if t is None else t.to(dev) for n, t in host.items()}
    out = torch.empty_like(d["v"])
    sT = torch.empty(inp.nseq, w.H, w.dk, w.dv, dtype=torch.float32,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    # the fused kernel takes these gates for bf16, d = 128, C = 64 (a scalar
    # or absent decay as the channel-wise one with all channels equal);
    # every other shape runs the staged path
    algo_used = args.algo
    if algo_used == "auto":
        algo_used = ("fused_tc" if (w.dtype == "bf16" and w.dk == 128 and
                                    w.dv == 128 and w.chunk == 64 and
                                    gdr_fused_available())
                     else "staged")

    def step():
        fwd(d["q"], d["k"], d["v"], d["er"], d["wr"], d["la"], d["s0"],
            chunk=w.chunk, gate=w.gate, cu_seqlens=d["cu"], out=out,
            final_state=sT, stream=stream, algo=algo_used)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_gpu_index(local)) as clocks:
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    if gdr.device_error() != 0:
        raise RuntimeError("device-side error during timing")
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    ms = ev[0].elapsed_time(ev[-1]) / args.steps
    # end to end: every input from pinned host memory, out and the final
    # state back, through the same device entry point
    pinned = {n: None if t is None else t.pin_memory()
              for n, t in host.items()}
    hout = torch.empty_like(inp.v).pin_memory()
    hsT = torch.empty(inp.nseq, w.H, w.dk, w.dv).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values()
              if t is not None)
    d2h = hout.numel() * hout.element_size() + hsT.numel() * 4

    def e2e_step():
        for n, t in pinned.items():
            if t is not None:
                d[n].copy_(t, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
        hsT.copy_(sT, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(1, min(args.steps, 10))
    ea, eb = (torch.cuda.Event(enable_timing=True),
              torch.cuda.Event(enable_timing=True))
    ea.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ea.elapsed_time(eb)
    ntok, H, dk, dv = inp.ntok, w.H, w.dk, w.dv
    esz = 4 if w.dtype == "fp32" else 2
    la_b = {"none": 0, "scalar": 4, "channel": 4 * dk}[w.gate]
    # q, k, v, out in the I/O dtype, the two gates and log-alpha in fp32,
    # each read or written once; the states in and out
    by = ntok * H * (esz * (2 * dk + 2 * dv) + 4 * (dk + dv) + la_b)
    by += inp.nseq * H * dk * dv * 4 * (1 + (1 if inp.s0 is not None else 0))
    peaks, peak_src = load_peaks()
    gbs = by / (statistics.mean(per_step) / 1e3) / 1e9
    line = {
        "metric": metric, "value": ntok / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {**workload_config(w, inp), "algo": algo_used,
                   "gates": gate_desc,
                   "l2": "inputs larger than L2 (no flush)",
                   "launch": "direct"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "traffic": None, "peak_source": peak_src,
                     "kernel": ("gdr_fused_tc_kernel" if algo_used == "fused_tc"
                                else "staged path (whole call)"),
                     "algorithmic_bytes_per_launch": by},
        "clocks": clocks.summary(),
        "e2e": {"value": ntok * e2e_steps / (e2e_ms / 1e3),
                "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "entry": f"{entry}, inputs copied from pinned host "
                         "memory and results back each step"},
        "gpu_launches": launches_per_step(algo_used, w) * args.steps,
        "ms_per_step_min": min(per_step), "ms_per_step_max": max(per_step),
        "ms_per_step_median": statistics.median(per_step),
    }
    if not args.no_cpu_baseline:
        import oracle
        f = lambda t, n: None if t is None else t[:n].double().numpy()  # noqa
        n = 1
        t0 = time.perf_counter()
        getattr(oracle, oracle_name)(
            f(inp.q, n), f(inp.k, n), f(inp.v, n), f(her, n), f(hwr, n),
            f(inp.log_alpha, n), w.gate, f(inp.s0, n))
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {
            "value": n * w.T / dt, "unit": "tokens/s", "cores": 1,
            "kind": "oracle",
            "sample": f"sequence 0 of {inp.nseq} ({w.T} tokens x {H} heads), "
                      "numpy token loop on one thread"}
    print(json.dumps(line), flush=True)
    return 0


def gdr_fused_available():
    from chunkwise_recurrence_b200 import fused_tc_available
    return fused_tc_available()


def local_gpu_index(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x for x in vis.split(",") if x.strip()]
        if local < len(ids):
            return ids[local]
    return local


def main(argv=None):
    from chunkwise_recurrence_b200.inputs import HEADLINE, WORKLOADS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=list(WORKLOADS))
    ap.add_argument("--algo", default="auto",
                    choices=["auto", "staged", "fused_tc", "recurrent"],
                    help="with --backward: auto / staged = the chunked "
                         "backward, recurrent = the reverse token recurrence")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seqs", type=int, default=4,
                    help="sequences in the CPU-baseline sample")
    ap.add_argument("--ref-seqs", type=int, default=2,
                    help="sequences per step in the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode", action="store_true",
                    help="time the single-token decode step instead")
    ap.add_argument("--decode-seqs", type=int, default=256,
                    help="sequences per decode step")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (gdr_backward) instead")
    ap.add_argument("--batch", type=int, default=0,
                    help="run a fixed-length workload with this many "
                         "sequences instead of its own")
    ap.add_argument("--segments", type=int, default=0,
                    help="context-parallel forward (gdr_chunk_fwd_segmented) "
                         "with this many pieces per sequence")
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="record the DRAM traffic of --algo (fused_tc or "
                         "decode) on --workload from an ncu --csv capture "
                         "into profiles/traffic.json, and exit")
    ap.add_argument("--capture-command", default="",
                    help="with --record-traffic: the command that made it")
    ap.add_argument("--launch-check", action="store_true",
                    help="check the multi-rank launcher on CPU (gloo ranks, "
                         "no GPU work)")
    ap.add_argument("--gdn2", action="store_true",
                    help="with Gated DeltaNet-2 erase and write gates "
                         "(gdr_chunk_fwd_gdn2; with --decode, "
                         "gdr_decode_step_gdn2)")
    ap.add_argument("--fg2", action="store_true",
                    help="with FG^2-GDN+'s per-key-channel rate and "
                         "per-value-channel target scaling "
                         "(gdr_chunk_fwd_fg2)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if args.record_traffic:
        algo = "decode" if args.decode else args.algo
        if algo not in TRAFFIC_KERNEL:
            raise SystemExit("--record-traffic takes --algo fused_tc or "
                             "--decode")
        wname = "gdn_decode_h16_d128_bf16" if args.decode else args.workload
        by = record_traffic(args.record_traffic, algo, wname,
                            args.capture_command)
        print(json.dumps({"recorded": f"{algo}:{wname}",
                          "dram_bytes_per_launch": by}))
        return 0
    # --gpus N runs N ranks, one per GPU: launched here unless a launcher
    # (torch.distributed.run) already did, in which case the two must agree
    if "WORLD_SIZE" not in os.environ:
        if args.gpus > 1:
            return launch_ranks(sys.argv[1:] if argv is None else list(argv),
                                args.gpus)
    elif int(os.environ["WORLD_SIZE"]) != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE="
                         f"{os.environ['WORLD_SIZE']}")
    if args.launch_check:
        return run_launch_check(args)
    w = WORKLOADS[args.workload]
    if args.batch:
        if w.varlen_nseq or args.batch < 1:
            raise SystemExit("--batch needs a fixed-length workload and B >= 1")
        w = w.with_(B=args.batch, name=f"{w.name}@B{args.batch}")
    if args.algo == "recurrent" and not args.backward:
        raise SystemExit("--algo recurrent is a backward algorithm")
    if args.fg2 and (args.decode or args.backward):
        raise SystemExit("--fg2 times the chunked forward pass only")
    if args.decode and args.impl == "ours":
        return run_decode(args)
    if args.backward and args.impl == "ours":
        return run_backward(args, w)
    if (args.gdn2 or args.fg2) and args.impl == "ours":
        kind = "gdn2" if args.gdn2 else "fg2"
        if args.gdn2 and args.fg2:
            raise SystemExit("--gdn2 and --fg2 are exclusive")
        if w.varlen_nseq:
            raise SystemExit(f"--{kind} takes a fixed-length workload")
        return run_gdn2(args, w, kind)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
