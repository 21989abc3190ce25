"""Host-side arithmetic of bench.py (no GPU): the algorithmic bytes and
flops behind every roofline figure, the launch counts it claims, and the
rule that a profile's DRAM traffic is reported only while the profiled
source is unchanged.

The expected figures are the per-unit counts of the chunked forward pass:
q, k, v, out in the I/O dtype, beta and the log-decay in fp32, each read or
written once, plus the fp32 states; and the six dense tile products per
token-head (K K^T, T K and Q K^T at 2 C dk flops each, T V and the masked
(Q K^T) V_new at 2 C dv, and W S, K^T V_new and Q S at 2 dk dv)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from chunkwise_recurrence_b200.inputs import WORKLOADS  # noqa: E402


def test_flops_per_token_head():
    # 6 C dk + 4 C dv + 6 dk dv at C = 64, dk = dv = 128
    assert bench.flops_per_token_head(64, 128, 128) == 180224
    assert bench.flops_per_token_head(16, 16, 16) == 6 * 256 + 4 * 256 + 6 * 256


def test_algorithmic_bytes_of_the_workloads():
    # headline: 524 288 token-heads x 1032 B + initial and final state
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"]
    assert w.init_state
    assert bench.algorithmic_bytes(w, 8 * 4096, 8) == (
        8 * 4096 * 16 * 1032 + 2 * 8 * 16 * 128 * 128 * 4)
    assert bench.algorithmic_bytes(w, 8 * 4096, 8) == 557842432
    # KDA: the log-decay per key channel (1540 B per token-head), zero
    # initial state (final state only)
    k = WORKLOADS["kda_b4_h16_t4096_d128_bf16"]
    assert not k.init_state
    assert bench.algorithmic_bytes(k, 4 * 4096, 4) == (
        4 * 4096 * 16 * 1540 + 4 * 16 * 128 * 128 * 4)


def test_decode_bytes():
    # state in and out (2 x 64 KiB), q, k, v, out in bf16 (1 KiB), beta and
    # a scalar log-decay (8 B) per (sequence, head)
    assert bench.decode_bytes(256, 16, 128, 128, 2, "scalar") == 541097984
    assert bench.decode_bytes(1, 1, 128, 128, 2, "scalar") == (
        2 * 65536 + 1024 + 8)
    # Gated DeltaNet-2: an erase gate per key channel and a write gate per
    # value channel in place of beta
    assert bench.decode_bytes(1, 1, 128, 128, 2, "scalar", gdn2=True) == (
        2 * 65536 + 1024 + 4 * 256 + 4)
    assert bench.decode_bytes(256, 16, 128, 128, 2, "scalar",
                              gdn2=True) == 545275904


def test_launches_per_step():
    w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"]
    assert bench.launches_per_step("fused_tc", w) == 1
    # chunk table, cumsum, WY, state, output
    assert bench.launches_per_step("staged", w) == 5
    d = WORKLOADS["deltanet_b1_h1_t256_d16_fp32"]
    assert d.gate == "none"
    assert bench.launches_per_step("staged", d) == 4   # no cumsum
    # three forward passes, the identity fill and the combine
    assert bench.launches_per_step("fused_tc", w, segments=4) == 5


def _ncu_csv(path, rows):
    hdr = ['"ID"', '"Kernel Name"', '"Metric Name"', '"Metric Unit"',
           '"Metric Value"']
    with open(path, "w") as f:
        f.write("==PROF== a line ncu prints that is not data\n")
        f.write(",".join(hdr) + "\n")
        for r in rows:
            f.write(",".join(f'"{x}"' for x in r) + "\n")


def test_traffic_from_an_ncu_capture(tmp_path):
    # two captured launches of the kernel (units as ncu prints them) and a
    # launch of another kernel that must not count
    p = tmp_path / "cap.csv"
    _ncu_csv(p, [
        ("0", "void gdr::gdr_fused_tc_kernel<1>(...)", "dram__bytes_read.sum",
         "Mbyte", "400.5"),
        ("0", "void gdr::gdr_fused_tc_kernel<1>(...)", "dram__bytes_write.sum",
         "byte", "1,000"),
        ("1", "void gdr::gdr_fused_tc_kernel<1>(...)", "dram__bytes_read.sum",
         "Mbyte", "399.5"),
        ("1", "void gdr::gdr_fused_tc_kernel<1>(...)", "dram__bytes_write.sum",
         "Kbyte", "3"),
        ("2", "fill_kernel", "dram__bytes_read.sum", "Gbyte", "9"),
    ])
    by, n = bench.traffic_from_ncu_csv(str(p), "gdr_fused_tc_kernel")
    assert n == 2
    assert by == (400.5e6 + 1000 + 399.5e6 + 3e3) / 2


def test_recorded_traffic_follows_the_source_hash(tmp_path):
    p = tmp_path / "cap.csv"
    _ncu_csv(p, [("0", "gdr_fused_tc_kernel", "dram__bytes_read.sum", "byte",
                  "100"),
                 ("0", "gdr_fused_tc_kernel", "dram__bytes_write.sum", "byte",
                  "20")])
    rec = tmp_path / "traffic.json"
    assert bench.record_traffic(str(p), "fused_tc", "w", "ncu ...",
                                path=str(rec)) == 120.0
    h = bench.kernel_source_hash("fused_tc")
    assert len(h) == 16
    assert bench.recorded_traffic("fused_tc:w", h, path=str(rec)) == 120.0
    # a record taken on other source is not reported
    assert bench.recorded_traffic("fused_tc:w", "0" * 16, path=str(rec)) is None
    assert bench.recorded_traffic("fused_tc:other", h, path=str(rec)) is None
    assert bench.recorded_traffic("fused_tc:w", h,
                                  path=str(tmp_path / "none.json")) is None
