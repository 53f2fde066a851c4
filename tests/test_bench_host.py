"""Host-side arithmetic and bookkeeping of bench.py (no GPU): the algorithmic bytes and
flops each workload's roofline divides by, and the staleness check of the committed
DRAM-traffic figures."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

WORKLOADS = ["retnet_1p3b", "retnet_6p7b_long", "gated", "decode", "gated_decode", "seqpar_6p7b", "backward_1p3b",
             "backward_gated", "msr_norm_1p3b", "retention_msr_1p3b"]


def test_backward_and_epilogue_arithmetic():
    B, H, N, dk, dv, C = 4, 8, 2048, 256, 512, 64
    bw = bench.workload("backward_1p3b")
    # read q, k, v, dO and write dq, dk, dv once (bf16)
    assert bw["bytes"] == B * H * N * (dk + dk + dv + dv + dk + dk + dv) * 2
    assert bw["flops"] == 3 * B * H * N * (2 * C * (dk + dv) + 4 * dk * dv)
    assert bw["units"] == B * N and bw["kind"] == "backward"
    # gated backward (B2 H8 N16384 dk = dv = 128): the same tensors, plus g read and dg written in fp32
    gb = bench.workload("backward_gated")
    Bg, Hg, Ng, d = 2, 8, 16384, 128
    assert gb["bytes"] == Bg * Hg * Ng * 7 * d * 2 + 2 * Bg * Hg * Ng * 4 and gb["gated"] and not bw["gated"]
    nm = bench.workload("msr_norm_1p3b")
    assert nm["bytes"] == 3 * B * H * N * dv * 2  # o and gate in, y out
    rm = bench.workload("retention_msr_1p3b")
    # q, k, v and the gate in, y out; o is an intermediate
    assert rm["bytes"] == B * H * N * (2 * dk + dv) * 2 + 2 * B * H * N * dv * 2
    gd = bench.workload("gated_decode")
    assert gd["bytes"] == bench.workload("decode")["bytes"] + 64 * 16 * 4  # plus the step's g [B, H]
    sp = bench.workload("seqpar_6p7b")
    assert sp["bytes"] == bench.workload("retnet_6p7b_long")["bytes"] and sp["kind"] == "seqpar"


def test_every_workload_has_sources_and_a_cli_choice():
    csrc = os.path.join(ROOT, "linear_attention_ret_b200", "csrc")
    for w in WORKLOADS:
        group = bench.WORKLOAD_KERNELS[w]
        for f in bench.KERNEL_SOURCES[group]:
            assert os.path.exists(os.path.join(csrc, f)), f
        assert len(bench.kernel_source_sha(w)) == 16
    # the command line accepts exactly these workloads, and each has its arithmetic
    assert sorted(bench.WORKLOAD_KERNELS) == sorted(WORKLOADS)
    for w in WORKLOADS:
        spec = bench.workload(w)
        assert spec["unit"] in ("tokens/s", "steps/s") and spec["bytes"] > 0


def test_traffic_records_are_well_formed_and_reported_only_while_current():
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    for w in WORKLOADS:
        r = rec[w]
        assert r["traffic_bytes_per_launch"] > 0 and r["kernel"]
        # a figure is reported only while the measured kernel's sources hash as at capture
        assert bench.ncu_traffic(w) == (r["traffic_bytes_per_launch"] if r["source_sha"] == bench.kernel_source_sha(w)
                                        else None)


def test_default_line_covers_every_headline_workload():
    # the default run's line carries the decode step, the 6.7B-shaped sequence and the gated
    # form as sub-records beside the 1.3B-shaped headline, each with its own roofline
    assert set(bench.DEFAULT_ALSO) == {"decode", "retnet_6p7b_long", "gated"}
    for w in bench.DEFAULT_ALSO:
        assert w in bench.WORKLOAD_KERNELS
    # the dtype field names the inputs' arithmetic type, per workload
    from linear_attention_ret_b200 import inputs as I
    assert bench.dtype_name(I.CONFIGS["retnet_1p3b"]) == "bf16"
    assert bench.dtype_name(I.CONFIGS["tiny"]) == "f32"
    d = bench.workload("decode")
    assert d["unit"] == "steps/s" and d["bytes"] == 2 * 64 * 16 * 256 * 512 * 4 + 64 * 16 * (2 * 256 + 2 * 512) * 2
