"""bench.py's host arithmetic without a GPU: the roofline's FLOP and byte
counts at the headline chunk, the roofline time against the measured peaks,
and the rule that the committed DRAM-traffic figure is reported only for the
kernel source it was captured on.

The expected numbers are written out from their definitions: F = 6 H I P
(gate, up and down, two FLOPs per multiply-add), the gate/up part 4 H I P;
B = touched experts x bytes per expert + x (bf16) + logits (fp32) + y (fp32);
an expert of format Q2 at H=2048, I=512 holds 2 x 512 rows x 8 blocks (gate,
up) plus 2048 rows x 2 blocks (down) of 69 bytes.
"""
import json
import os
import shutil

import pytest

import bench
from bit_routed_expert_top_b200 import synth

HEADLINE = synth.WORKLOADS[synth.HEADLINE]


def test_headline_is_the_2048_token_q2_chunk():
    wl = HEADLINE
    assert (wl.T, wl.H, wl.I, wl.E, wl.k, wl.fmt) == (2048, 2048, 512, 512, 10, synth.FMT_Q2)
    assert wl.pairs == 20480                     # the pages' 20,480 token/expert pairs


def test_layer_model_counts():
    m = bench.layer_model(HEADLINE, 512)
    P = 2048 * 10
    assert m["flops"] == 6 * 2048 * 512 * P == 128_849_018_880
    assert m["flops_gu"] == 4 * 2048 * 512 * P
    expert = (2 * 512 * 8 + 2048 * 2) * 69
    assert expert == 847_872 == synth.expert_bytes(synth.FMT_Q2, 2048, 512)
    act = 2 * 2048 * 2048 + 4 * 2048 * 512 + 4 * 2048 * 2048
    assert m["bytes"] == 512 * expert + act == 463_470_592
    # fewer touched experts: only the weight term shrinks
    assert bench.layer_model(HEADLINE, 100)["bytes"] == 100 * expert + act


def test_roofline_time_against_measured_peaks():
    m = bench.layer_model(HEADLINE, 512)
    t_f = m["flops"] / 1630.4e12
    t_b = m["bytes"] / 6540.2e9
    assert t_f == pytest.approx(79.03e-6, rel=1e-3)       # tensor bound
    assert t_b == pytest.approx(70.87e-6, rel=1e-3)
    assert max(t_f, t_b) == t_f


def test_traffic_reported_only_for_the_captured_source(tmp_path):
    kernel = os.path.join(bench.ROOT, "bit_routed_expert_top_b200", "csrc", "gemm_tc.cuh")
    with open(os.path.join(bench.ROOT, "profiles", "gateup_traffic.json")) as f:
        rec = json.load(f)
    same = rec["source_sha256_16"] == bench.source_hash(kernel)
    assert bench.read_traffic(kernel) == (rec["dram_bytes_per_launch"] if same else None)
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"]
    changed = tmp_path / "gemm_tc.cuh"
    shutil.copy(kernel, changed)
    with open(changed, "ab") as f:
        f.write(b"\n// edited\n")
    assert bench.read_traffic(str(changed)) is None


def test_replica_throughput():
    # 2 replicas x 4 steps x 20,480 pairs in 10 ms (slowest rank) = 16.384 M pairs/s
    assert bench.replica_throughput(2, 4, 20480, 10.0) == pytest.approx(16.384e6)
