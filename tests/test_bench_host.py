"""Host-side arithmetic of bench.py (no GPU): the algorithmic byte counts the
roofline divides by, the input ring that keeps every timed step's inputs out
of L2, and the gate that drops an ncu traffic figure once the kernel sources
it was measured on have changed."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from rotation_w4a4_quantization_b200 import synthetic as syn  # noqa: E402


def alg_bytes(name):
    c = syn.WORKLOADS[name]
    return c["M"] * c["K"] * 2 + bench.code_bytes(c["fmt"], c["M"], c["K"])


@pytest.mark.parametrize("name, expected", [
    # bf16 X read + packed codes + per-row fp32 scale / per-16 or per-32 byte scales
    ("q_proj_int4", 2048 * 4096 * 2 + 2048 * 2048 + 2048 * 4),
    ("down_proj_int4", 4096 * 12288 * 2 + 4096 * 6144 + 4096 * 4),
    ("q_proj_nvfp4", 2048 * 4096 * 2 + 2048 * 2048 + 2048 * 256),
    ("q_proj_mxfp4", 2048 * 4096 * 2 + 2048 * 2048 + 2048 * 128),
    ("q_proj_w4a8", 2048 * 4096 * 2 + 2048 * 4096 + 2048 * 4),
])
def test_algorithmic_bytes(name, expected):
    assert alg_bytes(name) == expected


def test_algorithmic_bytes_match_the_stated_per_launch_figures():
    assert alg_bytes("q_proj_int4") == 20_979_712
    assert alg_bytes("down_proj_int4") == 125_845_504
    assert alg_bytes("q_proj_nvfp4") == 21_495_808
    assert alg_bytes("q_proj_mxfp4") == 21_233_664


@pytest.mark.parametrize("name", [n for n in syn.WORKLOADS if n.startswith(("q_proj", "down_proj"))])
def test_ring_keeps_inputs_out_of_l2(name):
    slots = bench.ring_slots(name)
    assert 1 <= slots <= bench.RING_MAX
    if slots < bench.RING_MAX:
        assert bench.ring_bytes(name) >= 2 * bench.L2_BYTES
        # one slot fewer would not cover it (the ring is no larger than it must be)
        assert bench.ring_bytes(name) * (slots - 1) // slots < 2 * bench.L2_BYTES or slots == 1


def test_ring_sizes_of_the_timed_workloads():
    assert bench.ring_slots("q_proj_int4") == 11
    assert bench.ring_slots("down_proj_int4") == 3
    assert bench.ring_slots("kv4") == 1 and bench.ring_bytes("kv4") > 2 * bench.L2_BYTES


def test_traffic_dropped_when_sources_changed(monkeypatch):
    key = ("hadamard_quant", "q_proj_int4")
    fp = bench.source_fingerprint(bench.ROTATE_SOURCES)
    monkeypatch.setitem(bench.TRAFFIC, key, (123, fp))
    assert bench.traffic(*key) == 123
    monkeypatch.setitem(bench.TRAFFIC, key, (123, "0" * 16))
    assert bench.traffic(*key) is None
    assert bench.traffic("gemm", "no_such_workload") is None


def test_job_rate_and_rank_max():
    assert bench.job_rate(1000, 4, 2.0) == pytest.approx(2_000_000)
    assert list(bench.max_over_ranks([1.0, 3.0])) == [1.0, 3.0]


def test_reference_arm_config_matches_the_default_run():
    """With the default --workload all, both arms print the headline's config
    (down_proj), including the list of the other measured configurations."""
    import argparse
    args = argparse.Namespace(workload="all", y_dtype="bf16")
    cfg = bench.workload_config(args, bench.HEADLINE)
    assert cfg["workload"] == "down_proj_int4"
    assert cfg["also_measured"] == list(bench.ALSO_MEASURED)
    assert "also_measured" not in bench.workload_config(args, "q_proj_int4")
