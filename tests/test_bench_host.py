"""Host logic of bench.py (no GPU): the bytes a step moves, the buffer
rotation that keeps every timed read coming from HBM, the config block, the
source hash that keys the recorded DRAM traffic, and the reference arm's
JSON line (the float64 oracle on the host cores)."""

import contextlib
import io
import json
import types

import pytest

import bench
from hadamard_rotation_bit_b200 import workloads as W


def test_step_bytes_are_the_algorithmic_bytes_of_the_parts():
    # 4096 x 4096 bf16 in, int4 codes + fp16 scales per 128 out: 33,554,432 + 8,388,608 + 262,144
    assert bench.step_bytes("c2") == 42_205_184
    assert bench.step_bytes("c4") == W.WORKLOADS["c4q"].algorithmic_bytes + W.WORKLOADS["c4k"].algorithmic_bytes
    for cfg, parts in bench.STEP_PARTS.items():
        assert bench.step_bytes(cfg) == sum(W.WORKLOADS[k].algorithmic_bytes for k in parts)
    # a row slice scales every part by its share of rows
    assert bench.step_bytes("c2", rows=1024) == 42_205_184 // 4


@pytest.mark.parametrize("cfg", sorted(bench.STEP_PARTS))
def test_timed_reads_come_from_hbm(cfg):
    """Either one step's inputs exceed L2 or the rotated buffer sets together
    exceed three L2 capacities (the parity-size c1 excepted)."""
    nb = bench.n_buffers(cfg)
    sb = bench.step_bytes(cfg)
    assert 1 <= nb <= 8
    if cfg != "c1":
        assert nb * sb > bench.L2_BYTES
        assert nb == 8 or nb * sb >= 3 * bench.L2_BYTES


def test_config_block_names_the_workload():
    c = bench.config_block("c2")
    assert c["rows"] == 4096 and c["n"] == 4096 and c["block"] == 4096 and c["fmt"] == "int4" and c["group"] == 128
    assert c["algorithmic_bytes_per_step"] == 42_205_184
    assert "rotating buffer sets" in c["l2"]
    assert "+" in bench.config_block("c4")["workload"]          # Q and K parts
    assert bench.config_block("c2", rows=512)["rows_override"] == 512


def test_source_hash_ignores_comments():
    code = "int f(int x) { return x + 1; }\n"
    commented = "// the successor\nint f(int x) { /* one more */ return x + 1; }  // done\n"
    assert bench._strip_comments(code).split() == bench._strip_comments(commented).split()
    assert bench._strip_comments("a /* x\n y */ b").split() == ["a", "b"]
    h = bench.kernel_source_hash()
    assert len(h) == 16 and h == bench.kernel_source_hash()


def test_reference_arm_prints_one_json_line():
    args = types.SimpleNamespace(gpus=1, steps=30, warmup=30, impl="reference")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["value"] > 0 and line["steps"] == 30 and line["warmup"] == 30
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == W.WORKLOADS["c2"].name
