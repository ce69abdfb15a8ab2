"""Host logic of bench.py (no GPU): the bytes a step moves, the buffer
rotation that keeps every timed read coming from HBM, the config block, the
source hash that keys the recorded DRAM traffic, and the reference arm's
JSON line (the float64 oracle on the host cores), and the launcher that
starts one rank per GPU when --gpus N > 1 is given without torchrun."""

import contextlib
import io
import json
import os
import subprocess
import sys
import types

import pytest

import bench
from hadamard_rotation_bit_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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


def _bench(args, env_extra=None, timeout=600):
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    env.update(env_extra or {})
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                         env=env, timeout=timeout, cwd=ROOT)
    return res


def test_gpus_n_starts_n_ranks_itself():
    """Without a launcher, --gpus 2 starts two ranks (gloo dry run): the line
    reports n_gpus 2, and the two ranks drew different batches (per-rank
    seeds) and agreed on the max-over-ranks time."""
    res = _bench(["--gpus", "2", "--dry-run"])
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(v) for v in res.stdout.splitlines() if v.startswith("{")]
    assert len(lines) == 1, res.stdout          # rank 0 alone prints
    line = lines[0]
    assert line["n_gpus"] == 2 and line["impl"] == "dry-run"
    assert len(line["rank_digests"]) == 2 and line["rank_digests"][0] != line["rank_digests"][1]
    assert line["value"] > 0


def test_gpus_disagreeing_with_world_size_fails_loudly():
    res = _bench(["--gpus", "4", "--dry-run"], {"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"})
    assert res.returncode != 0 and "WORLD_SIZE=2" in (res.stderr + res.stdout)


def test_reference_arm_under_two_ranks_prints_once():
    """--impl reference --gpus 2: rank 0 alone times the oracle and prints."""
    res = _bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(v) for v in res.stdout.splitlines() if v.startswith("{")]
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
