"""Throughput of the fused Hadamard rotation + int4 quantization (libhadq).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hadq|reference]

One step = one hadq_rotate_quant launch over one batch of the R1 workload:
4096 tokens x hidden 4096 bf16 (1 % outlier channels x50), full 4096-point
Sylvester Hadamard, symmetric int4 RTN per group of 128 with fp16 scales.
The metric is GB/s of algorithmic traffic (input read once + codes and scales
written once) and its fraction of the measured HBM copy bandwidth.

Timing: inputs resident in HBM; for C2, 8 buffer sets (input + outputs) are
rotated so each step touches data last used 7 steps earlier (338 MB > L2).  The K steps
are captured back to back in one CUDA graph; the graph is replayed once
untimed and once timed between barriers and device synchronisations.  The
timed graph holds the W untimed warm-up steps, then the K timed steps, with
CUDA event record nodes inside it: the start event marks the last warm-up
step's completion (recorded on a side stream, so the first timed step keeps
its programmatic launch on the warm-up step), the end event follows the K-th
step.  The window holds exactly the K steps, back to back, and none of the
host's submission or the graph's launch latency.  `value` = bytes of all ranks / max-over-ranks elapsed time;
`roofline.achieved` = bytes per launch / mean launch interval (kernel plus
inter-kernel gap).  Beside it the line reports a K-step replay with host-side
events recorded while the host submits the graph (the window then also holds
the submission and graph-launch latency), a median over per-launch event
pairs, and (`roofline.two_streams`) the same K steps with consecutive steps
on two streams, as independent batches can be scheduled.
`e2e` repeats the metric through hadq_rotate_quant_host (pinned host input,
copies in and out inside the timed region).

Ranks: under torchrun (WORLD_SIZE set) every rank processes its own batch
(weak scaling, no collective on the data path); rank 0 prints one JSON line.
Without WORLD_SIZE, `--gpus N` with N > 1 starts the N ranks itself (one
process per local GPU, 127.0.0.1 rendezvous) and returns the worst exit code.
`--dry-run` runs the rank plumbing alone on CPU (gloo, each rank timing the
oracle on a few rows of its own batch) for tests of the launcher.
`--impl reference` times the float64 CPU oracle on the host cores instead.
`--rows R` keeps only the first R rows of every workload part (a smaller case
of the same kernel, for profiler captures); the default is the full workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hadamard_rotation_bit_b200 import workloads as W  # noqa: E402

METRIC = "fused Hadamard+quant GB/s and % of B200 HBM peak (4096x4096 bf16->int4 g128)"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
SLEEP_CYCLES = 20_000_000      # ~10 ms of GPU sleep ahead of a timed region

# A step is one pass of the fused path over one batch of a workload: the
# launches below, in order.  c4 (R3) rotates Q to bf16 and quantizes K.
STEP_PARTS = {"c1": ["c1"], "c2": ["c2"], "c3": ["c3"], "c4": ["c4q", "c4k"], "c5": ["c5"],
              "c2r": ["c2r"], "c2rb": ["c2rb"], "c2n": ["c2n"], "c5n": ["c5n"], "c3rb": ["c3rb"], "c5rb": ["c5rb"],
              "c3k": ["c3k"], "c3km": ["c3km"], "c2p": ["c2p"], "c2q": ["c2q"], "pl256": ["pl256"],
              "pl1024": ["pl1024"]}
WORKLOAD = W.WORKLOADS["c2"]


def _env_int(k, d):
    try:
        return int(os.environ.get(k, d))
    except ValueError:
        return d


def part_rows(key, rows=None):
    """Rows of one workload part: all of them, or the first `rows`."""
    w = W.WORKLOADS[key]
    return w.rows if rows is None else max(1, min(w.rows, rows))


def step_bytes(cfg, rows=None):
    return sum(W.WORKLOADS[k].algorithmic_bytes * part_rows(k, rows) // W.WORKLOADS[k].rows
               for k in STEP_PARTS[cfg])


def n_buffers(cfg, rows=None):
    """Distinct buffer sets rotated through so that every step reads data not
    touched for at least ~3 L2 capacities (or inputs larger than L2)."""
    return int(max(1, min(8, -(-3 * L2_BYTES // step_bytes(cfg, rows)))))


def config_block(cfg="c2", rows=None):
    parts = [W.WORKLOADS[k] for k in STEP_PARTS[cfg]]
    nb = n_buffers(cfg, rows)
    sb = step_bytes(cfg, rows)
    d = {"workload": " + ".join(w.name for w in parts), "algorithmic_bytes_per_step": sb,
         "l2": (f"inputs larger than L2 ({sb / 1e6:.0f} MB per step)" if nb == 1 else
                f"{nb} rotating buffer sets ({nb * sb / 1e6:.0f} MB > L2 126 MB)"
                if nb * sb > L2_BYTES else
                f"{nb} buffer sets, {nb * sb / 1e6:.1f} MB: L2-resident (parity-size config)")}
    if len(parts) == 1:
        w = parts[0]
        d.update({"rows": part_rows(w.key, rows), "n": w.n, "block": w.block, "fmt": w.fmt, "group": w.group,
                  "x_dtype": w.x_dtype})
    if rows is not None:
        d["rows_override"] = rows
    return d


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = json.load(f)["hbm_gbs"]
        if isinstance(v, dict):            # {"value": ...} form
            v = v.get("value", v.get("gbs"))
        return float(v), "measured"
    except (OSError, KeyError, ValueError, TypeError):
        return FALLBACK_HBM_GBS, "fallback"


# Sources of the C2 kernel and of its launch configuration.
C2_KERNEL_SOURCES = ("hadq_api.cu", "hadq_device.cuh", "hadq_launch.h", "hadq_tc.cuh", "kernels_tc.cu")


def _strip_comments(src):
    """C++ source without // and /* */ comments (they do not change the binary)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def kernel_source_hash():
    """Hash of the C2 kernel's sources with their comments removed."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hadamard_rotation_bit_b200", "csrc")
    for f in C2_KERNEL_SOURCES:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + _strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; otherwise None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic_c2.json")) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    return rec.get("dram_bytes_per_launch") if rec.get("kernel_source_hash") == kernel_source_hash() else None


class ClockSampler:
    """NVML samples of SM clock and throttle reasons while the timed region runs."""

    NAMES = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
             0x4: "sw_power_cap", 0x1: "gpu_idle", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index, period=0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.nv, self.err = None, str(e)

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in self.NAMES.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.nv:
            return {"error": getattr(self, "err", "no NVML")}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(self.reasons - {"gpu_idle"})}


def dist_setup(backend="nccl"):
    world = _env_int("WORLD_SIZE", 1)
    if world > 1:
        import datetime
        import torch.distributed as dist
        rank, local = _env_int("RANK", 0), _env_int("LOCAL_RANK", 0)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return dist, rank, world, local
    return None, 0, 1, 0


def check_world(gpus):
    """--gpus must agree with the world size a launcher gave us."""
    world = _env_int("WORLD_SIZE", 1)
    if "WORLD_SIZE" in os.environ and world != gpus:
        raise SystemExit(f"bench.py: --gpus {gpus} but WORLD_SIZE={world}")
    return world


def _free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(n, argv):
    """Start this script once per rank (RANK = LOCAL_RANK = i, WORLD_SIZE = n,
    rendezvous on 127.0.0.1) and wait for all of them; the worst exit code is
    returned.  Each rank takes the GPU of its local rank."""
    import subprocess
    port = str(_free_port())
    procs = []
    for i in range(n):
        env = dict(os.environ, RANK=str(i), LOCAL_RANK=str(i), WORLD_SIZE=str(n), LOCAL_WORLD_SIZE=str(n),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=port)
        procs.append(subprocess.Popen([sys.executable, os.path.abspath(__file__)] + argv, env=env))
    rc = 0
    for p in procs:
        r = p.wait()
        rc = r if rc == 0 else rc
    return rc


def barrier(dist):
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(dist, v):
    """Largest value over all ranks (device timings are reduced with MAX)."""
    if dist is None:
        return v
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(bytes_per_step, steps, world, elapsed_max_s):
    """Whole-job throughput: bytes every rank processed / the slowest rank's time."""
    return bytes_per_step * steps * world / elapsed_max_s / 1e9


def cpu_baseline(seconds=12.0):
    """The float64 oracle, as it stands, on this host's cores: whole C2 batches
    (or row slices of one) until about `seconds` of CPU work is done."""
    import oracle
    w = WORKLOAD
    rows = 512
    x = W.bits_to_float64(W.generate("c2", slice(0, rows)), "bf16")
    oracle.rotate_quant(x[:8], 0, "int4", 128)          # builds and caches H_4096
    done, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        oracle.rotate_quant(x, 0, "int4", 128)
        done += rows
    dt = time.perf_counter() - t0
    bytes_done = w.algorithmic_bytes * done / w.rows
    cores = len(os.sched_getaffinity(0))
    return {"value": bytes_done / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} rows of the 4096x4096 batch in slices of {rows} rows ({dt:.1f} s, float64 numpy/BLAS)"}


def run_reference(args):
    """The oracle as the reference arm: each step a row slice of the workload.
    Rank 0 alone runs it; the other ranks of a multi-rank launch exit at once."""
    if _env_int("RANK", 0) != 0:
        return
    import oracle
    w = WORKLOAD
    steps, warm = args.steps, args.warmup
    rows = int(max(1, min(w.rows, 60.0 * 80 / max(1, steps + warm))))   # ~80 rows/s of oracle work
    x = W.bits_to_float64(W.generate("c2", slice(0, rows)), "bf16")
    for _ in range(warm):
        oracle.rotate_quant(x, 0, "int4", 128)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.rotate_quant(x, 0, "int4", 128)
    dt = time.perf_counter() - t0
    value = w.algorithmic_bytes * rows / w.rows * steps / dt / 1e9
    cores = len(os.sched_getaffinity(0))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps, "warmup": warm,
            "ms_per_step": dt / steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": config_block("c2"), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{rows} rows of the 4096x4096 batch per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_dry(args):
    """Rank plumbing without a GPU: gloo process group, every rank times the
    oracle on a few rows of its own batch (per-rank seed), max over ranks,
    whole-job aggregate; rank 0 prints the line (impl "dry-run")."""
    import oracle
    dist, rank, world, _ = dist_setup("gloo")
    rows = 4
    x = W.bits_to_float64(W.generate("c2", slice(0, rows), seed=W.rank_seed(rank)), "bf16")
    if dist is not None:
        dist.barrier()
    t0 = time.perf_counter()
    _, codes, _ = oracle.rotate_quant(x, 0, "int4", 128)
    elapsed = max_over_ranks(dist, time.perf_counter() - t0)
    digest = int(codes.astype(np.int64).sum())
    digests = [digest]
    if dist is not None:
        t = torch.tensor([digest], dtype=torch.int64)
        gathered = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        digests = [int(g.item()) for g in gathered]
    if rank == 0:
        b = WORKLOAD.algorithmic_bytes * rows // WORKLOAD.rows
        print(json.dumps({"metric": METRIC, "value": aggregate_gbs(b, 1, world, elapsed), "unit": UNIT,
                          "n_gpus": world, "impl": "dry-run", "rank_digests": digests,
                          "elapsed_max_s": elapsed}), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def _device_input(key, seed, dev, workers, rows=None):
    w = W.WORKLOADS[key]
    stored = W.generate(key, None if rows is None else slice(0, part_rows(key, rows)), seed=seed, workers=workers)
    if w.x_dtype == "bf16":
        return stored, torch.from_numpy(stored.view(np.int16)).view(torch.bfloat16).to(dev)
    return stored, torch.from_numpy(stored).to(dev)


def _two_stream_interval(step, steps, warm, stream, side, dev, dist):
    """Max-over-ranks seconds of K steps alternating between two streams."""
    s1 = torch.cuda.Stream(device=dev)
    t2_start = torch.cuda.Event(enable_timing=True, external=True)
    t2_end = torch.cuda.Event(enable_timing=True, external=True)
    ev_fork2 = torch.cuda.Event()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        for i in range(warm):
            step(steps + i)
        ev_fork2.record(stream)
        side.wait_event(ev_fork2)
        t2_start.record(side)
        s1.wait_event(ev_fork2)
        for i in range(steps):
            step(i, stream if i % 2 == 0 else s1)
        stream.wait_stream(s1)
        stream.wait_stream(side)
        t2_end.record(stream)
    with torch.cuda.stream(stream):
        g2.replay()
    stream.synchronize()
    barrier(dist)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(SLEEP_CYCLES)
        g2.replay()
    stream.synchronize()
    barrier(dist)
    elapsed = max_over_ranks(dist, t2_start.elapsed_time(t2_end) / 1e3)
    del g2
    return elapsed


def run_hadq(args):
    from hadamard_rotation_bit_b200 import hadq as H
    dist, rank, world, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    H.load_library()
    cfg = args.config
    keys = STEP_PARTS[cfg]
    steps, warm = args.steps, max(3, args.warmup)
    nbuf = n_buffers(cfg, args.rows)
    workers = max(1, min(16, (os.cpu_count() or 2) // 2))

    host, bufs, signs, rpbh, thr = {}, [], {}, {}, {}
    for k in keys:
        w = W.WORKLOADS[k]
        host[k], x0 = _device_input(k, W.rank_seed(rank), dev, workers, args.rows)
        bufs.append([x0] + [x0.clone() for _ in range(nbuf - 1)])
        if w.signs is not None:
            signs[k] = torch.from_numpy(W.generate_signs(k, W.rank_seed(rank))).to(dev)
        if w.rpbh:
            rpbh[k] = tuple(torch.from_numpy(a).to(dev) for a in W.generate_rpbh(k, W.rank_seed(rank)))
        if w.fmt == "codebook":
            thr[k] = torch.from_numpy(H.hadq_codebook(w.n, w.group)[1].copy()).to(dev)

    def launch(j, i, stream=None, outs=None):
        w = W.WORKLOADS[keys[j]]
        x = bufs[j][i % nbuf]
        if w.fmt == "codebook":
            c, nr = (None, None) if outs is None else outs[j][i % nbuf]
            p, sg = rpbh.get(w.key, (None, None))
            return H.hadq_rotate_quant_codebook(x, w.group, thr[w.key], w.block, perm=p, signs=sg, codes=c, norms=nr,
                                                stream=stream)
        if w.rpbh:
            c, sc = (None, None) if outs is None else outs[j][i % nbuf]
            return H.hadq_rotate_quant_rpbh(x, rpbh[w.key][0], rpbh[w.key][1], w.block, w.fmt, w.group, codes=c,
                                            scales=sc, stream=stream)
        if w.signs is not None:
            c, sc = (None, None) if outs is None else outs[j][i % nbuf]
            return H.hadq_rotate_quant_signed(x, signs[w.key], w.signs, w.block, w.fmt, w.group, codes=c, scales=sc,
                                              stream=stream)
        if w.fmt is None:
            o = None if outs is None else outs[j][i % nbuf]
            return H.hadq_rotate(x, w.block, out=o, stream=stream,
                                 out_dtype=torch.bfloat16 if w.out_dtype == "bf16" else torch.float32)
        c, sc = (None, None) if outs is None else outs[j][i % nbuf]
        return H.hadq_rotate_quant(x, w.block, w.fmt, w.group, codes=c, scales=sc, stream=stream)

    outs = [[launch(j, i) for i in range(nbuf)] for j in range(len(keys))]   # allocate outputs, warm caches
    torch.cuda.synchronize()
    bytes_step = step_bytes(cfg, args.rows)
    stream = torch.cuda.Stream(device=dev)

    def step(i, st=None):
        for j in range(len(keys)):
            launch(j, i, stream if st is None else st, outs)

    with torch.cuda.stream(stream):
        for i in range(warm):
            step(i)
    stream.synchronize()

    # K back-to-back steps captured in one CUDA graph, replayed on `stream`.
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            step(i)
    with torch.cuda.stream(stream):
        g.replay()                       # untimed replay (warm-up of the graph itself)
    stream.synchronize()

    # Timed region: one graph holds the W untimed warm-up steps, then the K
    # timed steps, with CUDA events recorded inside the graph (event record
    # nodes on the launching stream's work).  The start event is recorded on
    # a side stream forked after the last warm-up step, so it marks that
    # step's completion while the first timed step keeps its programmatic
    # launch on the warm-up step, as every later step has on its predecessor;
    # the end event follows the K-th step.  The window holds exactly the K
    # steps, each measured from its predecessor's completion to its own, and
    # none of the host's submission or of the graph's launch latency.
    t_start = torch.cuda.Event(enable_timing=True, external=True)
    t_end = torch.cuda.Event(enable_timing=True, external=True)
    ev_fork = torch.cuda.Event()
    side = torch.cuda.Stream(device=dev)
    gt = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gt, stream=stream):
        for i in range(warm):
            step(steps + i)
        ev_fork.record(stream)
        side.wait_event(ev_fork)
        t_start.record(side)
        for i in range(steps):
            step(i)
        stream.wait_stream(side)
        t_end.record(stream)
    with torch.cuda.stream(stream):
        gt.replay()                      # untimed replay (warm-up of the graph itself)
    stream.synchronize()
    barrier(dist)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            torch.cuda._sleep(SLEEP_CYCLES)   # the host submits the graph while the GPU is held busy
            gt.replay()
        stream.synchronize()
    barrier(dist)
    elapsed = t_start.elapsed_time(t_end) / 1e3
    elapsed_max = max_over_ranks(dist, elapsed)
    interval_max = elapsed_max / steps

    # The same replay with the events recorded while the host submits the
    # graph: the window also holds the submission latency (reported beside).
    h_start = torch.cuda.Event(enable_timing=True)
    h_end = torch.cuda.Event(enable_timing=True)
    barrier(dist)
    with torch.cuda.stream(stream):
        h_start.record(stream)
        g.replay()
        h_end.record(stream)
    stream.synchronize()
    barrier(dist)
    host_submit_max = max_over_ranks(dist, h_start.elapsed_time(h_end) / 1e3)

    # Diagnostic: the same K steps with consecutive steps on two streams.  The
    # steps are independent batches, so a step need not wait for the one
    # before it on the other stream, and its CTAs start as the other step's
    # CTAs leave; each stream's steps keep their programmatic launch on the
    # step before them on that stream.  Events and warm-up as in the timed graph.
    # Consecutive steps write different buffer sets only when there are two.
    two_streams = None
    if nbuf >= 2:
        two_streams = _two_stream_interval(step, steps, warm, stream, side, dev, dist)

    # Diagnostic: an event pair around each step, all queued behind a sleep
    # kernel so the steps run back to back without host gaps.
    n_ev = min(steps, 200)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_ev)]
    with torch.cuda.stream(stream):
        torch.cuda._sleep(SLEEP_CYCLES)
        for i in range(n_ev):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
    stream.synchronize()
    step_ev = statistics.median(a.elapsed_time(b) / 1e3 for a, b in ev)

    # End to end through the host-buffer entry point (quantizing parts only):
    # consecutive steps alternate between two streams, each with its own
    # device staging and host output buffers, so the copy in of one step runs
    # while the copy out of the previous one drains (PCIe is full duplex).
    e2e = None
    qkeys = [k for k in keys if W.WORKLOADS[k].fmt not in (None, "codebook") and W.WORKLOADS[k].signs is None
             and not W.WORKLOADS[k].rpbh]
    if len(qkeys) == len(keys):
        e2e_steps = max(4, min(steps, 20))
        streams = [stream, torch.cuda.Stream(device=dev)]
        pinned, staging = [], []
        for j, k in enumerate(keys):
            xh = torch.from_numpy(host[k].view(np.int16)).view(torch.bfloat16) if W.WORKLOADS[k].x_dtype == "bf16" \
                else torch.from_numpy(host[k])
            c0, s0 = outs[j][0]
            xh = xh.pin_memory()
            pinned.append([(xh, torch.empty(c0.shape, dtype=c0.dtype).pin_memory(),
                            torch.empty(s0.shape, dtype=s0.dtype).pin_memory()) for _ in streams])
            per = []
            for q in range(len(streams)):       # staging q: buffer set q if there are two, else a copy
                if q < nbuf:
                    per.append((bufs[j][q], outs[j][q][0], outs[j][q][1]))
                else:
                    per.append((torch.empty_like(bufs[j][0]), torch.empty_like(c0), torch.empty_like(s0)))
            staging.append(per)

        def e2e_step(i):
            q = i % len(streams)
            for j, k in enumerate(keys):
                w = W.WORKLOADS[k]
                xh, ch, sh = pinned[j][q]
                xd, c, sc = staging[j][q]
                H.hadq_rotate_quant_host(xh, w.block, w.fmt, w.group, ch, sh, xd, c, sc, stream=streams[q])

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(dist)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(streams[0])
        streams[1].wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        done1 = torch.cuda.Event()
        done1.record(streams[1])
        streams[0].wait_event(done1)
        e1.record(streams[0])
        torch.cuda.synchronize()
        e2e_max = max_over_ranks(dist, e0.elapsed_time(e1) / 1e3)
        e2e = {"value": aggregate_gbs(bytes_step, e2e_steps, world, e2e_max), "unit": UNIT,
               "h2d_bytes_per_step": sum(W.WORKLOADS[k].in_bytes * part_rows(k, args.rows) // W.WORKLOADS[k].rows
                                         for k in keys),
               "d2h_bytes_per_step": sum(W.WORKLOADS[k].out_bytes * part_rows(k, args.rows) // W.WORKLOADS[k].rows
                                         for k in keys),
               "path": "hadq_rotate_quant_host (pinned host buffers, copies in and out inside the timed region; "
                       "steps alternate between two streams so copies in and out overlap)"}

    if rank == 0:
        peak, peak_kind = measured_peak()
        achieved = bytes_step / interval_max / 1e9
        rows_step = sum(part_rows(k, args.rows) for k in keys)
        line = {
            "metric": METRIC if cfg == "c2" else f"fused Hadamard+quant GB/s ({cfg})",
            "value": aggregate_gbs(bytes_step, steps, world, elapsed_max),
            "unit": UNIT,
            "n_gpus": world,
            "steps": steps,
            "warmup": warm,
            "ms_per_step": elapsed_max / steps * 1e3,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": config_block(cfg, args.rows),
            "impl": "hadq",
            "rows_per_s": rows_step * steps * world / elapsed_max,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "peak_kind": f"{peak_kind} hbm_gbs (copy)",
                         "traffic": recorded_traffic() if cfg == "c2" and args.rows is None else None,
                         "duration": "mean interval of K back-to-back steps in one CUDA graph after W untimed "
                                     "warm-up steps (CUDA event record nodes in the graph: start at the last "
                                     "warm-up step's completion, end at the K-th step's)",
                         "step_interval_us": interval_max * 1e6,
                         "step_interval_us_host_submit": host_submit_max / steps * 1e6,
                         "step_us_event_pairs_median": step_ev * 1e6,
                         "two_streams": None if two_streams is None else
                         {"step_interval_us": two_streams / steps * 1e6,
                          "frac": bytes_step / (two_streams / steps) / 1e9 / peak}},
            "e2e": e2e,
            "gpu_launches": steps * len(keys),
            "clocks": clocks.summary(),
        }
        if world == 1 and cfg == "c2" and args.rows is None and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    del g, gt
    if dist is not None:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["hadq", "reference"], default="hadq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config", choices=sorted(STEP_PARTS), default="c2",
                    help="workload (default c2, the metric's configuration; others for reference)")
    ap.add_argument("--rows", type=int, default=None,
                    help="only the first ROWS rows of each workload part (smaller case for profiler captures)")
    ap.add_argument("--dry-run", action="store_true",
                    help="rank plumbing only, on CPU (gloo): launcher, per-rank seeds, max-over-ranks")
    args = ap.parse_args()
    if args.gpus < 1:
        raise SystemExit("bench.py: --gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    check_world(args.gpus)
    if args.dry_run:
        run_dry(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_hadq(args)


if __name__ == "__main__":
    main()
