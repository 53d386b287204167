"""Benchmark of the quantized linear-layer GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole decode hot path over one batch: for each
token count M of the W8A8_INT8 decode workload (M in {1, 8, 32}, N = K = 4096,
per-token int8 activations, per-channel int8 weights, bf16 out) the dynamic
activation quantiser and the tcgen05 GEMM run with the configuration the
per-shape table dispatches (or the built-in default).  The timed steps run as
CUDA graphs of consecutive steps (capture_steps), as a decode forward
captures its layers.  Weights are quantised once at set-up; the steps rotate
over enough weight copies (more than twice the L2) that every GEMM streams
its weights from HBM.

After the step, the default run times every configured shape on its own
(the metric's M <= 32 decode shapes of all four formats, and Block_FP8 at
M = 4096 and 16384): one CUDA graph of back-to-back GEMMs per shape over
weight copies totalling more than 2 x L2, giving µs per shape, the fraction of
roofline per shape and their geomeans (``--no-suite`` skips this phase).
``--suite`` prints those per-shape lines (and other families, e.g.
``medium_m``) instead of the step; ``--suite moe`` times the grouped
(mixture-of-experts) launch.

Printed (rank 0, one JSON line): the metric of the workload as whole-job
algorithmic HBM throughput (GB/s) of the step, per-shape GEMM microseconds and
fraction of the HBM roofline, the geomean over every configured shape, the
dominant kernel's roofline object, the CPU oracle's throughput on a bounded
sample, the end-to-end number through the public API with host buffers,
clocks sampled (NVML) during the timed work and the count of library kernels
launched while timing.

``--impl reference`` times the CPU oracle on the same workload (the only
"reference" that exists: the pages ship no code).  Multi-GPU (torchrun): every
rank runs the same replica workload, no collective on the data path.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/shape and geomean % roofline (HBM GB/s or TC TFLOP/s), quantized GEMM M≤32"
WORKLOAD = ("W8A8_INT8 decode linear layer: A bf16 ~N(0,1) [M,4096] per-token int8 (amax/127), "
            "W ~N(0,0.02) [4096,4096] per-channel int8, int32 accumulate, fp32 scale epilogue, bf16 out; "
            "M in {1,8,32}; seed 0 (A) / 1 (W)")
FMT_INT8 = 1
MS = (1, 8, 32)
N = K = 4096
TABLE = os.path.join(ROOT, "precision_quantized_gemm_b200", "tables", "b200.qgt")
L2_POLICY = ("inputs larger than L2: every GEMM of the timed steps and of the per-shape phase reads weight "
             "copies from a rotation of more than 2 x L2 (126 MB), activations too at M >= 4096")


def bench_config(world):
    """The `config` of the bench line, the same dict for both arms."""
    return {"workload": WORKLOAD, "M": list(MS), "N": N, "K": K, "format": "W8A8_INT8",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU", "l2": L2_POLICY,
            "per_shape_workloads": "every configured shape: FP8_Dynamic 16x2048x2048; W8A8_INT8 M in {1,8,32} "
                                   "4096^2; Block_FP8 16 decode shapes; NVFP4 16 shapes; FP8_Dynamic and Block_FP8 "
                                   "sweep 144 shapes; Block_FP8 M in {4096,16384} 5120^2"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--table", default=TABLE)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-suite", action="store_true",
                    help="skip the per-shape phase over every configured shape (the metric's geomean)")
    ap.add_argument("--suite", default=None,
                    help="comma list of per-shape suites to time instead of the step: "
                         "fp8_tiny,int8,block_fp8,nvfp4,sweep,large_m,medium_m,moe (one JSON line per shape)")
    ap.add_argument("--only-m", default=None, help="comma list: keep only these token counts of the per-shape suites")
    ap.add_argument("--moe-tokens", default=None, help="comma list of token counts of the moe suite (default: all)")
    ap.add_argument("--moe-formats", default=None, help="comma list of format ids of the moe suite (default: 0,1,2)")
    return ap.parse_args()


# --------------------------------------------------------------- bytes ---
def gemm_bytes(M):
    """Algorithmic bytes of one INT8 GEMM call: W_q + W scales + A_q + A scales + Y (bf16)."""
    return N * K + 4 * N + M * K + 4 * M + 2 * M * N


def quant_bytes(M):
    """Algorithmic bytes of one activation quantisation: A (bf16) + A_q + scales."""
    return 2 * M * K + M * K + 4 * M


def step_bytes():
    return sum(gemm_bytes(m) + quant_bytes(m) for m in MS)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_code(text: str) -> str:
    """The code of a CUDA source: `//` comments, trailing blanks and empty
    lines removed (the kernel sources hold no `//` inside a string)."""
    out = []
    for line in text.splitlines():
        line = line.split("//", 1)[0].rstrip()
        if line:
            out.append(line)
    return "\n".join(out) + "\n"


def kernel_source_hash():
    """sha1 of the GEMM kernels' code (gemm_kernel.cuh, skinny.cuh,
    persist.cuh, pair.cuh and ptx.cuh, comments ignored): ties an ncu
    traffic figure to the code it measured."""
    import hashlib
    h = hashlib.sha1()
    for f in ("gemm_kernel.cuh", "skinny.cuh", "persist.cuh", "pair.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "precision_quantized_gemm_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(kernel_source_code(fh.read()).encode())
    return h.hexdigest()[:12]


def measured_traffic(key="w8a8_int8_decode_dram_bytes_per_launch"):
    """DRAM bytes per GEMM launch (read + write) recorded under `key` in the
    committed ncu summary (default: this workload, averaged over its three
    shapes), or None when the kernels have changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    kv = dict(line.split(None, 1) for line in open(p) if line.strip() and not line.startswith("#"))
    if kv.get("kernel_sources", "").strip() != kernel_source_hash() or key not in kv:
        return None
    return float(kv[key])


# ------------------------------------------------------------- clocks ---
CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
SMI_FIELDS = "clocks.sm,clocks.max.sm,power.draw"
SMI_REASON_FIELDS = ("clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                     "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_smi_row(line):
    """One nvidia-smi CSV row (noheader, nounits) of SMI_FIELDS, optionally
    followed by the four SMI_REASON_FIELDS -> a sample dict, or None."""
    f = [x.strip() for x in line.split(",")]
    if len(f) < 3:
        return None
    try:
        sm, mx = float(f[0]), float(f[1])
    except ValueError:
        return None
    try:
        pw = float(f[2])
    except ValueError:
        pw = None
    reasons = [CLOCK_REASONS[i] for i in range(4) if len(f) >= 7 and f[3 + i].lower() == "active"]
    return {"sm_mhz": sm, "sm_max_mhz": mx, "power_w": pw, "reasons": reasons}


def summarise_clocks(samples, error=None):
    """Median SM clock of the samples taken under load (the GPU busy, at
    least half of the largest clock seen), the largest max clock, and every
    throttle reason any sample reported."""
    if not samples:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"no samples: {error}" if error else "no samples"],
                "samples": 0}
    top = max(x["sm_mhz"] for x in samples)
    load = [x for x in samples if x.get("busy", True) and x["sm_mhz"] >= 0.5 * top] or samples
    return {"sm_mhz": statistics.median(x["sm_mhz"] for x in load),
            "sm_max_mhz": max(x["sm_max_mhz"] for x in samples),
            "reasons": sorted({r for x in samples for r in x["reasons"]}),
            "samples": len(samples), "samples_under_load": len(load),
            "power_w_max": max((x["power_w"] for x in samples if x.get("power_w") is not None), default=None)}


class Clocks:
    """Samples the SM clock, power and throttle reasons of this process's GPU
    every `period` seconds on a host thread while the timed work runs.  NVML
    (read-only queries) first; where NVML is missing, one-shot nvidia-smi
    queries.  The GPU is found by its PCI bus id, so the sample is of the
    device this process uses whatever CUDA_VISIBLE_DEVICES maps."""

    def __init__(self, bus_id, period=0.1):
        import threading
        self.bus_id = bus_id
        self.period = period
        self.samples = []
        self.error = None
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _nvml(self):
        import pynvml as N
        N.nvmlInit()
        h = N.nvmlDeviceGetHandleByPciBusId(self.bus_id.encode() if isinstance(self.bus_id, str) else self.bus_id)
        bits = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap}

        def one():
            sm = float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM))
            mx = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))
            try:
                pw = N.nvmlDeviceGetPowerUsage(h) / 1000.0
            except N.NVMLError:
                pw = None
            try:
                r = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                reasons = [k for k, b in bits.items() if r & b]
            except N.NVMLError:
                reasons = []
            try:
                busy = N.nvmlDeviceGetUtilizationRates(h).gpu > 0
            except N.NVMLError:
                busy = True
            return {"sm_mhz": sm, "sm_max_mhz": mx, "power_w": pw, "reasons": reasons, "busy": busy}
        return one, N.nvmlShutdown

    def _smi(self):
        def one():
            r = subprocess.run(["nvidia-smi", "-i", self.bus_id, f"--query-gpu={SMI_FIELDS},{SMI_REASON_FIELDS}",
                                "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
            if r.returncode != 0:     # an older driver may lack the reason fields: ask for the clocks alone
                r = subprocess.run(["nvidia-smi", "-i", self.bus_id, f"--query-gpu={SMI_FIELDS}",
                                    "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
            if r.returncode != 0:
                raise RuntimeError((r.stderr or r.stdout).strip().splitlines()[0][:120])
            x = parse_smi_row(r.stdout.strip().splitlines()[0])
            if x is None:
                raise RuntimeError(f"unparsed nvidia-smi row: {r.stdout.strip()[:120]}")
            return x
        return one, lambda: None

    def _run(self):
        try:
            one, done = self._nvml()
        except Exception as exc:                       # no NVML: nvidia-smi queries
            self.error = f"nvml: {type(exc).__name__}"
            one, done = self._smi()
        try:
            while not self._stop.is_set():
                t = time.perf_counter()
                try:
                    self.samples.append(dict(one(), t=t))
                except Exception as exc:
                    self.error = f"{type(exc).__name__}: {exc}"[:160]
                    if not self.samples:
                        break
                self._stop.wait(max(0.0, self.period - (time.perf_counter() - t)))
        finally:
            done()

    def start(self):
        self._thread.start()
        return self

    def stop(self):
        self._stop.set()
        self._thread.join(timeout=15)
        return summarise_clocks(self.samples, self.error)

    def window(self, t0, t1):
        """Summary of the samples taken between perf_counter times t0 and t1."""
        return summarise_clocks([x for x in self.samples if t0 <= x["t"] <= t1], self.error)


def device_bus_id(dev_index):
    import torch
    p = torch.cuda.get_device_properties(dev_index)
    return "%08X:%02X:%02X.0" % (getattr(p, "pci_domain_id", 0), p.pci_bus_id, p.pci_device_id)


# ------------------------------------------------------------ helpers ---
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl"
        try:
            import torch
            if not torch.cuda.is_available():
                backend = "gloo"
        except ImportError:
            backend = "gloo"
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_baseline(sample_steps=6):
    """The oracle (numpy, as it stands) on a bounded sample of the workload:
    ``sample_steps`` steps of quantise-3-activations + exact int64 GEMMs +
    bf16 epilogue; the weights are quantised once outside the timing."""
    import numpy as np
    import qg_synth
    from oracle import gemm as OG
    from oracle import quant as OQ
    w = qg_synth.weights(N, K)
    qw, sw = OQ.per_row_int8(w)
    acts = {m: qg_synth.activations(m, K) for m in MS}
    t0 = time.perf_counter()
    for _ in range(sample_steps):
        for m in MS:
            qa, sa = OQ.per_row_int8(acts[m])
            OG.w8a8_int8(qa, sa, qw, sw)
    dt = (time.perf_counter() - t0) / sample_steps
    return {"value": step_bytes() / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{sample_steps} full steps (3 activation quantisations + 3 exact int64 GEMMs "
                      f"M in {{1,8,32}}, N=K=4096 + bf16 epilogue), weights quantised once; numpy int64 "
                      f"matmul runs on one thread",
            "seconds_per_step": dt}


# Worker side of the all-cores oracle timing: each process holds the
# oracle-quantised weights and computes the oracle GEMMs of a step on a block
# of output columns (weight rows).  The oracle functions run as they stand.
_ORACLE_W = None


def _oracle_worker_init(qw, sw):
    global _ORACLE_W
    _ORACLE_W = (qw, sw)


def _oracle_block(job):
    from oracle import gemm as OG
    n0, n1, acts_q = job
    qw, sw = _ORACLE_W
    return [OG.w8a8_int8(qa, sa, qw[n0:n1], sw[n0:n1]) for qa, sa in acts_q]


def cpu_baseline_all_cores(sample_steps=6, warmup=1):
    """The same oracle step on every host core: a process pool (started with
    spawn, as a CUDA process must) splits each step's three GEMMs over blocks
    of output columns; the activation quantisation runs in this process.  The
    blocks are checked to reassemble into the single-process result first."""
    import multiprocessing as mp

    import numpy as np
    import qg_synth
    from oracle import gemm as OG
    from oracle import quant as OQ
    avail = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    # each worker holds the 16 MB of weight codes and a step's int64
    # temporaries (~0.4 GB at most): bounded by the host's memory
    try:
        mem = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_AVPHYS_PAGES")
    except (ValueError, OSError):
        mem = 8 << 30
    cores = max(1, min(avail, int(mem // (1 << 30)), 64))
    acts = {m: qg_synth.activations(m, K) for m in MS}
    qw, sw = OQ.per_row_int8(qg_synth.weights(N, K))
    bounds = np.linspace(0, N, cores + 1).astype(int)
    ctx = mp.get_context("spawn")
    with ctx.Pool(cores, initializer=_oracle_worker_init, initargs=(qw, sw)) as pool:
        def step():
            acts_q = [OQ.per_row_int8(acts[m]) for m in MS]
            jobs = [(int(bounds[i]), int(bounds[i + 1]), acts_q) for i in range(cores)]
            # bounded: a stalled worker raises (TimeoutError) instead of
            # holding the bench; leaving the `with` terminates the pool
            parts = pool.map_async(_oracle_block, jobs).get(timeout=300)
            return [np.concatenate([p[j] for p in parts], axis=1) for j in range(len(MS))]
        got = step()                                   # warm-up, and the reassembly check
        for j, m in enumerate(MS):
            qa, sa = OQ.per_row_int8(acts[m])
            if not np.array_equal(got[j], OG.w8a8_int8(qa, sa, qw, sw)):
                raise RuntimeError("oracle column blocks do not reassemble into the single-process result")
        for _ in range(max(0, warmup - 1)):           # the check above was the first warm-up step
            step()
        t0 = time.perf_counter()
        for _ in range(sample_steps):
            step()
        dt = (time.perf_counter() - t0) / sample_steps
    return {"value": step_bytes() / dt / 1e9, "unit": "GB/s", "cores": cores, "host_cores": avail,
            "kind": "oracle",
            "sample": f"{sample_steps} full steps (3 activation quantisations + 3 exact int64 GEMMs "
                      f"M in {{1,8,32}}, N=K=4096 + bf16 epilogue), weights quantised once; the GEMMs "
                      f"split over {cores} processes by output-column blocks (numpy int64 matmul is "
                      f"single-threaded; {avail} host cores available)",
            "seconds_per_step": dt}


# ---------------------------------------------------------- reference ---
def run_reference(args, world, rank):
    """The oracle on the host cores, on the same workload, `config`, metric and
    step count as the GPU arm: `--warmup` untimed steps, then `--steps` timed
    steps, each one full step of the workload (three activation quantisations
    and three exact GEMMs)."""
    if rank != 0:
        return
    steps = max(1, args.steps)
    single = cpu_baseline(1)
    try:
        cb = cpu_baseline_all_cores(steps, warmup=max(1, args.warmup))
    except Exception as exc:       # the pool is measurement harness: time the oracle in this process
        cb = dict(cpu_baseline(steps), all_cores_error=f"{type(exc).__name__}: {exc}"[:200])
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "GB/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup, "ms_per_step": 1000 * cb["seconds_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic", "config": bench_config(world),
            "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "host_cores", "kind", "sample",
                                                  "all_cores_error") if k in cb},
            "cpu_baseline_single_thread": {k: single[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- ours ---
def run_ours(args, world, rank, local):
    import numpy as np
    import torch

    import precision_quantized_gemm_b200 as qg
    import qg_synth

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    table = qg.Table(args.table) if os.path.exists(args.table) else None

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    # weights: quantised once, then copied so the rotation exceeds 2 x L2
    w = bf16(qg_synth.weights(N, K))
    layer = qg.Linear(FMT_INT8, w, table=table)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    wbytes = layer.Wq.q.numel() + layer.Wq.scale.numel()
    copies = max(4, min(64, (2 * l2) // wbytes + 2))
    Ws = [layer.Wq]
    for _ in range(copies - 1):
        o = qg.Operand(FMT_INT8, True, N, K, dev)
        o.q.copy_(layer.Wq.q)
        o.scale.copy_(layer.Wq.scale)
        Ws.append(o)
    cfgs, hits = {}, {}
    for m in MS:
        if table is not None:
            cfgs[m], hits[m] = table.dispatch(FMT_INT8, m, N, K)
        else:
            cfgs[m], hits[m] = qg.qgemm_default_config(FMT_INT8, m, N, K), 0

    acts = {m: bf16(qg_synth.activations(m, K)) for m in MS}
    # one captured step per rotation slot: shape i of step s uses copy (3s+i) % copies;
    # a slot's three activations (and results) are views of one buffer, so
    # that the end-to-end step moves them with one copy each way
    nslots = copies
    steps_g, slot_in, slot_out = [], [], []
    rows = sum(MS)
    for s in range(nslots):
        per = []
        a_all = torch.zeros(rows * K, dtype=torch.bfloat16, device=dev)
        y_all = torch.empty(rows * N, dtype=torch.bfloat16, device=dev)
        r0 = 0
        for i, m in enumerate(MS):
            gs = qg.GraphStep(layer, m, W=Ws[(len(MS) * s + i) % copies], cfg=cfgs[m],
                              A=a_all[r0 * K:(r0 + m) * K].view(m, K), Y=y_all[r0 * N:(r0 + m) * N].view(m, N))
            gs.A.copy_(acts[m])
            per.append(gs)
            r0 += m
        steps_g.append(per)
        slot_in.append(a_all)
        slot_out.append(y_all)
    # a single graph per step slot holding the three shapes back to back
    step_graphs = []
    for s in range(nslots):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for gs in steps_g[s]:
                gs._launch()
        step_graphs.append(g)
    launches_per_step = sum(2 + (1 if (cfgs[m].split_k > 1 and cfgs[m].reduce_mode == 1) else 0) for m in MS)
    # The timed steps run as chunks of consecutive steps captured back to back
    # in one CUDA graph each, as a decode forward captures its layers' linear
    # layers in one graph: the kernels of step s + 1 overlap the tail of step
    # s through programmatic dependent launch instead of waiting out a graph
    # launch.  Every step keeps its own work: three activation quantisations
    # and three GEMMs on its own rotation slot of weight copies.
    chunk = max(1, min(args.steps, nslots))
    timed_graphs = []
    s0 = 0
    while s0 < args.steps:
        n = min(chunk, args.steps - s0)
        timed_graphs.append(qg.capture_steps([gs for s in range(s0, s0 + n) for gs in steps_g[s % nslots]]))
        s0 += n
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    # ---- warm-up (every timed graph replays once as well)
    for s in range(args.warmup):
        step_graphs[s % nslots].replay()
    for g in timed_graphs:
        g.replay()
    torch.cuda.synchronize()

    # ---- timed region: K full steps
    clocks = Clocks(device_bus_id(local)).start()
    # Keep the GPU on the same steps for half a second (more untimed warm-up)
    # so that the clock samples of this window show the conditions the timed
    # region runs under (the region itself is far shorter than a sample).
    t_load = time.perf_counter()
    while time.perf_counter() - t_load < 0.5:
        for g in timed_graphs:
            g.replay()
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for g in timed_graphs:
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t_step_end = time.perf_counter()
    barrier(world)
    ms_step = e0.elapsed_time(e1) / args.steps

    # ---- kernel-level timing on the same stream: per shape, graphs of
    # back-to-back GEMM launches (and activation quantisations) over the rotation
    per_shape = []
    gemm_total_us = 0.0
    gemm_total_bytes = 0
    for m in MS:
        gsz = steps_g[0][MS.index(m)]
        reps = 2 * copies
        def capture(kind):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for r in range(reps):
                    gs = gsz
                    st = qg._stream(None)
                    if kind == "quant":
                        qg.check(qg.qgemm_quantize_act(FMT_INT8, gs.A.data_ptr(), m, K, K, None, gs.act.c,
                                                       gs.qws.data_ptr(), gs.qws.numel(), st))
                    else:
                        Wop = Ws[r % copies]
                        wsp, wsb = gs.ws.get(qg.qgemm_workspace_size(FMT_INT8, m, N, K, gs.cfg))
                        qg.check(qg.qgemm_run(FMT_INT8, gs.act.c, Wop.c, m, N, K, gs.cfg, wsp, wsb,
                                              gs.Y.data_ptr(), N, qg.QG_OUT_BF16, st))
            return g
        gg = capture("gemm")
        gq = capture("quant")
        for g in (gg, gq):
            g.replay()
        torch.cuda.synchronize()
        res = {}
        for name, g in (("gemm", gg), ("quant", gq)):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(5):
                g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            res[name] = 1000.0 * a.elapsed_time(b) / (5 * reps)
        gb = gemm_bytes(m)
        peak, peak_src = peaks()
        gbs = gb / (res["gemm"] * 1e-6) / 1e9
        per_shape.append({"M": m, "N": N, "K": K, "gemm_us": round(res["gemm"], 3),
                          "quant_us": round(res["quant"], 3), "gemm_bytes": gb,
                          "gemm_gbs": round(gbs, 1), "frac_hbm": round(gbs / peak, 4),
                          "config": cfgs[m].as_dict(), "table_hit": hits[m]})
        gemm_total_us += res["gemm"]
        gemm_total_bytes += gb
    # ---- every configured shape (the metric's M <= 32 decode shapes and the
    # large-M companion), single GPU only: one graph of back-to-back GEMMs per
    # shape, dispatched from the same table
    fam = None
    if world == 1 and not args.no_suite:
        fam_results, fam_peaks = time_families(HEADLINE_FAMILIES, dev, table)
        fam = dict(summarise_families(fam_results), peaks=fam_peaks,
                   block_fp8_m4096_traffic={"dram_bytes_per_launch": measured_traffic("block_fp8_m4096_dram_bytes_per_launch"),
                                            "algorithmic_bytes": shape_bytes(2, 4096, 5120, 5120),
                                            "source": "profiles/traffic.txt (ncu, hash-gated)"},
                   per_shape=[[r["format"], r["M"], r["N"], r["K"], r["us"], r["frac_roofline"], r["bound"]]
                              for r in fam_results])
    clk_step = clocks.window(t_load, t_step_end)
    clk = clocks.stop()
    clk["step_window"] = clk_step

    # ---- end to end through the public API with host buffers: per step the
    # three activations are copied in from pinned host memory (one copy: they
    # are contiguous there and on the device), the step's graph replays, the
    # results are copied out (one copy), and the host synchronises.  (The
    # copies captured inside the step's graph were slower: 75.5 against 66.2 us.)
    host_in = torch.empty(rows * K, dtype=torch.bfloat16, pin_memory=True)
    host_out = torch.empty(rows * N, dtype=torch.bfloat16, pin_memory=True)
    host_in.copy_(torch.cat([acts[m].reshape(-1) for m in MS]).cpu())

    def e2e_step(s):
        slot_in[s % nslots].copy_(host_in, non_blocking=True)
        step_graphs[s % nslots].replay()
        host_out.copy_(slot_out[s % nslots], non_blocking=True)
        stream.synchronize()
    for s in range(args.warmup):
        e2e_step(s)
    barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for s in range(args.steps):
        e2e_step(s)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_e2e = a.elapsed_time(b) / args.steps

    ms_step_max = max_over_ranks(ms_step, world, dev)
    ms_e2e_max = max_over_ranks(ms_e2e, world, dev)
    peak, peak_src = peaks()
    value = world * step_bytes() / (ms_step_max * 1e-3) / 1e9
    achieved = gemm_total_bytes / (gemm_total_us * 1e-6) / 1e9
    geo = math.exp(sum(math.log(max(p["frac_hbm"], 1e-9)) for p in per_shape) / len(per_shape))
    traffic = measured_traffic()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": bench_config(world),
        "method": {"l2": f"{copies} rotating weight copies ({copies * wbytes / 1e6:.0f} MB > 2 x {l2 / 1e6:.0f} MB L2)",
                   "step": "per M: activation quant + GEMM; the K timed steps run as CUDA graphs of up to "
                           f"{chunk} consecutive steps each (qg.capture_steps); e2e: per step one copy in from pinned "
                           "host memory, one graph replay, one copy out, sync",
                   "per_shape": "one CUDA graph of back-to-back qgemm_run launches per shape over weight copies "
                                "totalling more than 2 x L2, 5 replays after a warm one, CUDA events",
                   "table": os.path.relpath(args.table, ROOT) if table is not None else "built-in default"},
        "per_shape": per_shape,
        "int8_decode_geomean_frac_hbm_roofline": round(geo, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "the step's three INT8 GEMM launches, launch-weighted (configurations per "
                               "shape from the table: " + ", ".join(
                                   f"M={m}: " + ("decode kernel" if cfgs[m].variant == 1 else "tile kernel")
                                   for m in MS) + ")",
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                     else "fallback 6650 GB/s"},
        "e2e": {"value": round(world * step_bytes() / (ms_e2e_max * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": sum(2 * m * K for m in MS),
                "d2h_bytes_per_step": sum(2 * m * N for m in MS), "ms_per_step": round(ms_e2e_max, 5)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if fam is not None:
        # the metric over every configured shape: µs per shape and the
        # geomean fraction of roofline for M <= 32 (HBM-bound decode shapes),
        # plus the tensor-bound M >= 4096 shapes
        line["geomean_frac_roofline_M_le_32"] = round(fam["geomean_frac_roofline_M_le_32"], 4)
        line["frac_tensor_peak_M_ge_4096"] = round(fam["geomean_frac_roofline_M_ge_4096"], 4)
        line["shapes"] = fam
    if not args.no_cpu_baseline and world == 1:
        single = cpu_baseline(2)
        line["cpu_baseline_single_thread"] = {k: single[k] for k in ("value", "unit", "cores", "kind", "sample")}
        try:
            cb = cpu_baseline_all_cores()
        except Exception as exc:   # the pool is measurement harness, not the product path
            cb = dict(single, all_cores_error=f"{type(exc).__name__}: {exc}"[:200])
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "host_cores", "kind", "sample",
                                                     "all_cores_error") if k in cb}
    elif world > 1:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- suites ---
# (format, M list, (N, K) list) of the workloads the linear backend is measured
# on; the (N, K) pairs of the sweep are LLM projection shapes of the FlashInfer
# mm_fp4 benchmark list.
SWEEP_NK = [(896, 5120), (1024, 7168), (1280, 8192), (1792, 5120), (2560, 8192), (4096, 4096),
            (4608, 7168), (5120, 640), (5120, 2048), (6144, 4096), (7168, 2048), (8192, 8192)]
SUITES = {
    "fp8_tiny": [(0, [16], [(2048, 2048)])],
    "int8": [(1, [1, 8, 32], [(4096, 4096)])],
    "block_fp8": [(2, [1, 4, 16, 32], [(512, 7168), (4608, 7168), (5120, 640), (2560, 8192)])],
    "nvfp4": [(3, [1, 8, 64, 512], [(896, 1024), (1792, 5120), (5120, 2048), (1280, 8192)])],
    "sweep": [(0, [1, 2, 4, 8, 16, 32], SWEEP_NK), (2, [1, 2, 4, 8, 16, 32], SWEEP_NK)],
    "large_m": [(2, [4096, 16384], [(5120, 5120)])],
    "medium_m": [(0, [64, 128, 256, 512, 1024, 2048], [(1792, 5120), (4096, 4096), (5120, 2048), (8192, 8192)]),
                 (2, [64, 128, 256, 512, 1024, 2048], [(1792, 5120), (4096, 4096), (5120, 2048), (8192, 8192)])],
}
FMT_NAME = {0: "FP8_Dynamic", 1: "W8A8_INT8", 2: "Block_FP8", 3: "NVFP4"}


def shape_bytes(fmt, M, N, K):
    """Algorithmic bytes of one GEMM call: codes + scales of A and W, bf16 Y."""
    if fmt == 3:
        return N * K // 2 + M * K // 2 + (N + M) * K // 16 + 8 + 2 * M * N
    if fmt == 2:
        return N * K + 4 * ((N + 127) // 128) * (K // 128) + M * K + 4 * M * (K // 128) + 2 * M * N
    return N * K + 4 * N + M * K + 4 * M + 2 * M * N


def tensor_peak(fmt, bf16_tflops):
    """Dense tensor peak for the format: the measured bf16 peak times the
    nominal ratio (fp8 and int8 2x, fp4 4x)."""
    return bf16_tflops * (4.0 if fmt == 3 else 2.0)


# Mixture-of-experts layer of 128 experts, top-8 routing, hidden size 2048
# and expert intermediate size 768 (gate and up projections stacked: N = 1536,
# K = 2048; down projection: N = 2048, K = 768), at decode token counts.
MOE_EXPERTS, MOE_TOPK = 128, 8
MOE_NK = [(1536, 2048), (2048, 768)]
MOE_TOKENS = [1, 4, 16, 64]
MOE_FMTS = [0, 1, 2, 3]


def moe_routing(T, seed):
    """Seeded top-k routing: each token picks MOE_TOPK distinct experts
    uniformly.  Returns tokens per expert (assignments sorted by expert)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    picks = np.stack([rng.permutation(MOE_EXPERTS)[:MOE_TOPK] for _ in range(T)])
    return np.bincount(picks.ravel(), minlength=MOE_EXPERTS)


def run_moe_suite(args, local):
    import numpy as np
    import torch

    import precision_quantized_gemm_b200 as qg

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
    hbm = float(pk["hbm_gbs"])
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    E = MOE_EXPERTS
    results = []
    fmts = [int(x) for x in args.moe_formats.split(",")] if args.moe_formats else MOE_FMTS
    tokens = [int(x) for x in args.moe_tokens.split(",")] if args.moe_tokens else MOE_TOKENS
    for fmt in fmts:
        for (N, K) in MOE_NK:
            w = (torch.randn(E * N, K, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
            Wq = qg.quantize_weight_grouped(fmt, w, E)   # NVFP4: one tensor scale per expert
            del w
            qbw, sbw = qg.qgemm_operand_bytes(fmt, 1, N, K)   # one expert's codes / scales
            for T in tokens:
                counts = moe_routing(T, seed=1000 + T)
                rows = int(counts.sum())
                offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
                offsets = torch.from_numpy(offs).to(dev)
                active = [e for e in range(E) if counts[e] > 0]
                # algorithmic bytes: active experts' codes + scales, activations' codes + scales, bf16 y
                sb_row = 4 * (K // 128) if fmt == 2 else (K // 16 if fmt == 3 else 4)
                qrow = K // 2 if fmt == 3 else K
                w_bytes = len(active) * (qbw + (N * K // 16 + 4 if fmt == 3 else sbw))
                byts = w_bytes + rows * (qrow + sb_row) + 2 * rows * N
                # rotate weight copies past 2 x L2 so each call streams from HBM
                copies = int(max(1, min(32, (2 * l2) // max(w_bytes, 1) + 2)))
                Ws = [Wq]
                for _ in range(copies - 1):
                    o = qg.Operand(fmt, True, E * N, K, dev, n_global=E)
                    o.q.copy_(Wq.q)
                    o.scale.copy_(Wq.scale)
                    o.global_scale.copy_(Wq.global_scale)
                    Ws.append(o)
                a = torch.randn(rows, K, device=dev, generator=gen).to(torch.bfloat16)
                A = qg.quantize_act_grouped(fmt, a, offsets)   # NVFP4: per-expert scale atoms
                cfg = qg.qgemm_grouped_default_config(fmt, E, rows, N, K)
                ws = qg.Workspace(dev)
                wsp, wsb = ws.get(qg.qgemm_workspace_size(fmt, rows, N, K, cfg))
                Y = torch.empty(rows, N, dtype=torch.bfloat16, device=dev)
                reps = max(2 * copies, 8)

                def grouped(Wo, st):
                    qg.check(qg.qgemm_run_grouped(fmt, E, offsets.data_ptr(), A.c, Wo.c, N, K, cfg, wsp, wsb,
                                                  Y.data_ptr(), N, 0, st))

                # the baseline: one qgemm_run per active expert on its slices
                ecfg = {e: qg.qgemm_default_config(fmt, int(counts[e]), N, K) for e in active}
                ews = qg.Workspace(dev)
                ewsp, ewsb = ews.get(max(qg.qgemm_workspace_size(fmt, int(counts[e]), N, K, ecfg[e])
                                         for e in active))

                # NVFP4: expert e's activation scales start at its first 128-row atom
                sf_row0, r = {}, 0
                for e in range(E):
                    sf_row0[e] = r
                    r += -(-int(counts[e]) // 128) * 128

                def per_expert(Wo, st):
                    for e in active:
                        m0, m = int(offs[e]), int(counts[e])
                        if fmt == 3:
                            s_a = A.scale.data_ptr() + sf_row0[e] * ((K + 255) // 256 * 16)
                            g_w = Wo.global_scale.data_ptr() + 4 * e
                        else:
                            s_a = A.scale.data_ptr() + m0 * sb_row
                            g_w = Wo.global_scale.data_ptr()
                        s_w = Wo.scale.data_ptr() + e * sbw
                        Ae = qg.qg_operand(A.q.data_ptr() + m0 * qrow, s_a, A.global_scale.data_ptr(), m, K)
                        We = qg.qg_operand(Wo.q.data_ptr() + e * qbw, s_w, g_w, N, K)
                        qg.check(qg.qgemm_run(fmt, Ae, We, m, N, K, ecfg[e], ewsp, ewsb,
                                              Y.data_ptr() + m0 * N * 2, N, 0, st))

                times = {}
                for name, fn in (("grouped", grouped), ("per_expert", per_expert)):
                    fn(Ws[0], qg._stream(None))
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        st = qg._stream(None)
                        for r in range(reps):
                            fn(Ws[r % copies], st)
                    g.replay()
                    torch.cuda.synchronize()
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    for _ in range(5):
                        g.replay()
                    e1.record()
                    torch.cuda.synchronize()
                    times[name] = 1000.0 * e0.elapsed_time(e1) / (5 * reps)
                    del g
                us = times["grouped"]
                t_hbm = byts / (hbm * 1e9) * 1e6
                rec = {"suite": "moe", "format": FMT_NAME[fmt], "experts": E, "top_k": MOE_TOPK, "tokens": T,
                       "assignments": rows, "active_experts": len(active), "N": N, "K": K, "us": round(us, 3),
                       "GB/s": round(byts / us / 1e3, 1), "bound": "hbm", "roofline_us": round(t_hbm, 3),
                       "frac_roofline": round(t_hbm / us, 4), "per_expert_launches_us": round(times["per_expert"], 3),
                       "speedup_vs_per_expert": round(times["per_expert"] / us, 2), "config": cfg.as_dict(),
                       "rotating_copies": copies}
                print(json.dumps(rec), flush=True)
                results.append(rec)
                del Ws[1:], Y, A
                torch.cuda.empty_cache()
    fr = [r["frac_roofline"] for r in results]
    sp = [r["speedup_vs_per_expert"] for r in results]
    print(json.dumps({"summary": True, "suite": "moe", "shapes": len(results),
                      "geomean_frac_roofline": math.exp(sum(math.log(x) for x in fr) / len(fr)),
                      "geomean_speedup_vs_per_expert": math.exp(sum(math.log(x) for x in sp) / len(sp)),
                      "peaks": {"hbm_gbs": hbm}}), flush=True)


def rotation(qg, torch, Wq, fmt, rows, K, is_weight, total_min, dev, cap=4096):
    """Copies of a quantised operand in one pool, enough that their total
    exceeds `total_min` bytes (so a pass over them streams from HBM): returns
    (qg_operand structs, pool tensor that owns them)."""
    qb, sb = Wq.q.numel(), Wq.scale.numel()
    qs, ss = -(-qb // 256) * 256, -(-sb // 256) * 256
    per = qs + ss
    copies = int(max(2, min(cap, -(-total_min // (qb + sb)) + 2)))
    pool = torch.empty(copies, per, dtype=torch.uint8, device=dev)
    pool[0, :qb].copy_(Wq.q)
    pool[0, qs:qs + sb].copy_(Wq.scale)
    pool[1:].copy_(pool[0].expand(copies - 1, per))
    base = pool.data_ptr()
    ops = [qg.qg_operand(base + i * per, base + i * per + qs, Wq.global_scale.data_ptr(), rows, K)
           for i in range(copies)]
    return ops, pool


def time_shape(qg, torch, dev, fmt, M, N, K, Wq, cfg, l2, hbm, bf16, gen, single=False):
    """Device time of one qgemm_run of this shape: a CUDA graph of back-to-back
    launches (programmatic dependent launch on) over weight copies whose
    total exceeds 2 x L2 (and activation copies for M >= 4096), replayed
    after one warm replay, CUDA events on the launching stream."""
    flops = 2.0 * M * N * K
    byts = shape_bytes(fmt, M, N, K)
    a = torch.randn(M, K, device=dev, generator=gen).to(torch.bfloat16)
    A0 = qg.quantize_act(fmt, a)
    del a
    large = M >= 4096
    if large:
        Wrot, wpool = rotation(qg, torch, Wq, fmt, N, K, True, 2 * l2, dev, cap=16)
        Arot, apool = rotation(qg, torch, A0, fmt, M, K, False, 2 * l2, dev, cap=16)
        n = max(len(Wrot), len(Arot))
    else:
        Wrot, wpool = rotation(qg, torch, Wq, fmt, N, K, True, 2 * l2, dev)
        Arot, apool = [A0.c], None
        n = len(Wrot)
    ws = qg.Workspace(dev)
    wsp, wsb = ws.get(qg.qgemm_workspace_size(fmt, M, N, K, cfg))
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    reps = max(n, 8) if not large else 2 * n
    st = qg._stream(None)
    qg.check(qg.qgemm_run(fmt, Arot[0], Wrot[0], M, N, K, cfg, wsp, wsb, Y.data_ptr(), N, 0, st))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = qg._stream(None)
        for r in range(reps):
            qg.check(qg.qgemm_run(fmt, Arot[r % len(Arot)], Wrot[r % len(Wrot)], M, N, K, cfg, wsp, wsb,
                                  Y.data_ptr(), N, 0, st))
    g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_rep = 5 if not large else 2
    e0.record()
    for _ in range(n_rep):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = 1000.0 * e0.elapsed_time(e1) / (n_rep * reps)
    rec = {}
    if single:
        # one eager call on its own (after a sync, events on the same
        # stream): the device waits from the first event for the host's
        # submission (argument checks, two tensor map encodings, the launch),
        # so this is an eager call's cost from call to completion, with no
        # neighbour to overlap; its weight copy was last read a rotation ago
        st = qg._stream(None)
        e0.record()
        qg.check(qg.qgemm_run(fmt, Arot[reps % len(Arot)], Wrot[reps % len(Wrot)], M, N, K, cfg, wsp, wsb,
                              Y.data_ptr(), N, 0, st))
        e1.record()
        torch.cuda.synchronize()
        rec["single_launch_us"] = round(1000.0 * e0.elapsed_time(e1), 3)
    del g, Wrot, wpool, Arot, apool, Y, A0
    t_hbm = byts / (hbm * 1e9) * 1e6
    t_tc = flops / (tensor_peak(fmt, bf16) * 1e12) * 1e6
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    frac = max(t_hbm, t_tc) / us
    return dict({"format": FMT_NAME[fmt], "M": M, "N": N, "K": K, "us": round(us, 3),
                 "GB/s": round(byts / us / 1e3, 1), "TFLOP/s": round(flops / us / 1e6, 2), "bound": bound,
                 "roofline_us": round(max(t_hbm, t_tc), 3), "frac_roofline": round(frac, 4),
                 "config": cfg.as_dict(), "rotating_copies": n}, **rec)


def geomean(xs):
    xs = list(xs)
    return math.exp(sum(math.log(max(x, 1e-9)) for x in xs) / len(xs)) if xs else None


def time_families(names, dev, table, only_m=None, single=False, emit=None):
    """Per-shape device times of every shape of the named workload families,
    each with the configuration the table dispatches (or the scored
    default).  Returns the records; `emit` sees each as it is made."""
    import torch

    import precision_quantized_gemm_b200 as qg

    pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
    hbm, bf16 = float(pk["hbm_gbs"]), float(pk["bf16_tflops"])
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    results = []
    for name in names:
        for fmt, Ms, NKs in SUITES[name]:
            if only_m:
                Ms = [m for m in Ms if m in only_m]
                if not Ms:
                    continue
            for (N, K) in NKs:
                w = (torch.randn(N, K, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
                Wq = qg.quantize_weight(fmt, w)
                del w
                for M in Ms:
                    cfg, hit = (table.dispatch(fmt, M, N, K) if table is not None
                                else (qg.qgemm_default_config(fmt, M, N, K), 0))
                    rec = dict({"suite": name}, **time_shape(qg, torch, dev, fmt, M, N, K, Wq, cfg, l2, hbm, bf16,
                                                              gen, single=single))
                    rec["table_hit"] = hit
                    results.append(rec)
                    if emit:
                        emit(rec)
                    torch.cuda.empty_cache()
                del Wq
    return results, {"hbm_gbs": hbm, "bf16_tflops": bf16,
                     "note": "fp8/int8 tensor peak = 2 x measured bf16, fp4 = 4 x"}


# The families of the headline metric (M <= 32 decode shapes) and its
# large-M companion: every configured workload.
HEADLINE_FAMILIES = ["fp8_tiny", "int8", "block_fp8", "nvfp4", "sweep", "large_m"]


def summarise_families(results):
    small = [r["frac_roofline"] for r in results if r["M"] <= 32]
    medium = [r["frac_roofline"] for r in results if 32 < r["M"] < 4096]
    large = [r["frac_roofline"] for r in results if r["M"] >= 4096]
    by_fmt = {}
    for r in results:
        if r["M"] <= 32:
            by_fmt.setdefault(r["format"], []).append(r["frac_roofline"])
    return {"shapes": len(results), "shapes_M_le_32": len(small),
            "geomean_frac_roofline_M_le_32": geomean(small),
            "geomean_frac_roofline_M_33_to_4095": geomean(medium),
            "geomean_frac_roofline_M_ge_4096": geomean(large),
            "geomean_frac_roofline_all": geomean(r["frac_roofline"] for r in results),
            "geomean_frac_roofline_M_le_32_by_format": {k: round(geomean(v), 4) for k, v in by_fmt.items()}}


def run_suite(args, names, local):
    import torch

    import precision_quantized_gemm_b200 as qg

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    table = qg.Table(args.table) if os.path.exists(args.table) else None
    only = {int(x) for x in args.only_m.split(",")} if args.only_m else None
    results, peaks_used = time_families(names, dev, table, only_m=only, single=True,
                                        emit=lambda r: print(json.dumps(r), flush=True))
    print(json.dumps(dict({"summary": True}, **summarise_families(results), peaks=peaks_used)), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup()
    try:
        if args.suite:
            names = [s.strip() for s in args.suite.split(",") if s.strip()]
            if "moe" in names:
                run_moe_suite(args, local)
                names.remove("moe")
            if names:
                run_suite(args, names, local)
        elif args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
