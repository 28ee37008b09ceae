#!/usr/bin/env python
"""Benchmark of the RQ-LUT logits serving step on B200.

One step = the whole hot path for one batch of B tokens on the Gemma-2
shaped artifact (V=256000, D=2304, M=384, L=2, K=1024, uint16 codes):
build the per-token lookup tables, stream the code matrix once with lookup +
sum, Gemma-2 softcap, write the fp32 logits and the argmax, then rebuild the
bf16 input rows of the B tokens picked (the next step's embeddings).
Default workload: decode batch 1.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  `value` = vocabulary rows scored per second
over all ranks (V * B * steps / max-over-ranks device time); the code matrix
(393 MB) is larger than L2, so every step streams it from HBM.
Multi-GPU: independent replicas, one per rank (no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lut_logits_serving_b200 import synth  # noqa: E402

METRIC = "LUT logits vocab-rows/s & µs/call at V=256000 (1 B200), % of HBM roofline"
UNIT = "vocab-rows/s"
ENC_METRIC = "RQ encode rows/s (greedy residual nearest codeword, fp32), % of FP32-pipe roofline"
DEC_METRIC = "input rows rebuilt/s (bf16, Zipf ids, L2 flushed between calls), % of HBM roofline"
DEC_UNIT = "rows/s"
ENC_UNIT = "rows/s"
# FP32 pipe: 148 SMs x 128 lanes per clock (B200); the clock is the sampled
# maximum (clocks.max.sm), 1965 MHz when no sample exists.
SMS, FP32_LANES, NOMINAL_SM_MHZ = 148, 128, 1965.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="g2_b1",
                    choices=["g2_b1", "g2_b1_packed10", "g2_b16", "g2_b32", "packed_b64", "mlp_gate_b1",
                             "mlp_down_b1", "encode_g2", "g2_b1_topk50", "decode512"])
    ap.add_argument("--codes", default=None, choices=["u16", "sched", "u8", "rot10"],
                    help="code layout of the unpacked workloads timed for `value`: "
                         "bank-scheduled once by rq_prepare_sched (the default at B <= 4), as "
                         "drawn (the default for batches, whose full token groups decode rows "
                         "on the tensor cores), or one byte per code; the other layouts are "
                         "reported under other_layouts")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sustain-seconds", type=float, default=1.0,
                    help="after the timed steps, replay the same step for this long so the "
                         "clock record has samples under load (0: skip)")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the workload alone (by default the batch-1 run also measures "
                         "g2_b32, packed_b64, decode512 and batch 1 on packed codes)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


def workload_config(w, codes="u16"):
    rb = code_bytes(w, codes) // w.V
    fmt = (f"packed10 ({rb} B/row)" if w.packed10 or codes == "packed10" else
           f"10-bit ({rb} B/row) in the rotated slices of rq_prepare_rot10" if codes == "rot10" else
           f"uint16 ({rb} B/row)" if codes == "u16" else
           f"uint8 ({rb} B/row, K <= 256)" if codes == "u8" else
           f"uint16 ({rb} B/row) in the bank-scheduled order of rq_prepare_sched")
    if w.argmax:
        what = (f"softcap {w.softcap:g}, logits + argmax, then the {w.B} picked tokens' input "
                f"rows rebuilt (bf16)")
    elif w.topk:
        what = (f"softcap {w.softcap:g}, logits, top-{w.topk} + draw at temperature "
                f"{w.temperature:g}, then the drawn tokens' input rows rebuilt (bf16)")
    else:
        what = "y = W x, no softcap (RQ-coded MLP weight)"
    return {
        "workload": f"{w.name}: V={w.V} D={w.D} M={w.M} L={w.L} K={w.K} B={w.B}, {fmt} codes, "
                    f"{what}",
        "V": w.V, "D": w.D, "M": w.M, "L": w.L, "K": w.K, "B": w.B,
        "codes": "packed10" if w.packed10 else codes,
        "l2": ("inputs larger than L2: the code matrix is streamed from HBM every step"
               if code_bytes(w, codes) > 2 * 126 * 2**20 else
               "inputs smaller than L2: a 256 MB buffer is written between timed steps"),
    }


def headline_layout(w, codes=None, available=("sched", "u16", "u8")):
    """Code layout timed for `value` (both arms name it in `config`): 10-bit
    packed workloads are packed; otherwise --codes if given, else the
    bank-scheduled layout at B <= 4 and the drawn uint16 layout for batches
    (whose full token groups decode rows on the tensor cores)."""
    if w.packed10:
        return "packed10"
    if codes in available:
        return codes
    return "sched" if w.B <= 4 else "u16"


def code_bytes(w, codes="u16"):
    if w.packed10 or codes == "packed10":
        return w.V * (w.P * 10 // 8)
    if codes == "rot10":                      # packed rows + one rotation byte per slice
        return w.V * (w.P * 10 // 8 + w.P // 32)
    return w.V * w.P * (1 if codes == "u8" else 2)


# --------------------------------------------------------- multi-rank math

def aggregate(local_ms, world, device="cpu"):
    """Job time of a weak-scaling replica run: the slowest rank's device time
    (all_reduce MAX over the default process group when world > 1)."""
    if world <= 1:
        return float(local_ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(units_per_rank, world, job_ms):
    """Whole-job rate: units processed by all ranks over the job time."""
    return world * units_per_rank / (job_ms / 1e3)


def parallelism():
    """The config key both arms print: one replica per rank."""
    return f"replicas x{int(os.environ.get('WORLD_SIZE', '1'))}"


def rank_seed(rank):
    """Each replica scores its own seeded batch and artifact."""
    return 1000 * rank


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (every 100 ms) of the SM clock and the throttle
    reasons.  A reader thread stamps each sample with the host time it
    arrived; `window()` / `close_window()` bracket the region of interest and
    `summary()` keeps the samples inside it (all samples when no window was
    opened)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []            # (host time, line)
        self.t_open = self.t_close = None
        self._thread = None
        self._first = None

    def __enter__(self):
        import threading
        self._first = threading.Event()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self

        def read():
            for line in self.proc.stdout:
                self.lines.append((time.monotonic(), line))
                self._first.set()
        self._thread = threading.Thread(target=read, daemon=True)
        self._thread.start()
        return self

    def wait_first(self, timeout=5.0):
        """Block until the sampler has produced its first line (it takes
        nvidia-smi a moment to start), so the timed region is covered."""
        if self.proc is not None:
            self._first.wait(timeout)

    def window(self):
        self.t_open = time.monotonic()

    def close_window(self):
        self.t_close = time.monotonic()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            if self._thread is not None:
                self._thread.join(timeout=5)

    @property
    def out(self):
        return "".join(l for _, l in self.lines)

    def summary(self):
        rows = []
        lo = self.t_open if self.t_open is not None else -1e300
        hi = self.t_close if self.t_close is not None else 1e300
        for t, line in self.lines:
            if not (lo <= t <= hi):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def cpu_info():
    """Host cores and CPU model of the box the oracle is timed on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


# ------------------------------------------------------------ CPU oracle

def oracle_step_fn(w, data):
    """One pass of the whole path in the CPU oracle (fp64 tables and sums,
    softcap, argmax, input-row decode), optionally on a subset of rows."""
    import oracle

    def step(rows=None):
        T = oracle.lut_build(data["h"], data["C"], "f64")
        z = oracle.logits_lut(data["codes"], T, rows)
        y = oracle.softcap(z, w.softcap)
        if w.topk:
            _, _, pick = oracle.sample(y.astype(np.float32), w.topk, w.temperature, 1234, 0)
        else:
            pick = oracle.argmax(y.astype(np.float32))
        oracle.decode_rows_bf16(data["ids"], data["codes"], data["C"], w.decode_scale)
        return pick
    return step


def cpu_baseline(w, data, seconds, threads=0):
    """Time the oracle as it stands on full-vocabulary steps until `seconds`
    (threads < 1: all host cores, else that many)."""
    import oracle
    used = oracle.set_threads(threads)
    try:
        step = oracle_step_fn(w, data)
        n, t0 = 0, time.perf_counter()
        while True:
            step()
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    finally:
        oracle.set_threads(0)
    pick = f"top-{w.topk} draw" if w.topk else "argmax"
    return dict({"value": w.V * w.B * n / el, "unit": UNIT, "cores": used, "kind": "oracle",
                 "sample": f"{n} full steps of {w.name} (all {w.V} rows x {w.B} tokens, fp64 "
                           f"tables, softcap, {pick}, row decode), C with {used} OpenMP "
                           f"thread(s) over vocabulary rows, {el:.1f} s"}, **cpu_info())


def encode_terms(w, rows):
    """Distance terms (one fp32 subtract + one fma each) of encoding `rows`."""
    return rows * w.M * w.L * w.K * w.ds


def run_reference_encode(args, w):
    import oracle
    threads = oracle.set_threads(0)
    data = synth.make(w, V=4096)
    X, C = data["X"], data["C"]
    t0 = time.perf_counter()
    oracle.encode(X[:4], C)
    per_row = (time.perf_counter() - t0) / 4
    budget = 120.0 / max(1, args.steps + args.warmup)
    nrows = int(max(1, min(X.shape[0], budget / max(per_row, 1e-9))))
    for _ in range(args.warmup):
        oracle.encode(X[:nrows], C)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.encode(X[:nrows], C)
    el = time.perf_counter() - t0
    value = nrows * args.steps / el
    line = {
        "impl": "reference", "metric": ENC_METRIC, "value": value, "unit": ENC_UNIT,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(encode_config(w), parallelism=parallelism()),
        "cpu_baseline": dict({"value": value, "unit": ENC_UNIT, "cores": threads, "kind": "oracle",
                              "sample": f"{nrows} of {w.V} rows per step, {threads} OpenMP "
                                        f"thread(s) over rows"}, **cpu_info()),
        "e2e": {"value": value, "unit": ENC_UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def decode_config(w):
    return {"workload": f"{w.name}: {w.n_ids} ids drawn Zipf(s={w.zipf_s:g}) over V={w.V} rows "
                        f"(repeats kept), each rebuilt from M={w.M} x L={w.L} uint16 codes and "
                        f"K={w.K} codebooks, x {w.decode_scale:g}, bf16 rows of D={w.D}",
            "V": w.V, "D": w.D, "M": w.M, "L": w.L, "K": w.K, "ids": w.n_ids,
            "l2": "inputs smaller than L2: a 256 MB buffer is written between timed calls"}


def decode_bytes(w):
    """Bytes a call touches: each id's code row, its L codewords per subspace
    and its bf16 output row (repeated ids counted again)."""
    return w.n_ids * (w.P * 2 + w.P * w.ds * 4 + w.D * 2)


def run_reference_decode(args, w):
    import oracle
    threads = oracle.set_threads(0)
    data = synth.make(w)
    ids, codes, C = data["ids"], data["codes"], data["C"]
    # each step rebuilds the first n ids, n sized so that warmup + steps end
    # within about two minutes
    t0 = time.perf_counter()
    oracle.decode_rows_bf16(ids, codes, C, w.decode_scale)
    per_id = (time.perf_counter() - t0) / w.n_ids
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(w.n_ids, budget / max(per_id, 1e-9))))
    sample = ids[:n]
    for _ in range(args.warmup):
        oracle.decode_rows_bf16(sample, codes, C, w.decode_scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.decode_rows_bf16(sample, codes, C, w.decode_scale)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    line = {
        "impl": "reference", "metric": DEC_METRIC, "value": value, "unit": DEC_UNIT,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(decode_config(w), parallelism=parallelism()),
        "cpu_baseline": dict({"value": value, "unit": DEC_UNIT, "cores": threads, "kind": "oracle",
                              "sample": f"the first {n} of the {w.n_ids} ids per step, "
                                        f"{threads} OpenMP thread(s) over ids"}, **cpu_info()),
        "e2e": {"value": value, "unit": DEC_UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def encode_config(w):
    return {"workload": f"{w.name}: encode V={w.V} rows of D={w.D} fp32 against M={w.M} x "
                        f"L={w.L} codebooks of K={w.K} ({w.ds}-dim) codewords -> uint16 codes",
            "V": w.V, "D": w.D, "M": w.M, "L": w.L, "K": w.K,
            "l2": "inputs larger than L2: the 2.36 GB of rows are read every step"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if w.encode:
        return run_reference_encode(args, w)
    if w.B == 0:
        return run_reference_decode(args, w)
    import oracle
    threads = oracle.set_threads(0)
    data = synth.make(w)
    step = oracle_step_fn(w, data)
    # size each step's row sample so that warmup + steps end within ~2 minutes
    probe = np.arange(min(w.V, 20000), dtype=np.int64)
    t0 = time.perf_counter()
    step(probe)
    per_row = (time.perf_counter() - t0) / probe.size
    budget = 120.0 / max(1, args.steps + args.warmup)
    nrows = int(max(1000, min(w.V, budget / max(per_row, 1e-9))))
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(w.V, nrows, replace=False)).astype(np.int64)
    for _ in range(args.warmup):
        step(rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(rows)
    el = time.perf_counter() - t0
    value = nrows * w.B * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": dict(workload_config(w, headline_layout(w, args.codes)),
                       parallelism=parallelism()),
        "cpu_baseline": dict({"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                              "sample": f"{nrows} of {w.V} rows per step, {w.B} token(s), "
                                        f"{threads} OpenMP thread(s) over rows"}, **cpu_info()),
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- our arm

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tf32_peak():
    """Dense tf32 tensor peak (TFLOP/s): the measured bf16 burst figure times
    the nominal tf32/bf16 ratio (1.1 / 2.25 PFLOP/s dense)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]) * 1.1 / 2.25, "measured bf16 x 1.1/2.25"
    return 1590.0 * 1.1 / 2.25, "fallback bf16 x 1.1/2.25"


# Shared memory delivers 128 bytes per clock per SM (32 banks x 4 bytes).
SMEM_BYTES_PER_CLK = 128


def smem_peak(mhz):
    """Aggregate shared-memory bandwidth (GB/s) at an SM clock."""
    return SMS * SMEM_BYTES_PER_CLK * (mhz or NOMINAL_SM_MHZ) * 1e6 / 1e9


def kernel_source_hash(kernel="logits_chunk"):
    """Hash of the sources a kernel is built from (its .cu file and the common
    header), to tell whether committed ncu counters still describe it."""
    src = ("logits_decode_mma.cu" if kernel.startswith("logits_decode_mma") else
           "decode_rows.cu" if kernel.startswith("decode_rows") else
           "lut_build.cu" if kernel.startswith("lut_build") else
           "logits_l2.cu" if kernel.startswith("logits_l2") else "logits_chunk.cu")
    h = hashlib.sha256()
    for name in (src, "rq_common.cuh"):
        with open(os.path.join(ROOT, "lut_logits_serving_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(kernel)
    if not e or e.get("source_sha") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


def topk_launches(V, k):
    """Kernels of one rq_topk_sample call: the histogram pass and the gather
    pass whose last CTA per token sorts and draws (plus a memset)."""
    return 2


def decodable(w):
    """Full token groups (64, then 32) of uint16, bank-scheduled or 10-bit
    packed codes at ds = 6, L = 2 decode their rows on the tensor cores."""
    return (w.ds == 6 and w.L == 2 and 16 <= w.K <= 1024 and w.B >= 32 and
            w.M % (32 if w.packed10 else 8) == 0)


def token_groups(w, decoded):
    groups, b0 = [], 0
    while b0 < w.B:
        g = 64 if decoded and w.B - b0 >= 64 else 32 if decoded and w.B - b0 >= 32 else \
            min(32, w.B - b0)
        groups.append(g)
        b0 += g
    return groups


def launches_per_step(w, decoded):
    """Kernels of one step: (table build, tiled pass, reduce) at B <= 4, else
    two kernels per token group (hidden split + tensor-core decode, or table
    build + L2 pass); then the argmax finish that also rebuilds the picked
    rows, or the top-k draw and the row decode."""
    if w.B <= 4 and (not w.packed10 or w.B == 1):
        n = 3 + (1 if w.argmax else 0)
    else:
        n = 2 * len(token_groups(w, decoded)) + (1 if w.argmax else 0)
    if w.topk:
        n += topk_launches(w.V, w.topk) + 1
    return n


class Rig:
    """Our arm's process state: ranks, the launching stream, and the timing
    helpers (CUDA events on that stream, barrier + max over ranks)."""

    def __init__(self, args):
        import torch
        import torch.distributed as dist
        self.torch, self.dist, self.args = torch, dist, args
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world != args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={self.world}")
        torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", self.local))
        self.stream = torch.cuda.current_stream()
        self.graphs = []

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, x):
        return aggregate(x, self.world, device="cuda")

    def close(self):
        self.graphs.clear()
        if self.world > 1:
            self.dist.barrier()
            self.dist.destroy_process_group()

    def graphed(self, step):
        """Warm `step` up, then capture it as a CUDA graph (unless --no-graph)."""
        torch = self.torch
        for _ in range(max(3, self.args.warmup)):
            step()
        torch.cuda.synchronize()
        if self.args.no_graph:
            return step
        s2 = torch.cuda.Stream()
        s2.wait_stream(self.stream)
        with torch.cuda.stream(s2):
            step()
        self.stream.wait_stream(s2)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        self.graphs.append(g)
        return g.replay

    def time_steps(self, run, n, flush=None):
        """Device time (ms) of n steps, max over ranks.  With `flush` each step
        is timed alone and the buffer is written between steps."""
        torch = self.torch
        self.barrier()
        torch.cuda.synchronize()
        if flush is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            for _ in range(n):
                run()
            e1.record(self.stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(n)]
            for a0, a1 in evs:
                flush.fill_(1)
                a0.record(self.stream)
                run()
                a1.record(self.stream)
            torch.cuda.synchronize()
            ms = sum(a0.elapsed_time(a1) for a0, a1 in evs)
        self.barrier()
        return self.max_over_ranks(ms)

    def code_pass_us(self, step, n, flush=None):
        """Mean device time (us) of the code-streaming pass alone: profile
        events the library records around it on the launching stream."""
        torch = self.torch
        import lut_logits_serving_b200 as rq
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        stops = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for ev in starts + stops:       # torch creates the CUDA event on first record
            ev.record(self.stream)
        torch.cuda.synchronize()
        for i in range(n):
            if flush is not None:
                flush.fill_(1)
            rq.rq_set_profile_events(starts[i], stops[i])
            step()
        rq.rq_set_profile_events(None, None)
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in zip(starts, stops)])) * 1e3


class Artifact:
    """The resident RQ artifact on the device: codebooks and the code matrix
    in each layout a step may read (prepared once, outside timed regions)."""

    def __init__(self, w, data, need=("sched", "u16", "u8", "packed10", "rot10")):
        import torch
        import lut_logits_serving_b200 as rq
        self.d = rq.dims(w.V, w.D, w.M, w.L, w.K)
        self.C = torch.from_numpy(data["C"]).cuda()
        c16 = torch.from_numpy(data["codes"].reshape(w.V, -1)).cuda()
        self.layouts = {}
        self.sched_passes = None
        if "packed10" in need and w.K <= 1024:
            self.layouts["packed10"] = (rq.PACKED10, rq.rq_pack10(c16, self.d))
        if "sched" in need and w.K <= 1024 and w.P % 32 == 0:
            sched, (st, ps) = rq.rq_prepare_sched(c16, self.d, stats=True)
            self.layouts["sched"] = (rq.SCHED, sched)
            self.sched_passes = ps / st
        self.rot_passes = None
        if "rot10" in need and w.K <= 1024 and w.P % 64 == 0:
            rot, (st, ps) = rq.rq_prepare_rot10(c16, self.d, stats=True)
            self.layouts["rot10"] = (rq.ROT10, rot)
            self.rot_passes = ps / st
        if "u8" in need and w.K <= 256:
            self.layouts["u8"] = (rq.U8, rq.rq_pack8(c16, self.d))
        if "u16" in need:
            self.layouts["u16"] = (rq.U16, c16)

    def bytes(self, layout):
        t = self.layouts[layout][1]
        return t.numel() * t.element_size() + self.C.numel() * 4


def kernel_of(w, layout):
    decoded = layout in ("u16", "packed10", "sched") and decodable(w)
    packed = w.packed10 or layout in ("packed10", "rot10")
    if w.B <= 4 and (not packed or w.B == 1):
        return "logits_chunk_u16_kernel", decoded
    return ("logits_decode_mma_kernel" if decoded else "logits_l2_kernel"), decoded


def measure_logits(rig, w, art, layout, h_np, full=False, clk=None):
    """Time one workload's step on the resident artifact: K steps as CUDA-graph
    replays, the code pass alone, end to end from host buffers, and the
    device memory the step adds.  With `full`, also the other code layouts and
    the kernel choices of full token groups; with `clk`, the timed steps and
    a sustained run of at least a second after them are the clock window."""
    torch, args = rig.torch, rig.args
    import lut_logits_serving_b200 as rq
    d, dC = art.d, art.C
    fmt, dcodes = art.layouts[layout]
    stream = rig.stream
    dh0 = torch.from_numpy(h_np).cuda()

    def outputs():
        return (torch.empty((w.B, w.V), dtype=torch.float32, device="cuda"),
                torch.empty((w.B,), dtype=torch.int32, device="cuda"),
                torch.empty((w.B, w.D), dtype=torch.bfloat16, device="cuda"),
                torch.empty((w.B,), dtype=torch.int32, device="cuda"))
    logits0, am0, rows0, tok0 = outputs()
    tws = (torch.empty(rq.rq_topk_workspace_bytes(w.V, w.B, w.topk), dtype=torch.uint8,
                       device="cuda") if w.topk else None)

    def make_step(fmt, codes, out=None):
        ws = torch.empty(rq.rq_fused_workspace_bytes(d, w.B, fmt, True), dtype=torch.uint8,
                         device="cuda")
        # the step's input and outputs (a second set lets the end-to-end loop
        # overlap the copies of one step with the compute of another)
        dh, logits, am, rows, tok = out if out is not None else (dh0, logits0, am0, rows0, tok0)

        if w.topk:
            def step():
                # logits, the top-k draw, and the drawn tokens' input rows
                rq.rq_logits_from_hidden(dh, dC, codes, fmt, d, w.softcap, logits=logits, ws=ws)
                rq.rq_topk_sample(logits, w.topk, w.temperature, seed=1234, step=0, token=tok,
                                  want_topk=False, ws=tws)
                rq.rq_decode_rows(tok, codes, fmt, dC, d, w.decode_scale, out=rows)
        elif not w.argmax:
            def step():
                # an RQ-coded weight matrix applied without reconstruction
                rq.rq_logits_from_hidden(dh, dC, codes, fmt, d, w.softcap, logits=logits, ws=ws)
        else:
            def step():
                # logits of this step's hidden states, the greedy picks, and the
                # input rows of the picked tokens (the next step's embeddings)
                rq.rq_greedy_step(dh, dC, codes, fmt, d, w.softcap, scale=w.decode_scale,
                                  logits=logits, argmax=am, rows=rows, ws=ws)
        step.ws_bytes = ws.numel()
        return step

    # Inputs smaller than twice the 126 MB L2 would stay cached between steps:
    # then every step is timed by its own event pair and a 256 MB buffer is
    # written between steps, outside the pairs.
    flush = None
    if code_bytes(w, layout) + dC.numel() * 4 < 2 * 126 * 2**20:
        flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")

    step = make_step(fmt, dcodes)
    run = rig.graphed(step)

    # ---- timed region: K steps, device time, max over ranks
    if clk is not None:
        clk.wait_first()
        clk.window()
    t_ms = rig.time_steps(run, args.steps, flush)
    sustained = None
    if clk is not None:
        # the same step replayed for at least a second, so that the clock
        # record has samples under this load
        per = max(t_ms / args.steps, 1e-3)
        n_sus = int(min(200000, 1000.0 * args.sustain_seconds / per))
        if n_sus > 0:
            s_ms = rig.time_steps(run, n_sus, flush)
            sustained = {"steps": n_sus, "seconds": s_ms / 1e3,
                         "us_per_step": s_ms / n_sus * 1e3}
        else:
            sustained = {"steps": 0, "seconds": 0.0, "us_per_step": None}
        clk.close_window()
    res = {"us_per_call": t_ms / args.steps * 1e3,
           "value": throughput(w.V * w.B * args.steps, rig.world, t_ms),
           "unit": UNIT, "steps": args.steps, "codes": layout, "t_ms": t_ms,
           "sustained": sustained}

    # ---- the dominant kernel alone, live CUDA events
    kern_us = rig.code_pass_us(step, min(args.steps, 2000), flush)
    peak, peak_kind = load_peaks()
    algo_bytes = code_bytes(w, layout)
    achieved = algo_bytes / (kern_us / 1e6) / 1e9
    kname, decoded = kernel_of(w, layout)
    kkey = f"{kname}/{layout}/{w.name}"
    res["roofline"] = {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
                       "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                       "traffic": profiled_traffic(kkey), "algorithmic_bytes": algo_bytes,
                       "kernel_us": kern_us}
    res["step_hbm_frac"] = algo_bytes / (t_ms / args.steps / 1e3) / 1e9 / peak
    if decoded:
        # the decode-then-multiply kernels: their binding pipes, on
        # algorithmic work (2 B V D flops; two L-level codeword gathers of ds
        # fp32 per row and subspace, per group)
        groups = token_groups(w, True)
        flops = 2.0 * w.B * w.V * w.D
        tpk, tpk_kind = tf32_peak()
        smem_bytes = len(groups) * w.V * w.M * w.L * w.ds * 4
        mhz = (clk.summary().get("sm_mhz") if clk is not None else None) or NOMINAL_SM_MHZ
        res["pipes"] = {
            "tensor": {"achieved": flops / (kern_us / 1e6) / 1e12, "peak": tpk,
                       "peak_kind": tpk_kind, "unit": "TFLOP/s",
                       "frac": flops / (kern_us / 1e6) / 1e12 / tpk},
            "smem": {"achieved": smem_bytes / (kern_us / 1e6) / 1e9,
                     "peak": smem_peak(mhz), "unit": "GB/s",
                     "peak_kind": f"derived: {SMS} SMs x {SMEM_BYTES_PER_CLK} B x {mhz:g} MHz",
                     "frac": smem_bytes / (kern_us / 1e6) / 1e9 / smem_peak(mhz),
                     "algorithmic_bytes": smem_bytes}}

    # ---- device memory: the resident artifact, the caller's workspace, and
    # what a step adds on top (the library allocates nothing itself)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    step()
    torch.cuda.synchronize()
    res["memory"] = {"resident_bytes": art.bytes(layout), "workspace_bytes": step.ws_bytes,
                     "peak_delta_bytes": torch.cuda.max_memory_allocated() - base,
                     "outputs_bytes": w.B * w.V * 4 + w.B * 4 + w.B * w.D * 2,
                     "how": "torch.cuda.max_memory_allocated around one eager step"}

    if full:
        # ---- the other layouts, same step (context for the headline)
        others = {}
        for name, (f2, c2) in art.layouts.items():
            if name == layout or (name == "packed10") != w.packed10:
                continue
            if name == "rot10" and w.B > 1:   # the batch-1 layout of 10-bit codes
                continue
            st2 = make_step(f2, c2)
            r2 = rig.graphed(st2)
            n2 = min(args.steps, 3000)
            t2 = rig.time_steps(r2, n2, flush)
            k2 = rig.code_pass_us(st2, min(n2, 1000), flush)
            others[name] = {"us_per_call": t2 / n2 * 1e3,
                            "value": throughput(w.V * w.B * n2, rig.world, t2),
                            "code_pass_us": k2,
                            "code_pass_frac": code_bytes(w, name) / (k2 / 1e6) / 1e9 / peak}
        res["other_layouts"] = others
        # ---- the kernel choices of full token groups: logits and argmax of
        # one rq_logits_from_hidden_path call per step
        paths = {}
        if decoded:
            pws = torch.empty(rq.rq_fused_workspace_bytes(d, w.B, fmt, True), dtype=torch.uint8,
                              device="cuda")
            choices = [("tables", rq.PATH_TABLES), ("decode_tc", rq.PATH_DECODE_TC)]
            if layout == "u16":
                choices.insert(1, ("decode_fp32", rq.PATH_DECODE_FP32))
            for name, pth in choices:
                def pstep(pth=pth):
                    rq.rq_logits_from_hidden(dh0, dC, dcodes, fmt, d, w.softcap,
                                             logits=logits0, argmax=am0, ws=pws, path=pth)
                rp = rig.graphed(pstep)
                n3 = min(args.steps, 200)
                t3 = rig.time_steps(rp, n3)
                paths[name] = {"us_per_call": t3 / n3 * 1e3,
                               "code_pass_us": rig.code_pass_us(pstep, min(n3, 50))}
        res["full_group_paths"] = paths or None

    # ---- end to end through the public API with host buffers: every step
    # copies its hidden states in from pinned host memory and reads its logits
    # (and picks) back.  With inputs larger than L2 the copies overlap other
    # steps' compute, as a serving loop does: two input/output sets, the input
    # of step i+2 and the readback of step i run on copy streams while step i+1
    # computes.  The L2-flushed workloads serialise each step and time it alone.
    h_host = torch.from_numpy(h_np).pin_memory()
    ne2e = min(args.steps, 2000)
    outs = [(dh0, logits0, am0, rows0, tok0), (torch.empty_like(dh0),) + outputs()]
    # the compute of each set replays as a CUDA graph, as in the device timing
    # (the step object, and so its workspace, lives as long as its graph: a
    # later capture empties torch's cache and would free a dropped workspace)
    step_b = make_step(fmt, dcodes, outs[1])
    steps2 = [run, rig.graphed(step_b)]
    hosts = [(torch.empty((w.B, w.V), dtype=torch.float32).pin_memory(),
              torch.empty((w.B,), dtype=torch.int32).pin_memory()) for _ in range(2)]
    d2h_stream, h2d_stream = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("in", "done", "copied")}

    def picked_of(o):
        return o[2] if w.argmax else (o[4] if w.topk else None)

    def copy_in(k):                    # the input of a step into set k, after set k's last compute
        h2d_stream.wait_event(ev["done"][k])
        with torch.cuda.stream(h2d_stream):
            outs[k][0].copy_(h_host, non_blocking=True)
            ev["in"][k].record(h2d_stream)

    def e2e_step(i=0):
        k = i % 2 if flush is None else 0
        o = outs[k]
        pk = picked_of(o)
        if flush is not None:
            o[0].copy_(h_host, non_blocking=True)
            steps2[0]()
            hosts[0][0].copy_(o[1], non_blocking=True)
            if pk is not None:
                hosts[0][1].copy_(pk, non_blocking=True)
            return
        stream.wait_event(ev["in"][k])           # this step's input has landed
        stream.wait_event(ev["copied"][k])       # the readback of step i-2 is done
        steps2[k]()
        ev["done"][k].record(stream)
        d2h_stream.wait_event(ev["done"][k])
        with torch.cuda.stream(d2h_stream):
            hosts[k][0].copy_(o[1], non_blocking=True)
            if pk is not None:
                hosts[k][1].copy_(pk, non_blocking=True)
            ev["copied"][k].record(d2h_stream)
        copy_in(k)                               # the input of step i+2

    def e2e_run(n):
        copy_in(0)
        copy_in(1)
        for i in range(n):
            e2e_step(i)
        stream.wait_stream(d2h_stream)           # the last readback is inside the region
        stream.wait_stream(h2d_stream)

    if flush is None:
        e2e_run(4)
        torch.cuda.synchronize()
        rig.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(ne2e)
        e1.record(stream)
        torch.cuda.synchronize()
        rig.barrier()
        e_ms = rig.max_over_ranks(e0.elapsed_time(e1))
    else:
        for i in range(3):
            e2e_step(i)
        e_ms = rig.time_steps(e2e_step, ne2e)
    picked = picked_of(outs[0])
    res["e2e"] = {"value": throughput(w.V * w.B * ne2e, rig.world, e_ms), "unit": UNIT,
                  "h2d_bytes_per_step": h_np.nbytes,
                  "d2h_bytes_per_step": w.B * w.V * 4 + (w.B * 4 if picked is not None else 0),
                  "ms_per_step": e_ms / ne2e}
    # the last step's host copy equals its device result
    last = (ne2e - 1) % 2 if flush is None else 0
    assert torch.equal(hosts[last][0], outs[last][1].cpu()), "logits readback mismatch"
    # the argmax must agree with the logits it came from
    if w.argmax:
        assert torch.equal(am0.long().cpu(), logits0.argmax(dim=1).cpu()), \
            "argmax/logits mismatch"
    assert rq.rq_device_error() == 0

    res["launches_per_step"] = launches_per_step(w, decoded)
    if w.topk:
        # the epilogue alone, on the step's own logits
        for _ in range(10):
            rq.rq_topk_sample(logits0, w.topk, w.temperature, 1234, 0, token=tok0,
                              want_topk=False, ws=tws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(200):
            rq.rq_topk_sample(logits0, w.topk, w.temperature, 1234, 0, token=tok0,
                              want_topk=False, ws=tws)
        e1.record(stream)
        torch.cuda.synchronize()
        res["topk_sample_us"] = e0.elapsed_time(e1) / 200 * 1e3
    rig.graphs.clear()
    return res


def measure_decode(rig, w, art, ids_np, clk=None):
    """Rebuild the bf16 input rows of a step's ids (decode512): each call
    timed alone by its own events, with the L2 written over in between; a
    burst of calls for the warm figure; end to end with the ids copied in and
    the rows read back."""
    torch, args = rig.torch, rig.args
    import lut_logits_serving_b200 as rq
    d, C = art.d, art.C
    codes = art.layouts["u16"][1]
    stream = rig.stream
    ids = torch.from_numpy(ids_np).cuda()
    rows = torch.empty((len(ids_np), w.D), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")

    def step():
        rq.rq_decode_rows(ids, codes, rq.U16, C, d, w.decode_scale, out=rows)

    def timed(fn, n, cold):
        rig.barrier()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n if cold else 1)]
        if cold:
            for a0, a1 in evs:
                flush.fill_(1)
                a0.record(stream)
                fn()
                a1.record(stream)
        else:
            evs[0][0].record(stream)
            for _ in range(n):
                fn()
            evs[0][1].record(stream)
        torch.cuda.synchronize()
        rig.barrier()
        return rig.max_over_ranks(sum(a0.elapsed_time(a1) for a0, a1 in evs))

    def graphed(calls):
        """`calls` back-to-back decode calls as one CUDA graph (a call is a
        few microseconds, shorter than a Python launch)."""
        s2 = torch.cuda.Stream()
        s2.wait_stream(stream)
        with torch.cuda.stream(s2):
            step()
        stream.wait_stream(s2)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(calls):
                step()
        g.replay()
        torch.cuda.synchronize()
        return g

    for _ in range(max(3, args.warmup)):
        step()
    burst = 20
    g1, gb = (None, None) if args.no_graph else (graphed(1), graphed(burst))
    if clk is not None:
        clk.wait_first()
        clk.window()
    t_ms = timed(step if g1 is None else g1.replay, args.steps, True)
    if clk is not None:
        clk.close_window()
    if gb is None:
        warm_ms = timed(step, args.steps, False)
    else:
        reps = max(1, args.steps // burst)
        warm_ms = timed(gb.replay, reps, False) * args.steps / (reps * burst)
    n_ids = len(ids_np)
    want = None
    if rig.rank == 0:
        import oracle
        want = oracle.decode_rows_bf16(ids_np, art.codes_np, art.C_np, w.decode_scale)
        assert np.array_equal(rows.view(torch.int16).cpu().numpy().view(np.uint16), want)
    assert rq.rq_device_error() == 0
    peak, peak_kind = load_peaks()
    kern_s = t_ms / args.steps / 1e3
    nbytes = decode_bytes(w)
    achieved = nbytes / kern_s / 1e9

    # end to end: ids in from pinned host memory, rows back to the host
    idh = torch.from_numpy(ids_np).pin_memory()
    rh = torch.empty((n_ids, w.D), dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        ids.copy_(idh, non_blocking=True)
        step() if g1 is None else g1.replay()
        rh.copy_(rows, non_blocking=True)

    e2e_step()
    e_ms = timed(e2e_step, args.steps, True)
    del g1, gb
    return {
        "metric": DEC_METRIC, "unit": DEC_UNIT, "steps": args.steps,
        "value": throughput(n_ids * args.steps, rig.world, t_ms),
        "us_per_call": t_ms / args.steps * 1e3, "us_per_call_warm": warm_ms / args.steps * 1e3,
        "ms_per_step": t_ms / args.steps,
        "launch": "eager" if args.no_graph else "cuda graph",
        "roofline": {"bound": "hbm", "kernel": "decode_rows_pair_kernel", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": profiled_traffic("decode_rows_pair_kernel/u16/decode512"),
                     "algorithmic_bytes": nbytes, "kernel_us": kern_s * 1e6},
        "e2e": {"value": throughput(n_ids * args.steps, rig.world, e_ms), "unit": DEC_UNIT,
                "h2d_bytes_per_step": n_ids * 4, "d2h_bytes_per_step": n_ids * w.D * 2,
                "ms_per_step": e_ms / args.steps},
        "memory": {"resident_bytes": art.bytes("u16"), "workspace_bytes": 0,
                   "outputs_bytes": n_ids * w.D * 2},
    }


# The default run measures the headline (decode batch 1) and, on the same
# resident artifact, the batched, packed and row-decode configurations.
EXTRA_WORKLOADS = ("g2_b32", "packed_b64", "decode512")


def run_ours(args, w):
    rig = Rig(args)
    torch = rig.torch
    data = synth.make(w, seed=rank_seed(rig.rank))
    extras = (not args.no_extras and w.name == "g2_b1" and not args.codes)
    need = ("sched", "u16", "u8", "packed10", "rot10") if extras else \
        ("sched", "u16", "u8", "packed10") if w.packed10 else ("sched", "u16", "u8") + \
        (("rot10",) if args.codes == "rot10" else ())
    art = Artifact(w, data, need)
    art.codes_np, art.C_np = data["codes"], data["C"]
    headline = headline_layout(w, args.codes, tuple(k for k in art.layouts if k != "packed10"))

    with ClockSampler(rig.local) as clk:
        res = measure_logits(rig, w, art, headline, data["h"], full=True, clk=clk)
    clocks = clk.summary()
    res["sustained"]["clocks"] = clocks
    if clocks.get("sm_mhz") and res["sustained"]["us_per_step"]:
        res["sustained"]["us_x_mhz"] = res["sustained"]["us_per_step"] * clocks["sm_mhz"]

    others = {}
    if extras:
        # the packed 10-bit layout at batch 1 (the pages' 3.59 bits/param form)
        p1 = measure_logits(rig, w, art, "packed10", data["h"])
        p1.pop("t_ms", None)
        others["g2_b1_packed10"] = dict(p1, config=workload_config(w, "packed10"))
        if "rot10" in art.layouts:
            # the same 10-bit codes in rotated slices (rq_prepare_rot10)
            r1 = measure_logits(rig, w, art, "rot10", data["h"])
            r1.pop("t_ms", None)
            r1["roofline"]["bank_passes_per_step"] = art.rot_passes
            others["g2_b1_rot10"] = dict(r1, config=workload_config(w, "rot10"))
        for name in EXTRA_WORKLOADS:
            w2 = synth.WORKLOADS[name]
            seed = rank_seed(rig.rank)
            with ClockSampler(rig.local) as c2:
                if w2.B == 0:
                    ids = synth.zipf_ids(w2.n_ids, w2.V, w2.zipf_s, seed + 3)
                    r2 = measure_decode(rig, w2, art, ids, clk=c2)
                    r2["config"] = decode_config(w2)
                else:
                    h2 = synth.hidden(w2.B, w2.D, w2.hidden_scale, seed + 2)
                    lay = headline_layout(w2, None, tuple(art.layouts))
                    # the 32-token batch also on the other layouts (the batch-1
                    # layout through the tensor cores) and every group kernel
                    r2 = measure_logits(rig, w2, art, lay, h2, full=name == "g2_b32")
                    r2["config"] = workload_config(w2, lay)
                    r2.pop("t_ms", None)
            r2["clocks"] = c2.summary()
            others[name] = r2

    cpu = None
    if rig.rank == 0 and rig.world == 1 and not args.no_cpu_baseline and (w.argmax or w.topk):
        cpu = cpu_baseline(w, data, args.cpu_seconds, threads=0)
        cpu["single_thread"] = cpu_baseline(w, data, args.cpu_seconds / 2, threads=1)
    rig.close()
    if rig.rank != 0:
        return
    t_ms = res["t_ms"]
    roof = dict(res["roofline"])
    if art.sched_passes is not None and headline == "sched":
        roof["bank_passes_per_step"] = art.sched_passes
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": rig.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms / args.steps,
        "us_per_call": res["us_per_call"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(w, headline), parallelism=parallelism()),
        "launch": "eager" if args.no_graph else "cuda graph",
        "roofline": roof,
        "step_hbm_frac": res["step_hbm_frac"],
        "pipes": res.get("pipes"),
        "memory": res["memory"],
        "other_layouts": res.get("other_layouts"),
        "full_group_paths": res.get("full_group_paths"),
        "topk_sample_us": res.get("topk_sample_us"),
        "other_workloads": others or None,
        "cpu_baseline": cpu,
        "e2e": res["e2e"],
        "gpu_launches": res["launches_per_step"] * args.steps,
        "clocks": dict(clocks, window=f"the {args.steps} timed steps and "
                                      f"{res['sustained']['steps']} more replays of the same "
                                      f"step right after them"),
        "sustained": res["sustained"],
    }
    print(json.dumps(line), flush=True)


def run_encode(args, w):
    """Encode all V rows per step (rows resident on the device)."""
    import torch
    import torch.distributed as dist

    import lut_logits_serving_b200 as rq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    data = synth.make(w, seed=rank_seed(rank))
    d = rq.dims(w.V, w.D, w.M, w.L, w.K)
    X = torch.from_numpy(data["X"]).cuda()
    C = torch.from_numpy(data["C"]).cuda()
    codes = torch.empty((w.V, w.P), dtype=torch.uint16, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        rq.rq_encode(X, C, d, out=codes)

    def timed(fn, n):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return aggregate(e0.elapsed_time(e1), world, device="cuda")

    for _ in range(args.warmup):
        step()
    with ClockSampler(local) as clk:
        t_ms = timed(step, args.steps)
    value = throughput(w.V * args.steps, world, t_ms)
    clocks = clk.summary()
    kern_s = t_ms / args.steps / 1e3                  # one launch per step
    ops = 2 * encode_terms(w, w.V)
    mhz = clocks["sm_max_mhz"] or NOMINAL_SM_MHZ
    peak = SMS * FP32_LANES * mhz * 1e6 / 1e12
    achieved = ops / kern_s / 1e12
    assert rq.rq_device_error() == 0

    # end to end: rows from pinned host memory, codes back to the host
    Xh = torch.from_numpy(data["X"]).pin_memory()
    ch = torch.empty((w.V, w.P), dtype=torch.uint16).pin_memory()

    def e2e_step():
        X.copy_(Xh, non_blocking=True)
        step()
        ch.copy_(codes, non_blocking=True)

    e2e_step()
    ne2e = 3
    e_ms = timed(e2e_step, ne2e)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.set_threads(0)
        n, t0, sample = 0, time.perf_counter(), 64 * threads
        while time.perf_counter() - t0 < args.cpu_seconds:
            oracle.encode(data["X"][:sample], data["C"])
            n += sample
        el = time.perf_counter() - t0
        cpu = dict({"value": n / el, "unit": ENC_UNIT, "cores": threads, "kind": "oracle",
                    "sample": f"{n} rows ({sample} per call) encoded by the C oracle, "
                              f"{threads} OpenMP thread(s) over rows, {el:.1f} s"}, **cpu_info())
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": ENC_METRIC, "value": value, "unit": ENC_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": dict(encode_config(w), parallelism=parallelism()),
        "launch": "eager",
        "roofline": {"bound": "alu", "kernel": "encode_pair_kernel<6,4>", "achieved": achieved,
                     "peak": peak, "peak_kind": f"derived: {SMS} SMs x {FP32_LANES} FP32 lanes "
                                                f"x {mhz:g} MHz",
                     "unit": "T fp32 lane-ops/s", "frac": achieved / peak, "traffic": None,
                     "algorithmic_ops": ops, "kernel_us": kern_s * 1e6},
        "cpu_baseline": cpu,
        "e2e": {"value": throughput(w.V * ne2e, world, e_ms), "unit": ENC_UNIT,
                "h2d_bytes_per_step": data["X"].nbytes, "d2h_bytes_per_step": w.V * w.P * 2,
                "ms_per_step": e_ms / ne2e},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_decode(args, w):
    """The row-decode workload alone (decode512)."""
    rig = Rig(args)
    data = synth.make(w, seed=rank_seed(rig.rank))
    art = Artifact(w, data, ("u16",))
    art.codes_np, art.C_np = data["codes"], data["C"]
    with ClockSampler(rig.local) as clk:
        res = measure_decode(rig, w, art, data["ids"], clk=clk)
    cpu = None
    if rig.rank == 0 and rig.world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.set_threads(0)
        n, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < min(args.cpu_seconds, 5.0):
            oracle.decode_rows_bf16(data["ids"], data["codes"], data["C"], w.decode_scale)
            n += w.n_ids
        el = time.perf_counter() - t0
        cpu = dict({"value": n / el, "unit": DEC_UNIT, "cores": threads, "kind": "oracle",
                    "sample": f"{n // w.n_ids} calls of {w.n_ids} ids, C with {threads} OpenMP "
                              f"thread(s) over ids, {el:.1f} s"}, **cpu_info())
    rig.close()
    if rig.rank != 0:
        return
    line = {
        "metric": DEC_METRIC, "value": res["value"], "unit": DEC_UNIT, "n_gpus": rig.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "us_per_call": res["us_per_call"], "us_per_call_warm": res["us_per_call_warm"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": dict(decode_config(w), parallelism=parallelism()),
        "launch": res["launch"], "roofline": res["roofline"], "memory": res["memory"],
        "cpu_baseline": cpu, "e2e": res["e2e"], "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    elif w.encode:
        run_encode(args, w)
    elif w.B == 0:
        run_decode(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
