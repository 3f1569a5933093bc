#!/usr/bin/env python
"""Throughput of the FP4 weight quantizer on a Llama-3-8B-shaped model.

Workload (one "step"): every linear weight of a synthetic Llama-3-8B-shaped
model -- 32 layers x {q, o: 4096x4096; k, v: 1024x4096; gate, up: 14336x4096;
down: 4096x14336}, 224 bf16 tensors, 6.98e9 elements, Student-t(4) * 0.02 --
is quantized to MXFP4 (E8M0 exponent sweep; the same pass reduces max|w|) and
to NVFP4 (the ScaleSweep MSE window search on that global scale); both emit
packed codes, scales and the bf16 reconstruction.  Inputs (13.96 GB) are resident in HBM and larger than L2, so
no L2 flush is needed between steps.  The step is captured once as a CUDA graph
and replayed.

Metric: weight GB/s of bf16 input quantized (2 bytes x elements / time), whole
job over all ranks; also elements/s and the fraction of the HBM roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun each rank quantizes its own copy of the model (seeded by rank):
weak scaling, no collective on the data path; ranks synchronise only around
the timed region and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np
import torch

METRIC = "weight GB/s (bf16 in) quantized to NVFP4/MXFP4 at 1 B200; % of HBM roofline"
WORKLOAD = "llama3-8b-shaped whole-model pass: 224 bf16 linear weights -> NVFP4-MSE + MXFP4"
# algorithmic bytes per element (bf16 in): absmax read 2; NVFP4 sweep read 2 + codes 0.5 +
# scales 1/16 + bf16 deq 2; MXFP4 read 2 + codes 0.5 + scales 1/32 + bf16 deq 2.  The step
# reads W twice (MXFP4 with the fused absmax, then the NVFP4 sweep).
B_ABSMAX = 2.0
B_NVFP4 = 2.0 + 0.5 + 1.0 / 16 + 2.0
B_MXFP4 = 2.0 + 0.5 + 1.0 / 32 + 2.0
SM_FP32_LANES = 128


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", 6650.0)), "measured", float(d.get("sm_max_mhz", 1965.0))
    return 6650.0, "fallback", 1965.0


HBM_SPEC_GBS = 8000.0     # B200 HBM3e bandwidth as specified (context only)


def tensor_sha256(t) -> str:
    """SHA-256 of a tensor's (or array's) raw bytes in memory order, any dtype,
    on any device (the bytes are copied to the host first)."""
    import hashlib
    if isinstance(t, torch.Tensor):
        t = t.detach().contiguous().reshape(-1).view(torch.uint8).cpu().numpy()
    return hashlib.sha256(memoryview(np.ascontiguousarray(t)).cast("B")).hexdigest()


def l2_flush_buffer(dev):
    """A buffer at least twice the device's L2 (and at least 512 MB): rewriting it
    between timed launches leaves none of their inputs in L2."""
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or 0)
    return torch.empty(max(512 << 20, 2 * l2), dtype=torch.uint8, device=dev)


def copy_probe_gbs(fq, dev, nbytes=512 << 20, reps=10):
    """Copy bandwidth of the library's own 16-byte streaming loads and stores
    (`fp4q_probe_copy`, nbytes read + nbytes written, source larger than L2):
    median of `reps` launches after 3 warm-up launches, CUDA events on the
    launching stream."""
    src = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    src.fill_(1)
    stream = torch.cuda.current_stream(dev)
    times = []
    for i in range(3 + reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fq.fp4q_probe_copy(src, dst, stream)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            times.append(a.elapsed_time(b))
    del src, dst
    return 2.0 * nbytes / (statistics.median(times) * 1e-3) / 1e9


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="fp4q_clocks_", suffix=".csv")
        os.close(fd)

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception as e:     # no nvidia-smi: report that instead of clocks
            log("clock sampling unavailable:", e)
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- workload

def group_bounds(n, size, layer_sizes=None):
    """[lo, hi) index ranges of the grouped launches over n weights: consecutive
    groups of `size`, or each layer's weights (sum(layer_sizes) of them) split
    into consecutive groups of layer_sizes.  Every weight is in exactly one
    range, in order."""
    if layer_sizes:
        if min(layer_sizes) < 1:
            raise ValueError("group sizes must be positive")
        per_layer = sum(layer_sizes)
        bounds = []
        for base in range(0, n, per_layer):
            for k in layer_sizes:
                if base < n:
                    bounds.append((base, min(base + k, n)))
                base += k
        return bounds
    if size < 1:
        raise ValueError("group size must be positive")
    return [(b, min(b + size, n)) for b in range(0, n, size)]


class Model:
    """Device buffers of the whole-model pass and the launch sequence of one step."""

    def __init__(self, fq, dev, seed: int, with_events: bool):
        import synth
        self.fq = fq
        self.dev = dev
        self.shapes = synth.llama3_8b_shapes()
        self.w, self.out = [], []
        t0 = time.time()
        for i, (name, r, c) in enumerate(self.shapes):
            self.w.append(synth.llama3_8b_tensor(i, r, c, seed=seed, device=dev))
            kw = dict(device=dev)
            self.out.append(dict(
                amax=torch.empty(1, dtype=torch.float32, **kw),
                S=torch.empty(1, dtype=torch.float32, **kw),
                nv_codes=torch.empty((r, c // 2), dtype=torch.uint8, **kw),
                nv_scales=torch.empty((r, c // 16), dtype=torch.uint8, **kw),
                nv_deq=torch.empty((r, c), dtype=torch.bfloat16, **kw),
                mx_codes=torch.empty((r, c // 2), dtype=torch.uint8, **kw),
                mx_scales=torch.empty((r, c // 32), dtype=torch.uint8, **kw),
                mx_deq=torch.empty((r, c), dtype=torch.bfloat16, **kw),
            ))
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        torch.cuda.synchronize()
        log(f"generated {len(self.w)} tensors in {time.time() - t0:.1f}s")
        self.elements = sum(r * c for _, r, c in self.shapes)
        self.events = None
        if with_events:
            self.events = [(torch.cuda.Event(enable_timing=True, external=True),
                            torch.cuda.Event(enable_timing=True, external=True)) for _ in self.shapes]
        self.launches_per_step = 2 * len(self.shapes)
        self.ready = [torch.cuda.Event() for _ in self.shapes]
        self.done = [torch.cuda.Event() for _ in self.shapes]

    def batch_setup(self, chunk):
        """Descriptors of every weight for fp4q_quantize_batch, split into launches of at
        most `chunk` weights (one workspace each) with events around each launch."""
        fq = self.fq
        self.chunks = []
        for base in range(0, len(self.w), chunk):
            items = []
            for w, o in zip(self.w[base:base + chunk], self.out[base:base + chunk]):
                items.append(dict(w=w, amax=o["amax"], global_scale=o["S"], nv_codes=o["nv_codes"],
                                  nv_scales=o["nv_scales"], nv_deq=o["nv_deq"], mx_codes=o["mx_codes"],
                                  mx_scales=o["mx_scales"], mx_deq=o["mx_deq"]))
            ws = torch.empty(fq.fp4q_batch_workspace_bytes(), dtype=torch.uint8, device=self.dev)
            n = sum(it["w"].numel() for it in items)
            ev = (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
            self.chunks.append((items, ws, n, ev))
        self.launches_per_step = len(self.chunks)

    def group_setup(self, size, layer_sizes=None):
        """Descriptors for the grouped calls, one MXFP4 and one NVFP4 launch per group:
        consecutive weights in groups of `size` (7 = one layer), or each layer's seven
        weights split into consecutive groups of `layer_sizes` (summing to 7)."""
        self.groups = []
        for lo, hi in group_bounds(len(self.w), size, layer_sizes):
            idx = range(lo, hi)
            mx = [dict(w=self.w[i], amax=self.out[i]["amax"], mx_codes=self.out[i]["mx_codes"],
                       mx_scales=self.out[i]["mx_scales"], mx_deq=self.out[i]["mx_deq"]) for i in idx]
            nv = [dict(w=self.w[i], amax=self.out[i]["amax"], global_scale=self.out[i]["S"],
                       nv_codes=self.out[i]["nv_codes"], nv_scales=self.out[i]["nv_scales"],
                       nv_deq=self.out[i]["nv_deq"]) for i in idx]
            ev = (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
            self.groups.append((mx, nv, torch.cuda.Event(), ev))
        self.group_done = [torch.cuda.Event() for _ in self.groups]
        self.launches_per_step = 2 * len(self.groups)

    def step_groups(self, stream, stream2, lag=0):
        """Per group: one MXFP4 launch (with each weight's max) on `stream`, then one
        NVFP4 launch on `stream2` after it, overlapping the next group's MXFP4 launch;
        with lag > 0 the MXFP4 launch of group g also waits for the NVFP4 launch of
        group g - lag."""
        fq = self.fq
        stream2.wait_stream(stream)
        for g, (mx, nv, ready, ev) in enumerate(self.groups):
            if lag > 0 and g >= lag:
                stream.wait_event(self.group_done[g - lag])
            fq.fp4q_mxfp4_quant_group(mx, self.status, stream)
            ready.record(stream)
            stream2.wait_event(ready)
            ev[0].record(stream2)
            fq.fp4q_nvfp4_sweep_group(nv, self.status, stream2)
            ev[1].record(stream2)
            self.group_done[g].record(stream2)
        stream.wait_stream(stream2)

    def step_batch(self, stream):
        """The whole model in one persistent launch per chunk of weights."""
        for items, ws, _, ev in self.chunks:
            ev[0].record(stream)
            self.fq.fp4q_quantize_batch(items, ws, self.status, stream)
            ev[1].record(stream)

    def step_schedule(self, streams, lag):
        """MXFP4 passes on streams[0]; NVFP4 sweeps round-robin on streams[1:], each
        after its own tensor's MXFP4 pass; with lag > 0 the MXFP4 pass of tensor t
        also waits for the sweep of tensor t - lag to finish (keeps the two kinds of
        kernels interleaved instead of letting the MXFP4 passes run ahead)."""
        fq = self.fq
        s0 = streams[0]
        for s in streams[1:]:
            s.wait_stream(s0)
        for i, (w, o) in enumerate(zip(self.w, self.out)):
            if lag > 0 and i >= lag:
                s0.wait_event(self.done[i - lag])
            fq.fp4q_mxfp4_quant_absmax(w, None, o["mx_codes"], o["mx_scales"], o["amax"], o["mx_deq"],
                                       None, self.status, s0)
            self.ready[i].record(s0)
            s2 = streams[1 + i % (len(streams) - 1)]
            s2.wait_event(self.ready[i])
            if self.events is not None:
                self.events[i][0].record(s2)
            fq.fp4q_nvfp4_sweepmse(w, o["amax"], o["nv_codes"], o["nv_scales"], o["S"], o["nv_deq"],
                                   None, self.status, s2)
            if self.events is not None:
                self.events[i][1].record(s2)
            self.done[i].record(s2)
        for s in streams[1:]:
            s0.wait_stream(s)

    def step(self, stream, stream2=None):
        """Per tensor: MXFP4 (which also reduces max|w|), then the NVFP4 ScaleSweep on
        that max -- the two launches of fp4q_quantize_dual, issued as its two C calls
        so that events can bracket the NVFP4 sweep.  With `stream2` the sweeps run on
        a second stream, each after its own tensor's MXFP4 pass, so that the sweep of
        one tensor overlaps the MXFP4 pass of the next."""
        fq = self.fq
        s2 = stream if stream2 is None else stream2
        if stream2 is not None:
            stream2.wait_stream(stream)
        for i, (w, o) in enumerate(zip(self.w, self.out)):
            fq.fp4q_mxfp4_quant_absmax(w, None, o["mx_codes"], o["mx_scales"], o["amax"], o["mx_deq"],
                                       None, self.status, stream)
            if stream2 is not None:
                self.ready[i].record(stream)
                stream2.wait_event(self.ready[i])
            if self.events is not None:
                self.events[i][0].record(s2)
            fq.fp4q_nvfp4_sweepmse(w, o["amax"], o["nv_codes"], o["nv_scales"], o["S"], o["nv_deq"],
                                   None, self.status, s2)
            if self.events is not None:
                self.events[i][1].record(s2)
        if stream2 is not None:
            stream.wait_stream(stream2)

    def sweep_ms(self):
        return [a.elapsed_time(b) for a, b in self.events]


PARITY_TENSORS = (0, 1, 2, 3, 4, 5, 6, 217, 218, 219, 220, 221, 222, 223)   # layers 0 and 31, all 7 shapes


def step_parity(model, tensors=PARITY_TENSORS, rows_per_tensor=2):
    """Outputs of the last timed step against the oracle, element by element, on
    sampled rows of sampled tensors (outside the timed region): per tensor the
    oracle's own global max over the whole weight gives S, which must equal the
    S the sweep wrote; on rows 0 and rows-1 the NVFP4 codes, scales and bf16
    reconstruction and the MXFP4 codes, scales and reconstruction must be
    identical.  A schedule that let a sweep read its weight's maximum before
    the MXFP4 pass had finished reducing it would show here."""
    import oracle
    oracle.build()
    bad = []
    checked = 0
    for t in tensors:
        if t >= len(model.w):
            continue
        w, o = model.w[t], model.out[t]
        x_all = w.float().cpu().numpy()
        rows = x_all.shape[0]
        idx = np.array(sorted({0, rows - 1})[:rows_per_tensor])
        x = np.ascontiguousarray(x_all[idx])
        S_o = oracle.global_scale(oracle.global_absmax(x_all))
        del x_all
        nv = oracle.nvfp4_quant(x, S=S_o)
        mx = oracle.mxfp4_quant(x)

        def u16(tt):
            return tt.detach().cpu().view(torch.int16).numpy().view(np.uint16)[idx]
        ok = (np.float32(o["S"].item()) == np.float32(S_o)
              and np.array_equal(o["nv_codes"].cpu().numpy()[idx], nv["codes"])
              and np.array_equal(o["nv_scales"].cpu().numpy()[idx], nv["scales"])
              and np.array_equal(u16(o["nv_deq"]), oracle.bf16_round(nv["y"]))
              and np.array_equal(o["mx_codes"].cpu().numpy()[idx], mx["codes"])
              and np.array_equal(o["mx_scales"].cpu().numpy()[idx], mx["scales"])
              and np.array_equal(u16(o["mx_deq"]), oracle.bf16_round(mx["y"])))
        checked += 1
        if not ok:
            bad.append(model.shapes[t][0])
    return {"ok": not bad and checked > 0, "tensors_checked": checked, "rows_per_tensor": rows_per_tensor,
            "mismatching": bad,
            "what": "last timed step: S, NVFP4 codes/scales/bf16 reconstruction, MXFP4 codes/scales/bf16 "
                    "reconstruction on rows 0 and rows-1 of layers 0 and 31, bit for bit against the oracle"}


def e2e_run(fq, model, steps, dev):
    """Same step through the public API with host buffers: every step copies each bf16
    weight from pinned host memory to the device, quantizes it, and copies the packed
    result (NVFP4 codes + scales + S, MXFP4 codes + scales) back to pinned host memory.
    Copies run on a copy stream and overlap the quantization of other tensors."""
    host_w = [w.cpu().pin_memory() for w in model.w]
    host_out = [dict(nv_codes=torch.empty_like(o["nv_codes"], device="cpu").pin_memory(),
                     nv_scales=torch.empty_like(o["nv_scales"], device="cpu").pin_memory(),
                     S=torch.empty(1, dtype=torch.float32).pin_memory(),
                     mx_codes=torch.empty_like(o["mx_codes"], device="cpu").pin_memory(),
                     mx_scales=torch.empty_like(o["mx_scales"], device="cpu").pin_memory())
                for o in model.out]
    h2d_bytes = sum(w.numel() * 2 for w in host_w)
    d2h_bytes = sum(sum(t.numel() * t.element_size() for t in h.values()) for h in host_out)
    compute = torch.cuda.Stream(device=dev)
    h2d = torch.cuda.Stream(device=dev)
    d2h = torch.cuda.Stream(device=dev)

    def one_step():
        for i, (hw, o, ho) in enumerate(zip(host_w, model.out, host_out)):
            with torch.cuda.stream(h2d):
                model.w[i].copy_(hw, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(h2d)
            compute.wait_event(ready)
            fq.fp4q_quantize_dual(model.w[i], None, None, o["amax"], o["nv_codes"], o["nv_scales"], o["S"],
                                  o["nv_deq"], None, o["mx_codes"], o["mx_scales"], o["mx_deq"], None,
                                  model.status, compute)
            done = torch.cuda.Event()
            done.record(compute)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                for k in ho:
                    ho[k].copy_(o[k], non_blocking=True)
        torch.cuda.synchronize()

    one_step()   # warm-up (also pages in the pinned buffers)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(steps):
        one_step()
    dt = (time.perf_counter() - t0) / steps
    del host_w, host_out
    return dt, h2d_bytes, d2h_bytes


# --------------------------------------------------------------------------- CPU baseline

CPU_SAMPLE_ROWS = 256          # rows per tensor of the calibration sample and the reference arm's step


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_pass(rows, threads=0):
    """The oracle on the first `rows` rows (at most each tensor's own) of each of
    the 7 tensor shapes of one layer: absmax + NVFP4-MSE sweep, and MXFP4, on
    `threads` OpenMP threads (0: all cores).  Returns (elements, seconds); the
    inputs are made before the clock starts."""
    import oracle
    import synth
    shapes = synth.llama3_8b_shapes()[:7]
    xs = [synth.llama3_8b_tensor(i, min(rows, r), c, seed=7).float().numpy()
          for i, (_, r, c) in enumerate(shapes)]
    n = sum(x.size for x in xs)
    t0 = time.perf_counter()
    for x in xs:
        g = oracle.global_absmax(x)
        oracle.nvfp4_quant(x, S=oracle.global_scale(g), threads=threads)
        oracle.mxfp4_quant(x, threads=threads)
    return n, time.perf_counter() - t0


def cpu_baseline(target_s=12.0):
    """The oracle, as it stands, on a bounded sample of the workload, all host
    cores (OpenMP): a calibration pass on the first 256 rows of each of the 7
    tensor shapes of one layer sets the row count of the timed pass so that it
    takes about `target_s` seconds (never more rows than a tensor has)."""
    import oracle
    import synth
    oracle.build()
    n, dt = _oracle_pass(CPU_SAMPLE_ROWS)
    rows = CPU_SAMPLE_ROWS
    want = n * target_s / max(dt, 1e-3)               # elements for about target_s seconds
    shapes = synth.llama3_8b_shapes()[:7]
    full = max(r for _, r, _ in shapes)
    grow = rows
    while grow < full and sum(min(grow, r) * c for _, r, c in shapes) < want:
        grow += 64
    if grow > rows:
        rows = grow
        n, dt = _oracle_pass(rows)
    n1, dt1 = _oracle_pass(64, threads=1)
    return {"value": 2.0 * n / dt / 1e9, "unit": "GB/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"first {rows} rows (at most each tensor's own) of each of the 7 tensor shapes of one "
                      f"layer ({n} elements): absmax + NVFP4-MSE sweep + MXFP4, {dt:.2f}s",
            "elements_per_s": n / dt, "cpu_model": _cpu_model(),
            "single_thread": {"value": 2.0 * n1 / dt1 / 1e9, "unit": "GB/s", "elements_per_s": n1 / dt1,
                              "sample": f"first 64 rows of each of the 7 tensor shapes ({n1} elements), "
                                        f"1 thread, {dt1:.2f}s"}}


def rank_seed(rank: int) -> int:
    """Seed of the replica on `rank`: every rank quantizes its own synthetic
    copy of the workload (weak scaling), drawn from seed 5 + 1000 * rank."""
    return 5 + 1000 * rank


def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time: an all-reduce (MAX) over the process group, or
    `ms` itself without one."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args):
    """--impl reference: the CPU oracle timed on the host cores, per step one bounded
    sample of the workload (see cpu_baseline)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import synth
    oracle.build()
    rows = CPU_SAMPLE_ROWS
    shapes = synth.llama3_8b_shapes()[:7]
    xs = [synth.llama3_8b_tensor(i, rows, c, seed=7).float().numpy() for i, (_, _, c) in enumerate(shapes)]
    n = sum(x.size for x in xs)

    def step():
        for x in xs:
            oracle.nvfp4_quant(x, S=oracle.global_scale(oracle.global_absmax(x)))
            oracle.mxfp4_quant(x)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = 2.0 * n / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample_rows_per_tensor": rows,
                                            "elements_per_step": n},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.max_threads(),
                             "kind": "oracle", "sample": f"first {rows} rows of the 7 tensor shapes of one layer"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- measured counters
# ncu counters of one nvfp4_sweep_kernel (MSE, bf16) launch on a 16384 x 8192
# weight, per element, with the sources they were taken on
# (profiles/nvfp4_sweep_mse_16384x8192.md): DRAM bytes (dram__bytes_read.sum +
# dram__bytes_write.sum), executed warp instructions (smsp__inst_executed.sum)
# and the issue-active fraction.  Traffic grows in proportion to the elements,
# so a launch of n elements moves about n times the per-element figure.  Once
# the sources differ the figures no longer describe the kernel and none is
# reported.
NVFP4_PROFILE = {"bytes_per_element": (268524544 + 287375616) / (16384 * 8192),
                 "warp_inst_per_element": 220760623 / (16384 * 8192),
                 "issue_active_pct": 78.18,
                 "kernel": "nvfp4_group_kernel (MSE, bf16), one 16384x8192 weight",
                 "sources": ("nvfp4.cu", "nvfp4_block.cuh", "screen.cuh", "device.cuh"),
                 "sha256": "06fb432f7bd8acf96936c9b18bb88a2aadbe58d1ec144ea4acf4c55f63a514f7"}


def nvfp4_profile_current():
    """NVFP4_PROFILE if the kernel's sources still hash to the profiled ones, else None."""
    import hashlib
    h = hashlib.sha256()
    for f in NVFP4_PROFILE["sources"]:
        with open(os.path.join(ROOT, "fp4_post_weight_grid_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return NVFP4_PROFILE if h.hexdigest() == NVFP4_PROFILE["sha256"] else None


def measured_traffic_per_launch(elements_per_launch):
    prof = nvfp4_profile_current()
    return None if prof is None else prof["bytes_per_element"] * elements_per_launch


# --------------------------------------------------------------------------- single-kernel mode

SINGLE_PATHS = {
    # name: (bytes per element, kernel description)
    "absmax": (B_ABSMAX, "absmax_kernel"),
    "nvfp4-mse": (B_NVFP4, "nvfp4_sweep_kernel MSE"),
    "nvfp4-wmse": (B_NVFP4, "nvfp4_sweep_kernel WMSE"),
    "mxfp4": (B_MXFP4, "mxfp4_kernel"),
    "mxfp4-absmax": (B_MXFP4, "mxfp4_kernel with the fused global max"),
    "mxfp4-hadamard": (B_MXFP4, "mxfp4_rot_pf_kernel (Hadamard, next block loaded during the current one)"),
    "nvfp4-mse-group": (B_NVFP4, "nvfp4_group_kernel MSE (fp4q_nvfp4_sweep_group, one weight)"),
    "mxfp4-absmax-group": (B_MXFP4, "mxfp4_group_kernel (fp4q_mxfp4_quant_group, one weight)"),
    "dequant-nvfp4": (0.5 + 1.0 / 16 + 2.0, "dequant_kernel NVFP4"),
    "mma-layout": (2.0 / 16, "mma_scale_layout_kernel (NVFP4 scales, read + write)"),
    "focus-nvfp4": (2.0 + 1.0 / 16 + 2.0 / 8 + 0.5 + 2.0, "focus_kernel NVFP4, sub-blocks of 8"),
    "focus-mxfp4": (2.0 + 1.0 / 32 + 2.0 / 8 + 0.5 + 2.0, "focus_kernel MXFP4, sub-blocks of 8"),
    "unrotate": (4.0, "unrotate_kernel (MXFP4 Hadamard inverse, bf16 in and out)"),
    "copy": (4.0, "probe_copy_kernel (the library's 16-byte streaming loads and stores, bf16 in and out)"),
}


def run_single(args):
    """Time one kernel on one synthetic bf16 weight (`--shape RxC`), `--steps` launches
    after `--warmup`, each launch timed with CUDA events on its stream; between
    launches a buffer of twice the L2 (at least 512 MB) is rewritten so that no launch
    starts with its input in L2.
    Prints one JSON line (not the benchmark line)."""
    import fp4_post_weight_grid_b200 as fq
    from fp4_post_weight_grid_b200 import build as fbuild
    import synth
    fbuild.build()
    rows, cols = (int(v) for v in args.shape.lower().split("x"))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = synth.t_weight(rows, cols, nu=4, scale=0.02, seed=11, device=dev)
    imp = synth.importance_diag_xtx(cols=cols, tokens=256, seed=11, device=dev)
    masks = torch.from_numpy(synth.sign_masks(cols, seed=11).view(np.int32)).to(dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    S = torch.empty(1, dtype=torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    sc16 = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    sc32 = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)
    deq = torch.empty_like(w)
    tiled = torch.empty(fq.fp4q_mma_scale_bytes(rows, cols // 16), dtype=torch.uint8, device=dev)
    coeffs = (1.0 + 0.25 * torch.rand((rows, cols // 8), device=dev)).to(torch.float16)
    flush = l2_flush_buffer(dev)
    fq.fp4q_global_absmax(w, amax)
    fq.fp4q_nvfp4_sweepmse(w, amax, codes, sc16, S, deq, None, st)
    fq.fp4q_mxfp4_quant(w, codes, sc32, None, None, st)
    stream = torch.cuda.current_stream()

    def launch():
        if args.single == "absmax":
            fq.fp4q_global_absmax(w, amax, stream=stream)
        elif args.single == "nvfp4-mse":
            fq.fp4q_nvfp4_sweepmse(w, amax, codes, sc16, S, deq, None, st, stream)
        elif args.single == "nvfp4-wmse":
            fq.fp4q_nvfp4_sweepwmse(w, amax, imp, codes, sc16, S, deq, None, st, stream)
        elif args.single == "mxfp4":
            fq.fp4q_mxfp4_quant(w, codes, sc32, deq, None, st, stream)
        elif args.single == "mxfp4-absmax":
            fq.fp4q_mxfp4_quant_absmax(w, None, codes, sc32, amax, deq, None, st, stream)
        elif args.single == "mxfp4-hadamard":
            fq.fp4q_mxfp4_quant_hadamard(w, masks, codes, sc32, deq, None, st, stream)
        elif args.single == "focus-nvfp4":
            fq.fp4q_focus_quant(fq.NVFP4, w, sc16, S, coeffs, 8, codes, deq, None, st, stream)
        elif args.single == "focus-mxfp4":
            fq.fp4q_focus_quant(fq.MXFP4, w, sc32, None, coeffs, 8, codes, deq, None, st, stream)
        elif args.single == "unrotate":
            fq.fp4q_mxfp4_unrotate(w, masks, deq, stream)
        elif args.single == "mma-layout":
            fq.fp4q_scales_to_mma_layout(sc16, tiled, stream)
        elif args.single == "copy":
            fq.fp4q_probe_copy(w, deq, stream)
        elif args.single == "dequant-nvfp4":
            fq.fp4q_dequant(fq.NVFP4, codes, sc16, S, rows, cols, deq, stream)
        elif args.single == "nvfp4-mse-group":
            fq.fp4q_nvfp4_sweep_group([dict(w=w, amax=amax, global_scale=S, nv_codes=codes, nv_scales=sc16,
                                            nv_deq=deq)], st, stream)
        elif args.single == "mxfp4-absmax-group":
            fq.fp4q_mxfp4_quant_group([dict(w=w, amax=amax, mx_codes=codes, mx_scales=sc32, mx_deq=deq)], st,
                                      stream)

    times = []
    for i in range(args.warmup + args.steps):
        flush.fill_(i & 0xFF)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        launch()
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(a.elapsed_time(b))
    hbm_peak, peak_kind, _ = load_peaks()
    per_elem, kname = SINGLE_PATHS[args.single]
    n = rows * cols
    med = statistics.median(times)
    gbs = per_elem * n / (med * 1e-3) / 1e9
    print(json.dumps({"single": args.single, "kernel": kname, "shape": [rows, cols],
                      "ms_median": med, "ms_min": min(times), "input_gbs": 2.0 * n / (med * 1e-3) / 1e9,
                      "algorithmic_gbs": gbs, "hbm_peak": hbm_peak, "peak_kind": peak_kind,
                      "hbm_frac": gbs / hbm_peak, "status": int(st.item())}), flush=True)
    return 0


# --------------------------------------------------------------------------- per-call latency

ACT_SHAPES = [(1, 4096), (16, 4096), (128, 4096), (1, 14336), (16, 14336), (2048, 4096), (4096, 14336)]


def run_act_latency(args):
    """Per-call latency of the NVFP4 sweep of a tensor quantized per call (an
    activation: tokens x hidden): the two-call path (fp4q_global_absmax, then
    fp4q_nvfp4_sweepmse) against the one-launch fp4q_nvfp4_sweep_dynamic, each
    issued `--steps` times back to back on one stream, eagerly and as one CUDA
    graph holding all the calls (device time per call without host launch
    cost); CUDA events around the whole run.  Prints one JSON line
    per shape (not the benchmark line)."""
    import fp4_post_weight_grid_b200 as fq
    from fp4_post_weight_grid_b200 import build as fbuild
    import synth
    fbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream()
    reps = max(args.steps, 20)
    for rows, cols in ACT_SHAPES:
        x = synth.t_weight(rows, cols, nu=4, scale=0.02, seed=13, device=dev)
        amax = torch.empty(1, device=dev)
        S = torch.empty(1, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
        deq = torch.empty_like(x)
        ws = torch.zeros(fq.fp4q_dynamic_workspace_bytes() // 4, dtype=torch.int32, device=dev)

        def two():
            fq.fp4q_global_absmax(x, amax, stream=stream)
            fq.fp4q_nvfp4_sweepmse(x, amax, codes, scales, S, deq, None, st, stream)

        def one():
            fq.fp4q_nvfp4_sweep_dynamic(x, None, amax, codes, scales, S, deq, None, ws, st, stream)

        res = {"act_latency": [rows, cols], "reps": reps}
        for name, fn in (("two_calls", two), ("dynamic", one)):
            for _ in range(max(args.warmup, 3)):
                fn()
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            res[name + "_eager_us"] = a.elapsed_time(b) * 1e3 / reps
            g = torch.cuda.CUDAGraph()                 # `reps` calls in one graph
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    fn()
            g.replay()
            torch.cuda.synchronize()
            a.record(stream)
            with torch.cuda.stream(stream):
                g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            res[name + "_graph_us"] = a.elapsed_time(b) * 1e3 / reps
            del g
        res["status"] = int(st.item())
        print(json.dumps(res), flush=True)
    return 0


# --------------------------------------------------------------------------- per-workload records

CONFIG_KEYS = ("cfg1", "cfg2", "cfg3", "cfg4", "focus")


def config_records(steps, warmup, keys=CONFIG_KEYS):
    """One record per smaller workload (not the benchmark line), yielded as it
    is measured: the outlier matrix (128 x 256 fp32, NVFP4-MSE), the
    q_proj-shaped 4096 x 4096 (NVFP4-MSE), the WMSE 11008 x 4096 with its
    importance vector, the rotated MXFP4 28672 x 8192 and, for context, the
    FOCUS forward quantizer on the q_proj shape.  Per record: the ABI sequence
    (global absmax + sweep, or the rotated MXFP4 pass) timed with CUDA events,
    median of `steps` launches after `warmup` (at least 3), a buffer of twice
    the L2 (at least 512 MB) rewritten between launches so that no launch
    starts with its input in L2; algorithmic bytes and their fraction of the
    measured HBM peak; parity with the oracle on sampled rows (all rows of the
    outlier matrix), element by element, the oracle's global scale coming from
    its own maximum over the whole weight; the aggregate reconstruction MSE of
    those rows on both sides (fp64); the oracle's time on those rows."""
    import fp4_post_weight_grid_b200 as fq
    from fp4_post_weight_grid_b200 import build as fbuild
    import oracle
    import synth
    fbuild.build()
    oracle.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm_peak, peak_kind, _ = load_peaks()
    flush = l2_flush_buffer(dev)
    stream = torch.cuda.current_stream()
    reps = max(steps, 5)
    warm = max(warmup, 3)

    def timed(fn):
        ts = []
        for i in range(warm + reps):
            flush.fill_(i & 0xFF)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            if i >= warm:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def bits(t):
        t = t.detach().cpu()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    workloads = {
        "cfg1": ("outliers 128x256 fp32, NVFP4-MSE", lambda: synth.small_outliers(), None, None, "nv"),
        "cfg2": ("q_proj 4096x4096 bf16, NVFP4-MSE", lambda: synth.q_proj(4096, 4096, seed=2, device=dev), None,
                 None, "nv"),
        "cfg3": ("WMSE 11008x4096 bf16, NVFP4-WMSE",
                 lambda: synth.t_weight(11008, 4096, nu=4, scale=0.02, seed=3, device=dev),
                 lambda: synth.importance_diag_xtx(cols=4096, tokens=2048, seed=3), None, "nv"),
        "cfg4": ("MXFP4+Hadamard 28672x8192 bf16",
                 lambda: synth.t_weight(28672, 8192, nu=3, scale=0.015, seed=4, device=dev),
                 None, lambda: synth.sign_masks(8192, seed=4), "mx"),
        "focus": ("FOCUS NVFP4 (sub-blocks of 8) 4096x4096 bf16",
                  lambda: synth.q_proj(4096, 4096, seed=2, device=dev), None, None, "focus"),
    }
    for key in keys:
        name, make_w, make_imp, make_masks, kind = workloads[key]
        w = make_w().to(dev)
        rows, cols = w.shape
        n = rows * cols
        isz = w.element_size()
        imp_np = make_imp().numpy() if make_imp else None
        imp = torch.from_numpy(imp_np).to(dev) if make_imp else None
        masks_np = make_masks() if make_masks else None
        masks = torch.from_numpy(masks_np.view(np.int32)).to(dev) if make_masks else None
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
        deq = torch.empty_like(w)
        if kind == "nv":
            amax = torch.empty(1, device=dev)
            S = torch.empty(1, device=dev)
            scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)

            def fn():
                fq.fp4q_global_absmax(w, amax, st, stream)
                if imp is None:
                    fq.fp4q_nvfp4_sweepmse(w, amax, codes, scales, S, deq, None, st, stream)
                else:
                    fq.fp4q_nvfp4_sweepwmse(w, amax, imp, codes, scales, S, deq, None, st, stream)
            nbytes = n * (isz + isz + 0.5 + 1.0 / 16 + isz)
        elif kind == "focus":
            nv0 = fq.nvfp4_quantize(w)                       # the stored scales to relax
            scales = nv0.scales
            S = nv0.global_scale
            gen = torch.Generator(device="cpu").manual_seed(8)
            coeffs = (0.8 + 0.45 * torch.rand((rows, cols // 8), generator=gen)).to(torch.float16).to(dev)

            def fn():
                fq.fp4q_focus_quant(fq.NVFP4, w, scales, S, coeffs, 8, codes, deq, None, st, stream)
            nbytes = n * (isz + 1.0 / 16 + 2.0 / 8 + 0.5 + isz)
        else:
            scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)

            def fn():
                fq.fp4q_mxfp4_quant_hadamard(w, masks, codes, scales, deq, None, st, stream)
            nbytes = n * (isz + 0.5 + 1.0 / 32 + isz)
        ms = timed(fn)
        # parity on sampled rows
        idx = np.arange(rows) if rows <= 128 else np.array([0, 1, rows // 2, rows - 1])
        x_all = w.float().cpu().numpy()
        x = np.ascontiguousarray(x_all[idx])
        t0 = time.perf_counter()
        if kind == "nv":
            S_o = oracle.global_scale(oracle.global_absmax(x_all))
            window = oracle.NVFP4_WMSE_WINDOW if imp_np is not None else oracle.NVFP4_MSE_WINDOW
            o = oracle.nvfp4_quant(x, S=S_o, importance=imp_np, window=window)
        elif kind == "focus":
            o = oracle.focus_quant(0, x, bits(scales)[idx], coeffs.cpu().numpy()[idx], 8, S=float(S.item()))
        else:
            o = oracle.mxfp4_quant(x, sign_masks=masks_np)
        t_orc = time.perf_counter() - t0
        del x_all
        deq_o = oracle.bf16_round(o["y"]) if w.dtype == torch.bfloat16 else o["y"]
        dg = bits(deq)[idx]
        same = (np.array_equal(bits(codes)[idx], o["codes"])
                and (kind == "focus" or np.array_equal(bits(scales)[idx], o["scales"]))
                and np.array_equal(dg.view(np.uint32) if dg.dtype == np.float32 else dg,
                                   deq_o.view(np.uint32) if deq_o.dtype == np.float32 else deq_o))
        if kind == "nv":
            same = same and bool(np.float32(S.item()) == np.float32(o["S"]))
        ref = o["rotated"] if kind == "mx" else x
        y_gpu = deq.float().cpu().numpy()[idx].astype(np.float64)
        y_orc = (deq_o.astype(np.uint32) << 16).view(np.float32).astype(np.float64) \
            if w.dtype == torch.bfloat16 else deq_o.astype(np.float64)
        mse_gpu = float(np.mean((ref.astype(np.float64) - y_gpu) ** 2))
        mse_orc = float(np.mean((ref.astype(np.float64) - y_orc) ** 2))
        gbs = nbytes / (ms * 1e-3) / 1e9
        rec = {"key": key, "workload": name, "shape": [rows, cols], "ms": ms,
               "input_gbs": n * isz / (ms * 1e-3) / 1e9,
               "elements_per_s": n / (ms * 1e-3), "algorithmic_bytes": nbytes, "algorithmic_gbs": gbs,
               "hbm_frac": gbs / hbm_peak, "peak_kind": peak_kind, "status": int(st.item()),
               "parity_rows": int(idx.size), "parity_bit_exact": bool(same),
               "mse_gpu": mse_gpu, "mse_oracle": mse_orc,
               "mse_rel_diff": abs(mse_gpu - mse_orc) / max(mse_orc, 1e-300),
               "oracle_s_on_rows": t_orc, "oracle_cores": oracle.max_threads(),
               "input_sha256": {"w": tensor_sha256(w),
                                **({"importance": tensor_sha256(imp_np)} if make_imp else {}),
                                **({"sign_masks": tensor_sha256(masks_np)} if make_masks else {})}}
        del w, deq, codes
        torch.cuda.empty_cache()
        yield rec
    del flush
    torch.cuda.empty_cache()


def run_configs(args):
    """--configs: one JSON record per smaller workload (config_records)."""
    for rec in config_records(args.steps, args.warmup):
        print(json.dumps(rec), flush=True)
    return 0


def per_config_summary(steps, warmup):
    """The benchmark line's `per_config`: for the four smaller workloads, the
    median time of their ABI sequence (L2 flushed between launches), the
    algorithmic GB/s and HBM fraction, and bit-exact parity with the oracle on
    sampled rows (config_records)."""
    out = {}
    for rec in config_records(steps, warmup, keys=("cfg1", "cfg2", "cfg3", "cfg4")):
        out[rec["key"]] = {"workload": rec["workload"], "us_median": rec["ms"] * 1e3,
                           "algorithmic_gbs": rec["algorithmic_gbs"], "hbm_frac": rec["hbm_frac"],
                           "parity_bit_exact": rec["parity_bit_exact"], "parity_rows": rec["parity_rows"],
                           "mse_rel_diff": rec["mse_rel_diff"], "status": rec["status"]}
    return out


# --------------------------------------------------------------------------- GPTQ

def run_gptq(args):
    """Time fp4q_nvfp4_gptq (ScaleSweep inside GPTQ) on one synthetic weight
    (`--shape`, default the WMSE workload's 11008 x 4096) with the Gram matrix
    of 2048 synthetic bf16 activations (N(0,1), 1% of the columns x50).  Each
    launch starts from a fresh fp32 copy of the weight (the call overwrites it;
    the copy is inside the timed region, ~0.1 ms).  Reports the time and the
    rate of the fused multiply-adds of the error updates (rows * cols^2 / 2)
    against the FP32 lane peak.  Prints one JSON line (not the benchmark line)."""
    import fp4_post_weight_grid_b200 as fq
    from fp4_post_weight_grid_b200 import build as fbuild
    import synth
    fbuild.build()
    rows, cols = (int(v) for v in args.shape.lower().split("x"))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w0 = synth.t_weight(rows, cols, nu=4, scale=0.02, seed=3, device=dev).float()
    g = torch.Generator(device="cpu").manual_seed(3)
    X = torch.randn(2048, cols, generator=g)
    X[:, torch.randperm(cols, generator=g)[:max(1, cols // 100)]] *= 50.0
    X = X.to(torch.bfloat16).to(dev, torch.float64)
    H = X.T @ X
    H += 0.01 * H.diagonal().mean() * torch.eye(cols, dtype=torch.float64, device=dev)
    U = torch.linalg.cholesky(torch.cholesky_inverse(torch.linalg.cholesky(H))).mT.contiguous().float()
    del X, H
    w = torch.empty_like(w0)
    amax = torch.empty(1, device=dev)
    S = torch.empty(1, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    deq = torch.empty_like(w0)
    ws = torch.empty(fq.fp4q_gptq_workspace_bytes(rows), dtype=torch.uint8, device=dev)
    fq.fp4q_global_absmax(w0, amax)
    stream = torch.cuda.current_stream()

    def launch():
        w.copy_(w0)
        fq.fp4q_nvfp4_gptq(w, U, amax, codes, scales, S, deq, ws, st, stream)

    times = []
    for i in range(max(args.warmup, 1) + args.steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        launch()
        b.record(stream)
        torch.cuda.synchronize()
        if i >= max(args.warmup, 1):
            times.append(a.elapsed_time(b))
    med = statistics.median(times)
    fmas = rows * cols * (cols - 1) / 2
    clk = load_peaks()[2]
    peak = 148 * SM_FP32_LANES * clk * 1e6 / 1e12
    # the oracle beside it: parity and time on 4 sampled rows (rows are independent)
    import oracle
    oracle.build()
    idx = np.array([0, 1, rows // 2, rows - 1])
    t0 = time.perf_counter()
    o = oracle.nvfp4_gptq(w0.cpu().numpy()[idx], U.cpu().numpy(), S=float(S.item()))
    t_orc = time.perf_counter() - t0
    got = codes.cpu().numpy()[idx]
    print(json.dumps({"gptq": [rows, cols], "ms_median": med, "ms_min": min(times),
                      "update_fma": fmas, "tfma_per_s": fmas / (med * 1e-3) / 1e12,
                      "fp32_lane_peak_tfma_per_s": peak, "frac": fmas / (med * 1e-3) / 1e12 / peak,
                      "status": int(st.item()), "parity_rows": 4,
                      "parity_bit_exact": bool(np.array_equal(got, o["codes"]) and
                                               np.array_equal(scales.cpu().numpy()[idx], o["scales"])),
                      "oracle_ms_per_row": t_orc / 4 * 1e3, "oracle_cores": oracle.max_threads()}), flush=True)
    return 0


# --------------------------------------------------------------------------- main

def build_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="leave out the per-workload records of the four smaller workloads")
    ap.add_argument("--configs", action="store_true",
                    help="one JSON record per small workload: time, bytes, roofline, parity, MSE, oracle time")
    ap.add_argument("--gptq", action="store_true",
                    help="time the ScaleSweep inside GPTQ on one weight (default 11008x4096)")
    ap.add_argument("--act-latency", action="store_true",
                    help="per-call latency of the NVFP4 sweep on activation-sized tensors, two calls vs one launch")
    ap.add_argument("--single", choices=sorted(SINGLE_PATHS), default=None,
                    help="time one kernel on one tensor instead of the benchmark step")
    ap.add_argument("--shape", default="16384x8192")
    ap.add_argument("--streams", type=int, default=2, choices=[1, 2, 3, 4],
                    help="1: one stream; n > 1: MXFP4 passes on one stream, NVFP4 sweeps "
                         "round-robin on n - 1 more, each after its own tensor's MXFP4 pass")
    ap.add_argument("--mode", default="groups", choices=["batch", "calls", "groups"],
                    help="batch: fp4q_quantize_batch (one persistent launch per chunk of weights); "
                         "calls: two launches per weight (fp4q_mxfp4_quant_absmax + the NVFP4 sweep); "
                         "groups: fp4q_mxfp4_quant_group + fp4q_nvfp4_sweep_group per --group weights")
    ap.add_argument("--group", type=int, default=4, help="weights per grouped launch (at most 32)")
    ap.add_argument("--prio", default="none", choices=["none", "nv", "mx"],
                    help="give the NVFP4 (nv) or the MXFP4 (mx) stream the higher CUDA stream priority")
    ap.add_argument("--layer-groups", default="",
                    help="split each layer's 7 weights (q,k,v,o,gate,up,down) into consecutive groups "
                         "of these sizes, e.g. 3,2,1,1 (overrides --group)")
    ap.add_argument("--chunk", type=int, default=128, help="weights per batch launch (at most 128)")
    ap.add_argument("--lag", type=int, default=0,
                    help="with --streams > 1: the MXFP4 pass of tensor (or group) t waits for the sweep of t - lag")
    return ap


def main():
    args = build_parser().parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.single:
        return run_single(args)
    if args.act_latency:
        return run_act_latency(args)
    if args.configs:
        return run_configs(args)
    if args.gptq:
        if args.shape == "16384x8192":
            args.shape = "11008x4096"
        return run_gptq(args)

    import fp4_post_weight_grid_b200 as fq
    from fp4_post_weight_grid_b200 import build as fbuild
    fbuild.build()
    fq.load()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    model = Model(fq, dev, seed=rank_seed(rank), with_events=True)
    p0 = p1 = 0
    if args.prio != "none":
        lo, hi = torch.cuda.Stream.priority_range()     # (least, greatest)
        p0 = hi if args.prio == "mx" else lo             # stream 0 carries the MXFP4 launches
        p1 = hi if args.prio == "nv" else lo             # the others the NVFP4 sweeps
    stream = torch.cuda.Stream(device=dev, priority=p0)
    streams = [stream] + [torch.cuda.Stream(device=dev, priority=p1) for _ in range(args.streams - 1)]
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()

    if args.mode == "batch":
        model.batch_setup(args.chunk)
    if args.mode == "groups":
        sizes = [int(v) for v in args.layer_groups.split(",")] if args.layer_groups else None
        model.group_setup(args.group, sizes)

    def run_step():
        if args.mode == "batch":
            model.step_batch(stream)
        elif args.mode == "groups":
            model.step_groups(stream, streams[1] if len(streams) > 1 else stream, args.lag)
        elif args.streams == 1:
            model.step(stream)
        else:
            model.step_schedule(streams, args.lag)

    with torch.cuda.stream(stream):
        run_step()                               # eager warm-up before capture
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            run_step()
    for _ in range(max(args.warmup, 3) - 1):
        graph.replay()
    torch.cuda.synchronize()
    if int(model.status.item()) != 0:
        raise RuntimeError(f"device status {int(model.status.item())} during warm-up")

    clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for _ in range(args.steps):
            graph.replay()
        t_end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(ms, dist, dev)
    status = int(model.status.item())

    hbm_peak, peak_kind, sm_max = load_peaks()
    copy_gbs = copy_probe_gbs(fq, dev)
    if copy_gbs > hbm_peak:      # the HBM peak is the larger of the two copies
        hbm_peak, peak_kind = copy_gbs, "own copy kernel"
    n = model.elements
    bytes_in = 2.0 * n * world
    value = bytes_in / (ms * 1e-3) / 1e9
    clock_mhz = clk.get("sm_mhz") or sm_max
    if args.mode == "batch":
        # the batch kernel: per-launch durations of the last timed step
        kname = "batch_kernel (NVFP4-MSE + MXFP4, bf16)"
        kern_ms = sum(ev[0].elapsed_time(ev[1]) for _, _, _, ev in model.chunks)
        kern_bytes = (B_NVFP4 + B_MXFP4) * n
        n_launch = len(model.chunks)
    elif args.mode == "groups":
        # the grouped NVFP4 sweep kernel: per-launch durations of the last timed step
        kname = "nvfp4_group_kernel (MSE, bf16)"
        kern_ms = sum(ev[0].elapsed_time(ev[1]) for _, _, _, ev in model.groups)
        kern_bytes = B_NVFP4 * n
        n_launch = len(model.groups)
    else:
        # the NVFP4 sweep kernel: per-launch durations of the last timed step
        kname = "nvfp4_sweep_kernel (MSE, bf16)"
        kern_ms = sum(model.sweep_ms())
        kern_bytes = B_NVFP4 * n
        n_launch = len(model.shapes)
    kern_gbs = kern_bytes / (kern_ms * 1e-3) / 1e9
    per_launch = {"launches_per_step": n_launch, "mean_launch_ms": kern_ms / n_launch,
                  "algorithmic_bytes_per_launch": kern_bytes / n_launch,
                  "bytes_basis": "2 B bf16 in + 0.5 B codes + 1/16 B scale + 2 B bf16 reconstruction per element"}
    traffic = None
    explain = {"note": "the kernel's time is set by its instruction issue rate, not by DRAM"}
    if args.mode != "batch":
        traffic = measured_traffic_per_launch(kern_bytes / n_launch / B_NVFP4)
        prof = nvfp4_profile_current()
        issue_peak = 148 * 4 * 32 * clock_mhz * 1e6             # lane-instructions/s at one warp-instruction/clk/SMSP
        if prof is not None:
            ipe = prof["warp_inst_per_element"]
            explain.update({
                "warp_instructions_per_element": ipe,
                "issue_active_pct_of_active_cycles": prof["issue_active_pct"],
                "basis": "ncu smsp__inst_executed.sum and smsp__issue_active on one 16384x8192 weight "
                         "through the same kernel "
                         "(profiles/nvfp4_sweep_mse_16384x8192.md)",
                "issue_bound_time_fraction": (n * ipe * 32 / issue_peak) / (kern_ms * 1e-3),
                "issue_peak_lane_inst_per_s": issue_peak})
        else:
            explain["basis"] = "no ncu counters for the current sources"
    roof = {"bound": "hbm", "achieved": kern_gbs, "peak": hbm_peak, "unit": "GB/s", "frac": kern_gbs / hbm_peak,
            "traffic": traffic, "kernel": kname, "peak_kind": peak_kind, **per_launch, "explain": explain}
    step_bytes = (B_NVFP4 + B_MXFP4) * n
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tensors": len(model.shapes), "elements": n,
                   "input_dtype": "bf16", "output_formats": "NVFP4 (E2M1 + E4M3 scales + fp32 S) and MXFP4 "
                                                           "(E2M1 + E8M0 scales), bf16 reconstructions",
                   "input_bytes": 2 * n, "l2": "inputs 13.96 GB > 126 MB L2, no flush",
                   "parallelism": f"replicas x{world} (weak)", "graph": "one CUDA graph per step",
                   "mode": args.mode},
        "elements_per_s": n * world / (ms * 1e-3),
        "hbm_frac_step": step_bytes / (ms * 1e-3) / 1e9 / hbm_peak,
        "hbm_frac_step_of_spec": step_bytes / (ms * 1e-3) / 1e9 / HBM_SPEC_GBS,
        "hbm_copy_probe": {"gbs": copy_gbs, "bytes_moved": 2 * (512 << 20), "kernel": "probe_copy_kernel",
                           "peak_used": hbm_peak, "peak_kind": peak_kind},
        "roofline": roof,
        "gpu_launches": model.launches_per_step * args.steps,
        "clocks": clk,
        "status": status,
    }
    if rank == 0:
        par = step_parity(model)
        line["parity"] = par["ok"]
        line["parity_detail"] = par
        try:
            if args.e2e_steps < 1:
                raise RuntimeError("skipped (--e2e-steps 0)")
            e2e_dt, h2d, d2h = e2e_run(fq, model, args.e2e_steps, dev)
            line["e2e"] = {"value": 2.0 * n / e2e_dt / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_dt * 1e3}
        except Exception as e:   # report, do not hide
            line["e2e"] = {"value": None, "unit": "GB/s", "error": repr(e)}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        if world == 1 and not args.no_per_config:
            del model, graph
            torch.cuda.empty_cache()
            line["per_config"] = per_config_summary(max(args.steps, 10), args.warmup)
            graph = None
        print(json.dumps(line), flush=True)
    if dist is not None:
        del graph
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
