"""Benchmark of the fused EntroPack decode on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --sweep      (every workload, one GPU: a table, not the bench line)
    python bench.py --linear     (decode-then-GEMM against a resident weight, one GPU)
    python bench.py --gemv       (the fused decode-GEMV on 1 to 8 tokens, one GPU)
    python bench.py --split      (the decode on part of the GPU beside the GEMM, one GPU)
    python bench.py --knee       (cycles per step against tiles per warp scheduler, one GPU)

One step = one ep_decode_tensor call: the whole hot path (tile setup, table
staging, payload staging, rANS decode, lattice reconstruction, row rescale,
conversion and store) over the 3840x10240 bf16 Student-t(6)*0.02 weight matrix
(the DiT FFN down-projection shape) compressed at 4 bpp, decoded to bf16.  The
timed steps replay a CUDA graph of decode calls (eager launches if capture fails).
Inputs are resident in HBM; steps rotate over 4 copies of (stream, output) so
the working set (4 x ~98 MB) exceeds the 126 MB L2.  Multi-GPU (weak scaling):
rank r decodes its own tensor of the same shape (seed 7 + r), as the layers of
a model are independent problems; nothing crosses between GPUs on the data
path.  The value is the weights of all ranks over the slowest rank's time.

Prints one JSON line on rank 0.  --impl reference times the CPU oracle instead
(the plain C decoder, threads over tile ranges) on a bounded sample of the same
stream.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from types import SimpleNamespace

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decoded G weights/s and achieved HBM GB/s vs B200 peak (BF16 out, 4 bpp)"
UNIT = "G weights/s"
ROWS, COLS, TARGET = 3840, 10240, 4.0
WORKLOAD = "3840x10240 bf16 Student-t(6)*0.02 weight (DiT FFN down projection), 4 bpp, decode to bf16"
# the pages' 0.23 ms for a 39.3 M-weight layer, BF16 out, 4 bpp, on one H20 ([tables] Table 6; context only)
PAGES_GWPS = 39321600 / 0.23e-3 / 1e9
ROTATE = 4
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _kernel_sha():
    """Hash of the decoder's source without comments and blank space (a comment edit keeps it)."""
    import re

    h = hashlib.sha256()
    for p in ("dit_weight_compression_ep_b200/csrc/decode.cu", "dit_weight_compression_ep_b200/csrc/ep_format.h"):
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            code = re.sub(r"//[^\n]*", "", f.read())
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


def _traffic_per_launch():
    """(DRAM bytes per launch, bytes the SMs wrote into L2 per launch) from the committed ncu
    summary, if it was taken on this kernel source; (None, None) otherwise."""
    try:
        with open(os.path.join(ROOT, "profiles", "decode_headline_traffic.json")) as f:
            d = json.load(f)
        if d.get("kernel_sha") == _kernel_sha():
            return float(d["dram_bytes_per_launch"]), float(d["l2_write_bytes_from_sm"])
    except Exception:
        pass
    return None, None


class Clocks:
    """nvidia-smi samples (SM clock, throttle reasons) taken while the benchmark runs."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        inside = [r for t, r in self.rows if t0 <= t <= t1]
        window = "timed region"
        if len(inside) < 3:
            inside = [r for _, r in self.rows]
            window = "whole run (timed region shorter than the sampling period)"
        sm = [float(r[2]) for r in inside if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in inside if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(4) if len(r) > 6 + i and r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "window": window}


# Other workloads the default timing can run instead of the headline (`--workload`), to time or
# profile them with the same protocol: name -> (target bpp, description).  Only the headline's
# line is the benchmark; these are for measurements.
OTHER_WORKLOADS = {
    "dit-qkv-8": (8.0, "11520x3840 bf16 Student-t(6)*0.02 weight (DiT qkv projection, block 0), 8 bpp "
                       "(b = 12, two-level table), decode to bf16"),
    "llm-prefill-8": (8.0, "5120x25600 bf16 N(0, 0.015^2) weight, 0.05% outliers at 10 sigma, row lognormal(0.5) "
                           "(LLM prefill), 8 bpp (b = 12, two-level table), decode to bf16"),
}


def _make_weights(rank: int = 0, workload: str = "headline"):
    from dit_weight_compression_ep_b200 import synth

    if workload == "dit-qkv-8":
        return synth.generate(synth.dit_stack_layer(rank, "qkv"))
    if workload == "llm-prefill-8":
        return synth.generate(synth.llm_prefill(True, seed=5 + rank))
    return synth.generate(synth.headline(seed=7 + rank))


def _workload(args):
    """(target bpp, description) of the workload this run times."""
    return (TARGET, WORKLOAD) if args.workload == "headline" else OTHER_WORKLOADS[args.workload]


def reduce_max(values, world: int, device=None):
    """Element-wise max over ranks of a few host floats.

    Every rank calls it at the same point with the same number of values; with
    one rank it returns them unchanged.  The tensor lives on `device` (the
    rank's GPU under NCCL, the CPU under gloo)."""
    values = [float(v) for v in values]
    if world == 1:
        return values
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def relaunch(n: int, script: str, argv, timeout_s: float = 3600.0, capture: bool = False):
    """Run `script argv` as n ranks on this node under torchrun, with a loopback rendezvous, and
    wait for them: `bench.py --gpus N` does this when no launcher started it (every rank then
    reads RANK / LOCAL_RANK / WORLD_SIZE from its environment).  Returns the CompletedProcess."""
    import socket
    import subprocess

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", script, *argv]
    return subprocess.run(cmd, timeout=timeout_s, capture_output=capture, text=capture)


def weak_value(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput in G units/s: every rank's units over the slowest rank's step time."""
    return world * units_per_rank / (ms_per_step * 1e-3) / 1e9


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    target, workload = _workload(args)
    W = _make_weights(rank, args.workload)
    t_enc = time.time()
    blob = ep.encode_tensor(W, target)
    t_enc = time.time() - t_enc
    numel = blob.rows * blob.cols
    read_bytes = blob.stored_device_bytes()
    write_bytes = numel * 2
    sets = [(ep.DeviceBlob(blob, dev), torch.empty((blob.rows, blob.cols), dtype=torch.bfloat16, device=dev))
            for _ in range(ROTATE)]
    stream = torch.cuda.Stream(dev)  # a side stream: graph capture is not allowed on the legacy default stream

    def step(i):
        db, out = sets[i % ROTATE]
        ep.decode_tensor(db, ep.BF16, out=out, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if ep.decode_status(stream) != 0:
        raise RuntimeError("decode reported a corrupt stream")

    clocks = Clocks(local_rank) if rank == 0 else None
    time.sleep(0.3 if clocks else 0.0)
    # The timed steps replay a CUDA graph of CH decode calls (CH divides K): one cooperative
    # launch per call, as launched eagerly, without the host's launch gaps.  The roofline's
    # launch duration is then the timed region over the launches (the short gaps between
    # the graph's kernels included: an upper bound of the kernel's own time).
    CH = max(d for d in range(1, min(50, args.steps) + 1) if args.steps % d == 0)
    graph, launch = None, "eager, one event pair around each launch"
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for j in range(CH):
                step(j)
        graph = g
        launch = (f"cuda graph of {CH} decode calls replayed {args.steps // CH} times; launch duration = "
                  f"timed region / launches")
        with torch.cuda.stream(stream):
            graph.replay()  # untimed
        torch.cuda.synchronize(dev)
    except Exception:  # capture unsupported here: eager launches, an event pair around each
        graph = None
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)] \
        if graph is None else []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0w = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        if graph is not None:
            for _ in range(args.steps // CH):
                graph.replay()
        else:
            for i in range(args.steps):
                ev[i][0].record(stream)
                step(i)
                ev[i][1].record(stream)
        end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t1w = time.time()
    ms_total = start.elapsed_time(end)
    launch_ms = [a.elapsed_time(b) for a, b in ev] if ev else [ms_total / args.steps]
    status = ep.decode_status(stream)
    if status != 0:
        raise RuntimeError(f"decode status {status}")
    ms_total, avg_launch_ms = reduce_max([ms_total, sum(launch_ms) / len(launch_ms)], world, dev)
    del graph
    if clocks:
        time.sleep(0.2)
        clocks.stop()

    # ---- the same decodes with each tensor's lookup table prepared once (ep_decode_prepare,
    # before the timed region: a weight decoded at every step keeps its table beside its
    # compressed bytes); same graph of CH calls, same rotation.  Reported beside `value`.
    luts = [ep.prepare_lut(db, stream=stream) for db, _ in sets]

    def pstep(i):
        db, out = sets[i % ROTATE]
        ep.decode_tensor_prepared(db, luts[i % ROTATE], ep.BF16, out=out, stream=stream)

    ref = sets[0][1].clone()
    pstep(0)
    torch.cuda.synchronize(dev)
    if ep.decode_status(stream) != 0 or not torch.equal(sets[0][1].view(torch.int16), ref.view(torch.int16)):
        raise RuntimeError("prepared decode differs from the per-call decode")
    local_prep = -1.0  # every rank takes the same barrier and reduction, whatever happens here
    try:
        pg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pg, stream=stream):
            for j in range(CH):
                pstep(j)
        with torch.cuda.stream(stream):
            pg.replay()
        torch.cuda.synchronize(dev)
    except RuntimeError:  # capture unsupported here: no prepared figure
        pg = None
    if world > 1:
        dist.barrier()
    if pg is not None:
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            pa.record(stream)
            for _ in range(args.steps // CH):
                pg.replay()
            pb.record(stream)
        torch.cuda.synchronize(dev)
        local_prep = pa.elapsed_time(pb) / args.steps
        del pg
    prep_max, neg_min = reduce_max([local_prep, -local_prep], world, dev)
    prep_ms = prep_max if -neg_min >= 0.0 else None  # None unless every rank has a figure
    if ep.decode_status(stream) != 0:
        raise RuntimeError("prepared decode reported a corrupt stream")

    # ---- end to end through the public API: pinned host stream in, pinned host weights out.
    # Two slots (device buffers, pinned output, stream) alternate, so one step's copy back
    # can overlap the next step's copy in and decode (the copy engines of the two
    # directions work in parallel); every step still moves its own bytes both ways.
    e2e_steps = max(3, min(args.steps, 20))
    h_pay = torch.from_numpy(blob.payload.view(np.int16)).pin_memory()
    h_tix = torch.from_numpy(blob.tile_index.view(np.int32)).pin_memory()
    h_ft = torch.from_numpy(blob.freq_tables).pin_memory()
    h_rs = torch.from_numpy(blob.row_scales).pin_memory()
    slots = [(sets[k][0], sets[k][1], torch.empty((blob.rows, blob.cols), dtype=torch.bfloat16).pin_memory(),
              torch.cuda.Stream(dev)) for k in range(2)]
    h2d = h_pay.numel() * 2 + h_tix.numel() * 4 + h_ft.numel() + h_rs.numel() * 4
    d2h = slots[0][2].numel() * 2

    def e2e_step(i):
        db, out, h_out, st = slots[i % 2]
        with torch.cuda.stream(st):
            db.payload.copy_(h_pay, non_blocking=True)
            db.tile_index.copy_(h_tix, non_blocking=True)
            db.freq_tables.copy_(h_ft, non_blocking=True)
            db.row_scales.copy_(h_rs, non_blocking=True)
            ep.decode_tensor(db, ep.BF16, out=out, stream=st)
            h_out.copy_(out, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _, _, _, st in slots:
        st.wait_event(a)
    for i in range(e2e_steps):
        e2e_step(i)
    for _, _, _, st in slots:
        stream.wait_stream(st)
    b.record(stream)
    torch.cuda.synchronize(dev)
    (e2e_ms,) = reduce_max([a.elapsed_time(b) / e2e_steps], world, dev)
    if ep.decode_status(stream) != 0:
        raise RuntimeError("e2e decode reported a corrupt stream")

    # ---- weight offload: each step streams the compressed layer from pinned host memory, decodes
    # it on the GPU and reads 16 bytes of the result back (the weights are consumed on the GPU);
    # beside it, the host-to-device time of the same layer in bf16
    def off_step(i):
        db, out, h_out, st = slots[i % 2]
        with torch.cuda.stream(st):
            db.payload.copy_(h_pay, non_blocking=True)
            db.tile_index.copy_(h_tix, non_blocking=True)
            db.freq_tables.copy_(h_ft, non_blocking=True)
            db.row_scales.copy_(h_rs, non_blocking=True)
            ep.decode_tensor(db, ep.BF16, out=out, stream=st)
            h_probe[i % 2].copy_(out.view(-1)[:8], non_blocking=True)

    h_probe = [torch.empty(8, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for i in range(3):
        off_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _, _, _, st in slots:
        st.wait_event(a)
    for i in range(e2e_steps):
        off_step(i)
    for _, _, _, st in slots:
        stream.wait_stream(st)
    b.record(stream)
    torch.cuda.synchronize(dev)
    h_bf16 = torch.empty((blob.rows, blob.cols), dtype=torch.bfloat16).pin_memory()
    d_bf16 = torch.empty_like(h_bf16, device=dev)
    a2, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            d_bf16.copy_(h_bf16, non_blocking=True)
        a2.record(stream)
        for _ in range(e2e_steps):
            d_bf16.copy_(h_bf16, non_blocking=True)
        b2.record(stream)
    torch.cuda.synchronize(dev)
    off_ms, bf16_h2d_ms = reduce_max([a.elapsed_time(b) / e2e_steps, a2.elapsed_time(b2) / e2e_steps], world, dev)
    del d_bf16, h_bf16
    if ep.decode_status(stream) != 0:
        raise RuntimeError("offload decode reported a corrupt stream")

    # ---- context: a torch bf16 matmul of the same layer with 4096 tokens
    X = torch.randn(4096, blob.cols, dtype=torch.bfloat16, device=dev)
    Wd = sets[0][1]
    for _ in range(3):
        torch.matmul(X, Wd.t())
    torch.cuda.synchronize(dev)
    ma, mb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    ma.record(cur)
    for _ in range(10):
        torch.matmul(X, Wd.t())
    mb.record(cur)
    torch.cuda.synchronize(dev)
    mm_ms = ma.elapsed_time(mb) / 10

    if rank != 0:
        return None
    ms_per_step = ms_total / args.steps
    value = weak_value(world, numel, ms_per_step)
    peak, peak_kind = _peaks()
    alg_bytes = read_bytes + write_bytes
    achieved = alg_bytes / (avg_launch_ms * 1e-3) / 1e9
    traffic, l2_writes = _traffic_per_launch() if args.workload == "headline" else (None, None)
    cpu = cpu_baseline(blob, seconds=args.cpu_seconds) if world == 1 else None
    return {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": round(value / (world * PAGES_GWPS), 3) if args.workload == "headline" else None,
        "dtype": "u32+f32", "data": "synthetic",
        "config": {"workload": workload, "rows": blob.rows, "cols": blob.cols, "target_bpp": target,
                   "stored_bpp": round(blob.stored_bpp, 4), "b": blob.b, "tile_vectors": blob.V,
                   "tiles": blob.ntiles, "out": "bf16", "launch": launch,
                   "ranks": ("rank r decodes its own tensor (seed 7 + r)" if args.workload == "headline" else
                             "rank r decodes its own tensor of this workload") + "; no collective on the data path",
                   "l2": f"inputs larger than L2: steps rotate over {ROTATE} stream/output copies "
                         f"({ROTATE * alg_bytes / 1e6:.0f} MB > {L2_BYTES / 1e6:.0f} MB L2)",
                   "vs_baseline_ref": "pages' 0.23 ms per 39.3 M-weight layer on one H20 (Table 6), context only",
                   "encode_s": round(t_enc, 3)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "traffic_note": "dram read + write of one ncu capture; the write side is low because the "
                                     "output is still dirty in L2 when the launch ends: the SMs' write sectors "
                                     "into L2 are in sm_write_bytes_into_l2",
                     "sm_write_bytes_into_l2": l2_writes,
                     "algorithmic_bytes_per_launch": alg_bytes, "read_bytes": read_bytes, "write_bytes": write_bytes,
                     "avg_launch_us": round(avg_launch_ms * 1e3, 3), "peak_kind": peak_kind},
        "cpu_baseline": cpu,
        "e2e": {"value": round(weak_value(world, numel, e2e_ms), 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "pinned host stream in, decode, pinned host weights out; two slots on two streams "
                       "alternate so one step's copy back overlaps the next step's copy in"},
        "e2e_offload": {"value": round(weak_value(world, numel, off_ms), 3), "unit": UNIT, "ms_per_step": round(off_ms, 4),
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 16,
                        "bf16_h2d_ms_same_layer": round(bf16_h2d_ms, 4),
                        "how": "each step: the compressed layer from pinned host memory, decoded on the GPU, 16 bytes "
                               "of the result read back (weights consumed on the GPU); two slots on two streams; "
                               "bf16_h2d_ms_same_layer: copying the same layer's bf16 weights instead"},
        "prepared": None if prep_ms is None else {
            "value": round(weak_value(world, numel, prep_ms), 2), "unit": UNIT, "ms_per_step": round(prep_ms, 5),
            "frac": round(alg_bytes / (prep_ms * 1e-3) / 1e9 / peak, 4),
            "how": "ep_decode_tensor_prepared: each tensor's lookup table built once by ep_decode_prepare before "
                   "the timed region (no per-call table build, no grid barrier, ordinary launch); same graph, "
                   "same rotation"},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(t0w, t1w) if clocks else None,
        "context": {"torch_bf16_matmul_4096_tokens_us": round(mm_ms * 1e3, 2),
                    "decode_over_matmul": round(avg_launch_ms / mm_ms, 4),
                    "pages_decode_over_matmul_h20": 0.094},
    }


def _oracle_threads(blob, t_ranges, nthreads, dtype):
    """Decode tile ranges with the oracle on nthreads host threads (the C call releases the GIL)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    pay = blob.payload[:blob.payload_words]

    def work(rng):
        t0, t1 = rng
        oracle.decode(pay, blob.tile_index, blob.freq_tables, blob.row_scales, blob.rows, blob.cols, dtype, t0, t1)
        return min(t1 * blob.V, blob.rows * blob.cols // 8) - t0 * blob.V

    with ThreadPoolExecutor(nthreads) as ex:
        return sum(ex.map(work, t_ranges)) * 8


def cpu_baseline(blob, seconds: float = 10.0):
    """The oracle decoder, as it stands, on all host cores over a bounded sample of the stream."""
    import oracle

    oracle.build()
    cores = os.cpu_count() or 1
    per = max(1, blob.ntiles // (4 * cores))
    ranges = [(t, min(t + per, blob.ntiles)) for t in range(0, blob.ntiles, per)]
    weights = 0
    t0 = time.time()
    passes = 0
    while True:
        weights += _oracle_threads(blob, ranges[: 2 * cores], cores, oracle.BF16)
        passes += 1
        if time.time() - t0 >= seconds:
            break
    dt = time.time() - t0
    # the same decoder on one thread, over a quarter of the time budget
    w1, p1 = 0, 0
    t1 = time.time()
    while True:
        w1 += _oracle_threads(blob, ranges[:1], 1, oracle.BF16)
        p1 += 1
        if time.time() - t1 >= seconds / 4:
            break
    dt1 = time.time() - t1
    return {"value": round(weights / dt / 1e9, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{passes} pass(es) over tiles 0..{ranges[min(2 * cores, len(ranges)) - 1][1]} of the "
                      f"{blob.ntiles}-tile stream ({weights / passes / 1e6:.1f} M weights per pass), "
                      f"{cores} threads, {dt:.1f} s",
            "single_thread": {"value": round(w1 / dt1 / 1e9, 5), "unit": UNIT,
                              "sample": f"{p1} pass(es) over tiles {ranges[0][0]}..{ranges[0][1]}, one thread, "
                                        f"{dt1:.1f} s"}}


def run_reference(args, world: int = 1):
    """The oracle as the reference arm: CPU decode, each step a bounded tile sample."""
    import oracle

    oracle.build()
    W = _make_weights()
    ob = oracle.encode(W, TARGET)
    blob = SimpleNamespace(payload=ob.payload, payload_words=ob.payload.size, tile_index=ob.tile_index,
                           freq_tables=ob.freq_tables, row_scales=ob.row_scales, rows=ob.rows, cols=ob.cols,
                           V=ob.V, ntiles=ob.ntiles)
    cores = os.cpu_count() or 1
    per = max(1, blob.ntiles // (4 * cores))
    ranges = [(t, min(t + per, blob.ntiles)) for t in range(0, blob.ntiles, per)][: 2 * cores]
    for _ in range(args.warmup):
        _oracle_threads(blob, ranges, cores, oracle.BF16)
    t0 = time.time()
    weights = 0
    for _ in range(args.steps):
        weights += _oracle_threads(blob, ranges, cores, oracle.BF16)
    dt = time.time() - t0
    value = weights / dt / 1e9
    sample = (f"tiles 0..{ranges[-1][1]} of the {blob.ntiles}-tile stream per step "
              f"({weights / args.steps / 1e6:.1f} M weights), {cores} threads")
    return {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": round(value / PAGES_GWPS, 6), "dtype": "u32+f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "target_bpp": TARGET, "out": "bf16"},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _timed_decodes(ep, db, dtype, out, runs: int = 15):
    """Min and median ms of `runs` decodes, each after an L2 flush (a 256 MiB write), timed with
    CUDA events on the launching stream after 3 warm-ups."""
    import torch

    st = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=out.device)
    for _ in range(3):
        ep.decode_tensor(db, dtype, out=out, stream=st)
    ts = []
    for _ in range(runs):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        ep.decode_tensor(db, dtype, out=out, stream=st)
        b.record(st)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    if ep.decode_status(st) != 0:
        raise RuntimeError("decode reported a corrupt stream")
    return min(ts), statistics.median(ts)


def _timed_matmul(rows: int, cols: int, tokens: int = 4096, runs: int = 15):
    """Min ms of a torch bf16 matmul X[tokens, cols] @ W[rows, cols]^T, same protocol."""
    import torch

    X = torch.randn(tokens, cols, dtype=torch.bfloat16, device="cuda")
    W = torch.randn(rows, cols, dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        torch.matmul(X, W.t())
    ts = []
    for _ in range(runs):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        torch.matmul(X, W.t())
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return min(ts)


def run_sweep(args):
    """Decode throughput on every workload: the headline's tile-size sweep, the attention
    projection (BF16, FP16), the FP8 / INT8 containers, the LLM-prefill rate sweep (with
    rel-L2), the DiT stack (one layer of every kind at every rate, against a bf16 matmul of the
    same shape with 4096 tokens, and the 30-block total from the per-layer rate allocation), and
    the oracle decoder on one and on all host cores.  Prints a markdown table and JSON lines."""
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build, synth
    from dit_weight_compression_ep_b200._lib import _torch_dtype

    build.build()
    peak, peak_kind = _peaks()
    out_bytes = {ep.BF16: 2, ep.FP16: 2, ep.FP8_E4M3: 1, ep.INT8: 1, ep.FP32: 4, ep.UINT8: 1}
    names = {ep.BF16: "bf16", ep.FP16: "fp16", ep.FP8_E4M3: "e4m3", ep.INT8: "int8", ep.FP32: "fp32", ep.UINT8: "uint8"}
    rows_out = []

    def case(label, blob, dtype, extra=None):
        db = ep.DeviceBlob(blob)
        out = torch.empty((blob.rows, blob.cols), dtype=_torch_dtype(dtype), device="cuda")
        tmin, tmed = _timed_decodes(ep, db, dtype, out)
        numel = blob.rows * blob.cols
        nbytes = blob.stored_device_bytes() + numel * out_bytes[dtype]
        r = {"case": label, "shape": f"{blob.rows}x{blob.cols}", "out": names[dtype], "stored_bpp":
             round(blob.stored_bpp, 3), "b": blob.b, "V": blob.V, "tiles": blob.ntiles,
             "us_min": round(tmin * 1e3, 2), "us_median": round(tmed * 1e3, 2),
             "gweights_s": round(numel / (tmin * 1e-3) / 1e9, 1), "gb_s": round(nbytes / (tmin * 1e-3) / 1e9, 1),
             "hbm_frac": round(nbytes / (tmin * 1e-3) / 1e9 / peak, 4)}
        if extra:
            r.update(extra(out))
        rows_out.append(r)
        print(json.dumps(r), flush=True)
        del db, out
        return r

    W = synth.generate(synth.headline())
    for V in (512, 910, 1820, 3640):
        case(f"headline 4 bpp, V={V}", ep.encode_tensor(W, 4.0, tile_vectors=V), ep.BF16)
    case("256x512 fp32 t5, 4 bpp, V=512, b=12", ep.encode_tensor(synth.generate(synth.small_fp32()), 4.0,
                                                                   tile_vectors=512, prob_bits=12), ep.BF16)
    blob = ep.encode_tensor(synth.generate(synth.dit_attn_proj()), 5.0)
    for dt in (ep.BF16, ep.FP16):
        case("DiT attention projection, 5 bpp", blob, dt)
    src = synth.generate(synth.lowp_source())
    for kind, dt in (("e4m3", ep.FP8_E4M3), ("int8", ep.INT8), ("uint8", ep.UINT8)):
        conv = {"e4m3": synth.to_e4m3_container, "int8": synth.to_int8_container, "uint8": synth.to_uint8_container}
        vals, _ = conv[kind](src)
        case(f"{kind} container, 5 bpp", ep.encode_tensor(vals, 5.0, has_container_scales=kind != "uint8"), dt)
    del src
    for wide in (True, False):
        W = synth.generate(synth.llm_prefill(wide))
        Wt = torch.from_numpy(W).cuda()
        nrm = float(torch.linalg.vector_norm(Wt))

        def rel_l2(out, Wt=Wt, nrm=nrm):
            return {"rel_l2": round(float(torch.linalg.vector_norm(out.float() - Wt)) / nrm, 5)}

        for bpp in (2, 3, 4, 5, 6, 7, 8):
            case(f"LLM prefill, {bpp} bpp", ep.encode_tensor(W, float(bpp)), ep.BF16, rel_l2)
        del Wt, W
        torch.cuda.empty_cache()
    # DiT stack: every kind at every rate (decode speed depends on shape and rate, not on the
    # block's seed), then the 30-block total from the per-layer rate allocation
    alloc = synth.dit_stack_bpp()
    per = {}
    for kind, (r_, c_) in synth.DIT_KINDS.items():
        Wk = synth.generate(synth.dit_stack_layer(0, kind))
        mm = _timed_matmul(r_, c_)
        for bpp in synth.DIT_BPP_CHOICES:
            r = case(f"DiT stack {kind}, {bpp} bpp", ep.encode_tensor(Wk, bpp), ep.BF16,
                     lambda out, mm=mm: {"matmul_4096_us": round(mm * 1e3, 2)})
            per[(kind, bpp)] = (r["us_min"], mm * 1e3)
    dec_total = sum(per[(k, bpp)][0] for (_, k), bpp in alloc.items())
    mm_total = sum(per[(k, bpp)][1] for (_, k), bpp in alloc.items())
    tot = {"case": "DiT stack, 30 blocks (sum over the allocation)", "decode_ms": round(dec_total / 1e3, 3),
           "matmul_4096_ms": round(mm_total / 1e3, 3), "decode_over_matmul": round(dec_total / mm_total, 4)}
    print(json.dumps(tot), flush=True)
    # the oracle decoder on the headline: one thread and all host cores, bounded samples
    import oracle

    oracle.build()
    blob = ep.encode_tensor(synth.generate(synth.headline()), 4.0)
    cores = os.cpu_count() or 1
    orc = {}
    for nth in (1, cores):
        per_t = max(1, blob.ntiles // (4 * nth))
        ranges = [(t, min(t + per_t, blob.ntiles)) for t in range(0, blob.ntiles, per_t)][: 2 * nth]
        t0 = time.time()
        wts = _oracle_threads(blob, ranges, nth, oracle.BF16)
        orc[nth] = wts / (time.time() - t0) / 1e9
    oc = {"case": "oracle decoder, headline sample", "gweights_s_1_thread": round(orc[1], 4),
          f"gweights_s_{cores}_threads": round(orc[cores], 4)}
    print(json.dumps(oc), flush=True)

    print("\n| case | shape | out | bpp | V | µs (min / median) | G w/s | GB/s | of HBM | extra |")
    print("|---|---|---|---|---|---|---|---|---|---|")
    for r in rows_out:
        extra = ", ".join(f"{k} {v}" for k, v in r.items() if k in ("rel_l2", "matmul_4096_us"))
        print(f"| {r['case']} | {r['shape']} | {r['out']} | {r['stored_bpp']} | {r['V']} | {r['us_min']} / "
              f"{r['us_median']} | {r['gweights_s']} | {r['gb_s']} | {100 * r['hbm_frac']:.1f} % | {extra} |")
    print(f"\nDiT stack total: decode {tot['decode_ms']} ms vs bf16 matmul (4096 tokens) {tot['matmul_4096_ms']} ms "
          f"= {100 * tot['decode_over_matmul']:.1f} %; oracle: {oc}; HBM peak {peak} GB/s ({peak_kind})")


def run_dit(args):
    """The whole 30-block DiT linear stack (150 layers at the per-layer rate allocation) decoded to
    bf16 three ways: one ep_decode_tensor per layer, one ep_decode_tensor_prepared per layer, and
    one ep_decode_batch per block (the block's five tensors in one launch); then the block-by-block
    sequence a denoising step runs (decode the block's weights, then its five bf16 matmuls with
    4096 tokens) against the matmuls alone.  Decode speed depends on a layer's shape and rate, not
    on its seed, so the 25 (kind, rate) streams are encoded once and every block uses its own
    combination of them.  Each figure: min and median of 5 timed passes of the whole stack (CUDA
    events around the pass, one stream, eager launches), after a warm-up pass."""
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build, synth

    build.build()
    peak, peak_kind = _peaks()
    dev = torch.device("cuda", 0)
    alloc = synth.dit_stack_bpp()
    kinds = list(synth.DIT_KINDS)
    nblocks = 1 + max(b for b, _ in alloc)
    streams = {}
    for kind in kinds:
        Wk = synth.generate(synth.dit_stack_layer(0, kind))
        for bpp in sorted({alloc[(b, kind)] for b in range(nblocks)}):
            blob = ep.encode_tensor(Wk, bpp)
            db = ep.DeviceBlob(blob, dev)
            streams[(kind, bpp)] = (blob, db, ep.prepare_lut(db))
        del Wk
    outs = {k: torch.empty(synth.DIT_KINDS[k], dtype=torch.bfloat16, device=dev) for k in kinds}
    blocks = [[(k, alloc[(b, k)]) for k in kinds] for b in range(nblocks)]
    batches = [ep.DecodeBatch([(streams[kb][1], streams[kb][2], outs[kb[0]]) for kb in blk], ep.BF16)
               for blk in blocks]
    numel = sum(streams[kb][0].rows * streams[kb][0].cols for blk in blocks for kb in blk)
    nbytes = sum(streams[kb][0].stored_device_bytes() + 2 * streams[kb][0].rows * streams[kb][0].cols
                 for blk in blocks for kb in blk)
    st = torch.cuda.current_stream(dev)
    X = {c: torch.randn(4096, c, dtype=torch.bfloat16, device=dev) for c in {synth.DIT_KINDS[k][1] for k in kinds}}

    def per_call():
        for blk in blocks:
            for kb in blk:
                ep.decode_tensor(streams[kb][1], ep.BF16, out=outs[kb[0]], stream=st)

    def prepared():
        for blk in blocks:
            for kb in blk:
                ep.decode_tensor_prepared(streams[kb][1], streams[kb][2], ep.BF16, out=outs[kb[0]], stream=st)

    def batched():
        for bt in batches:
            bt.run(stream=st)

    def matmuls_of(blk):
        for k, _ in blk:
            torch.matmul(X[synth.DIT_KINDS[k][1]], outs[k].t())

    def matmuls_only():
        for blk in blocks:
            matmuls_of(blk)

    def step_batched():
        for bt, blk in zip(batches, blocks):
            bt.run(stream=st)
            matmuls_of(blk)

    # the next block's weights decoded on a side stream while this block's matmuls run: two
    # output sets, block i decodes into set i % 2 once block i - 2's matmuls (the set's last
    # readers) are done
    outs_b = {k: torch.empty_like(o) for k, o in outs.items()}
    sets2 = (outs, outs_b)
    batches2 = [ep.DecodeBatch([(streams[kb][1], streams[kb][2], sets2[i % 2][kb[0]]) for kb in blk], ep.BF16)
                for i, blk in enumerate(blocks)]
    s_dec = torch.cuda.Stream(dev)

    def step_pipelined():
        ev_dec = [torch.cuda.Event() for _ in blocks]
        ev_mm = [torch.cuda.Event() for _ in blocks]
        s_dec.wait_stream(st)
        for i in range(len(blocks) + 1):
            if i < len(blocks):
                if i >= 2:
                    s_dec.wait_event(ev_mm[i - 2])
                batches2[i].run(stream=s_dec)
                ev_dec[i].record(s_dec)
            j = i - 1  # the matmuls of the block decoded one step earlier
            if j >= 0:
                st.wait_event(ev_dec[j])
                for k, _ in blocks[j]:
                    torch.matmul(X[synth.DIT_KINDS[k][1]], sets2[j % 2][k].t())
                ev_mm[j].record(st)
        st.wait_stream(s_dec)

    def step_per_call():
        for blk in blocks:
            for kb in blk:
                ep.decode_tensor(streams[kb][1], ep.BF16, out=outs[kb[0]], stream=st)
            matmuls_of(blk)

    def timed(fn, passes=5):
        fn()
        torch.cuda.synchronize(dev)
        ts = []
        for _ in range(passes):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b))
        if ep.decode_status(st) != 0:
            raise RuntimeError("decode reported a corrupt stream")
        return round(min(ts), 3), round(statistics.median(ts), 3)

    # the three decodes give the same bits
    batched()
    ref = {k: o.clone() for k, o in outs.items()}
    prepared()
    torch.cuda.synchronize(dev)
    if ep.decode_status(st) != 0 or not all(torch.equal(ref[k].view(torch.int16), outs[k].view(torch.int16))
                                            for k in kinds):
        raise RuntimeError("batched and prepared decodes differ")
    # several blocks' weights in one launch (each block into its own output set): more tiles per
    # launch, so the sub-partitions' loads even out
    multi = {}
    for n in (2, 3, 6):
        sets = [outs] + [{k: torch.empty_like(o) for k, o in outs.items()} for _ in range(n - 1)]
        groups = [blocks[i:i + n] for i in range(0, len(blocks), n)]
        multi[n] = [ep.DecodeBatch([(streams[kb][1], streams[kb][2], sets[j][kb[0]])
                                    for j, blk in enumerate(g) for kb in blk], ep.BF16) for g in groups]
    res = {"case": f"DiT linear stack, {nblocks} blocks x {len(kinds)} layers, per-layer rates {synth.DIT_BPP_CHOICES}",
           "weights": numel, "algorithmic_bytes": nbytes, "hbm_peak_gbs": peak, "peak_kind": peak_kind}
    for n, gb in multi.items():
        tmin, tmed = timed(lambda gb=gb: [b.run(stream=st) for b in gb])
        res[f"batches_of_{n}_blocks_ms"] = [tmin, tmed]
        res[f"batches_of_{n}_blocks_gweights_s"] = round(numel / (tmin * 1e-3) / 1e9, 1)
        res[f"batches_of_{n}_blocks_hbm_frac"] = round(nbytes / (tmin * 1e-3) / 1e9 / peak, 4)
        print(json.dumps({f"batches_of_{n}_blocks": [tmin, tmed]}), flush=True)
    del multi
    for name, fn in (("per_layer_decode", per_call), ("per_layer_prepared", prepared), ("block_batches", batched),
                     ("matmuls_only_4096", matmuls_only), ("step_block_batches_then_matmuls", step_batched),
                     ("step_block_batches_pipelined", step_pipelined),
                     ("step_per_layer_decode_then_matmuls", step_per_call)):
        tmin, tmed = timed(fn)
        res[name + "_ms"] = [tmin, tmed]
        print(json.dumps({name: [tmin, tmed]}), flush=True)
    for name in ("per_layer_decode", "per_layer_prepared", "block_batches"):
        t = res[name + "_ms"][0] * 1e-3
        res[name + "_gweights_s"] = round(numel / t / 1e9, 1)
        res[name + "_hbm_frac"] = round(nbytes / t / 1e9 / peak, 4)
    mm = res["matmuls_only_4096_ms"][0]
    res["step_overhead_block_batches"] = round(res["step_block_batches_then_matmuls_ms"][0] / mm - 1, 4)
    res["step_overhead_per_layer"] = round(res["step_per_layer_decode_then_matmuls_ms"][0] / mm - 1, 4)
    res["step_overhead_pipelined"] = round(res["step_block_batches_pipelined_ms"][0] / mm - 1, 4)
    print(json.dumps(res), flush=True)


def run_encode(args):
    """Conversion speed: the 3840x10240 headline at 4 bpp through the CPU packer (all host
    threads) and the GPU encoder (weights already on the GPU, blob returned in host memory; the
    two blobs are checked identical), and from bf16 weights on the GPU into a device blob; then
    the whole DiT stack (150 layers at the per-layer rates) through the GPU encoder, each layer's
    float32 weights copied from pinned host memory inside the timed loop, and from resident bf16
    weights into device blobs.  Wall-clock times (the encoder synchronises its stream)."""
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build, synth

    build.build()
    W = synth.generate(synth.headline())
    Wd = torch.from_numpy(W).cuda()
    cpu_t, gpu_t = [], []
    for _ in range(3):
        t0 = time.time()
        cb = ep.encode_tensor(W, 4.0)
        cpu_t.append(time.time() - t0)
    ep.encode_tensor_gpu(Wd, 4.0)  # warm-up (module load, first allocations)
    for _ in range(5):
        torch.cuda.synchronize()
        t0 = time.time()
        gb = ep.encode_tensor_gpu(Wd, 4.0)
        gpu_t.append(time.time() - t0)
    same = (np.array_equal(gb.payload, cb.payload) and np.array_equal(gb.tile_index, cb.tile_index) and
            np.array_equal(gb.freq_tables, cb.freq_tables) and
            np.array_equal(gb.row_scales.view(np.uint32), cb.row_scales.view(np.uint32)))
    # load-time compression: bf16 weights already on the GPU, the stream left there
    Wb = Wd.to(torch.bfloat16)
    dev_t = []
    ep.encode_tensor_gpu_to_device(Wb, 4.0)
    for _ in range(5):
        torch.cuda.synchronize()
        t0 = time.time()
        ep.encode_tensor_gpu_to_device(Wb, 4.0)
        dev_t.append(time.time() - t0)
    res = {"case": "encode 3840x10240 at 4 bpp", "cpu_packer_s": round(min(cpu_t), 4),
           "cpu_threads": os.cpu_count(), "gpu_encoder_s": round(min(gpu_t), 4), "identical_blobs": same,
           "gpu_encoder_bf16_to_device_s": round(min(dev_t), 4),
           "pages_gpu_ms_per_39m_layer": "11-36 (their GPU, context)"}
    print(json.dumps(res), flush=True)
    # the per-row refinement (App. C.2), K = 4 candidates, one sweep, at 3 bpp
    t0 = time.time()
    cr = ep.encode_tensor(W, 3.0, rdo_candidates=4)
    cpu_rdo = time.time() - t0
    ep.encode_tensor_gpu(Wd, 3.0, rdo_candidates=4)
    torch.cuda.synchronize()
    t0 = time.time()
    gr = ep.encode_tensor_gpu(Wd, 3.0, rdo_candidates=4)
    gpu_rdo = time.time() - t0
    print(json.dumps({"case": "encode 3840x10240 at 3 bpp with the per-row refinement (K = 4, one sweep)",
                      "cpu_packer_s": round(cpu_rdo, 3), "gpu_encoder_s": round(gpu_rdo, 4),
                      "identical_blobs": bool(np.array_equal(gr.payload, cr.payload) and
                                              np.array_equal(gr.tile_index, cr.tile_index) and
                                              np.array_equal(gr.row_scales.view(np.uint32),
                                                             cr.row_scales.view(np.uint32)))}), flush=True)
    del Wd, Wb
    alloc = synth.dit_stack_bpp()
    kinds = list(synth.DIT_KINDS)
    host = {k: torch.from_numpy(synth.generate(synth.dit_stack_layer(0, k))).pin_memory() for k in kinds}
    dev = {k: torch.empty(host[k].shape, dtype=torch.float32, device="cuda") for k in kinds}
    order = sorted(alloc.items())
    for k in kinds:  # warm-up
        dev[k].copy_(host[k])
    torch.cuda.synchronize()
    t0 = time.time()
    nweights, nbytes = 0, 0
    for (_, k), bpp in order:
        dev[k].copy_(host[k], non_blocking=True)
        b = ep.encode_tensor_gpu(dev[k], bpp)
        nweights += b.rows * b.cols
        nbytes += b.stored_bytes
    tot = time.time() - t0
    # the same stack compressed at load: bf16 weights resident, device blobs out
    devb = {k: dev[k].to(torch.bfloat16) for k in kinds}
    del dev
    torch.cuda.synchronize()
    t0 = time.time()
    for (_, k), bpp in order:
        ep.encode_tensor_gpu_to_device(devb[k], bpp)
    tot_dev = time.time() - t0
    res2 = {"case": "encode the DiT stack (150 layers, per-layer rates) on the GPU", "seconds": round(tot, 3),
            "layers": len(order), "weights": nweights, "stored_bytes": nbytes,
            "stored_bpp": round(8.0 * nbytes / nweights, 4),
            "seconds_bf16_resident_to_device": round(tot_dev, 3),
            "pages_whole_model_s": "3.5 (their GPU, context)"}
    print(json.dumps(res2), flush=True)


def run_linear(args):
    """A linear layer whose weight is stored compressed (CompressedLinear: decode with the library's
    prepared table, then the library GEMM, cuBLAS through torch), against the same GEMM with the
    weight resident (BF16 X @ W^T; FP8-e4m3 `_scaled_mm` with per-row weight scales; INT8 `_int_mm`
    with the per-token and per-row scales).  The
    3840x10240 layer at 4 bpp, tokens 256 .. 16384; each time is the minimum of 15 runs, each
    after a 256 MiB L2 flush.  Prints a markdown table and JSON lines."""
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build, synth

    build.build()
    dev = torch.device("cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def tmin(fn, runs=15):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(runs):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return min(ts) * 1e3

    W = synth.generate(synth.headline())
    rows, cols = W.shape
    routes = []
    # BF16
    blob = ep.encode_tensor(W, TARGET)
    db = ep.DeviceBlob(blob)
    Wb = torch.from_numpy(W).to(dev).to(torch.bfloat16)
    Wd = torch.empty_like(Wb)
    routes.append(("bf16", db, ep.BF16, Wb, Wd))
    # FP8-e4m3 container, per-row scales
    vals, wsc = synth.to_e4m3_container(W)
    blob8 = ep.encode_tensor(vals, TARGET, has_container_scales=True)
    W8 = torch.from_numpy(vals).to(dev).to(torch.float8_e4m3fn)
    routes.append(("fp8 e4m3", ep.DeviceBlob(blob8), ep.FP8_E4M3, W8, torch.empty_like(W8)))
    wscale = torch.from_numpy(wsc).to(dev).view(1, -1)
    # INT8 container, per-row scales
    vali, wsci = synth.to_int8_container(W)
    wscale_i = torch.from_numpy(wsci).to(dev).view(1, -1)
    blobi = ep.encode_tensor(vali, TARGET, has_container_scales=True)
    Wi = torch.from_numpy(vali).to(dev).to(torch.int8)
    routes.append(("int8", ep.DeviceBlob(blobi), ep.INT8, Wi, torch.empty_like(Wi)))
    out = []
    for tokens in (256, 1024, 4096, 16384):
        X = (torch.randn(tokens, cols, device=dev) * 0.5)
        Xb = X.to(torch.bfloat16)
        X8 = X.clamp(-448, 448).to(torch.float8_e4m3fn)
        Xi = X.mul(20).round().clamp(-127, 127).to(torch.int8)
        xs = torch.ones(tokens, 1, device=dev)
        for name, dbr, dt, Wres, Wdec in routes:
            # the resident side runs the same GEMM (and scaling) as CompressedLinear's route
            if name == "bf16":
                lin = ep.CompressedLinear(dbr, "bf16", scratch=Wdec)
                gemm = lambda Wm: torch.matmul(Xb, Wm.t())
                call = lambda lin=lin: lin(Xb)
            elif name == "fp8 e4m3":
                lin = ep.CompressedLinear(dbr, "fp8", weight_scales=wscale, scratch=Wdec)
                gemm = lambda Wm: torch._scaled_mm(X8, Wm.t(), scale_a=xs, scale_b=wscale, out_dtype=torch.bfloat16)
                call = lambda lin=lin: lin(X8, xs)
            else:
                lin = ep.CompressedLinear(dbr, "int8", weight_scales=wscale_i, scratch=Wdec)
                gemm = lambda Wm: (torch._int_mm(Xi, Wm.t()).float() * xs * wscale_i).to(torch.bfloat16)
                call = lambda lin=lin: lin(Xi, xs)
            try:
                t_res = tmin(lambda: gemm(Wres))
            except Exception as exc:  # a route torch's GEMMs do not offer on this device
                print(json.dumps({"route": name, "tokens": tokens, "unavailable": str(exc)[:160]}), flush=True)
                continue
            t_dec = tmin(lambda lin=lin: lin.decoded_weight())
            t_both = tmin(call)
            r = {"route": name, "tokens": tokens, "gemm_resident_us": round(t_res, 2), "decode_us": round(t_dec, 2),
                 "decode_then_gemm_us": round(t_both, 2), "overhead": round(t_both / t_res - 1.0, 4)}
            out.append(r)
            print(json.dumps(r), flush=True)
        if ep.decode_status() != 0:
            raise RuntimeError("decode reported a corrupt stream")
    print("\n| route | tokens | GEMM, weight resident (µs) | decode (µs) | decode then GEMM (µs) | overhead |")
    print("|---|---|---|---|---|---|")
    for r in out:
        print(f"| {r['route']} | {r['tokens']} | {r['gemm_resident_us']} | {r['decode_us']} | {r['decode_then_gemm_us']} | "
              f"{100 * r['overhead']:.1f} % |")


def run_gemv(args):
    """A linear layer on 1, 2, 4 and 8 tokens whose weight is decoded inside the product
    (ep_decode_gemv, prepared table and per call), against decoding the weight to BF16 with the
    prepared table and then the GEMM (cuBLAS through torch), and against the GEMM on a resident BF16
    weight.  The 3840x10240 layer at 4 bpp; each time is the minimum of 15 runs, each after a
    256 MiB L2 flush.  Prints JSON lines and a markdown table."""
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build, synth

    build.build()
    dev = torch.device("cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def tmin(fn, runs=15):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(runs):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return min(ts) * 1e3

    W = synth.generate(synth.headline())
    rows, cols = W.shape
    blob = ep.encode_tensor(W, TARGET)
    db = ep.DeviceBlob(blob)
    lut = ep.prepare_lut(db)
    Wb = torch.from_numpy(W).to(dev).to(torch.bfloat16)
    Wd = torch.empty_like(Wb)
    stream_bytes = blob.stored_device_bytes()
    out = []
    for ntok in ep.GEMV_TOKENS:
        xb = (torch.randn(ntok, cols, device=dev) * 0.5).to(torch.bfloat16)
        y = torch.empty(ntok, rows, device=dev)
        t_res = tmin(lambda: torch.matmul(xb, Wb.t()))
        t_fused = tmin(lambda: ep.decode_gemv(db, xb, lut=lut, y=y))
        t_fused_call = tmin(lambda: ep.decode_gemv(db, xb, y=y))
        t_dec = tmin(lambda: ep.decode_tensor_prepared(db, lut, ep.BF16, out=Wd))
        t_both = tmin(lambda: torch.matmul(xb, ep.decode_tensor_prepared(db, lut, ep.BF16, out=Wd).t()))
        if ep.decode_status() != 0:
            raise RuntimeError("decode reported a corrupt stream")
        r = {"tokens": ntok, "gemv_resident_bf16_us": round(t_res, 2), "fused_prepared_us": round(t_fused, 2),
             "fused_per_call_us": round(t_fused_call, 2), "decode_prepared_us": round(t_dec, 2),
             "decode_then_gemm_us": round(t_both, 2), "fused_vs_decode_then_gemm": round(t_both / t_fused, 3),
             "fused_hbm_gbs": round((stream_bytes + xb.nbytes + y.nbytes) / (t_fused * 1e-6) / 1e9, 1)}
        out.append(r)
        print(json.dumps(r), flush=True)
    print("\n| tokens | GEMV, BF16 weight resident (µs) | fused decode-GEMV, prepared (µs) | fused, per call (µs) | "
          "decode (µs) | decode then GEMM (µs) | decode then GEMM / fused |")
    print("|---|---|---|---|---|---|---|")
    for r in out:
        print(f"| {r['tokens']} | {r['gemv_resident_bf16_us']} | {r['fused_prepared_us']} | {r['fused_per_call_us']} | "
              f"{r['decode_prepared_us']} | {r['decode_then_gemm_us']} | {r['fused_vs_decode_then_gemm']} |")


def run_split(args):
    """The decode on part of the GPU beside the GEMM: 16 consecutive 3840x10240 layers at 4 bpp,
    the next layer's weight decoded on s SMs (a one-tensor batch from ep_batch_create_on) on a
    second stream while the current layer's bf16 GEMM runs on the main stream, two output buffers.
    Against decode then GEMM on one stream, for 256, 1,024 and 4,096 tokens.  Each figure is the
    minimum of 5 passes over the 16 layers, each pass after a 256 MiB L2 flush, in µs per layer."""
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build, synth

    build.build()
    dev = torch.device("cuda")
    st = torch.cuda.current_stream()
    s_dec = torch.cuda.Stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    nl = 16

    def per_layer(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return round(min(ts) * 1e3 / nl, 1)

    W = synth.generate(synth.headline())
    rows, cols = W.shape
    db = ep.DeviceBlob(ep.encode_tensor(W, TARGET))
    lut = ep.prepare_lut(db)
    bufs = [torch.empty(rows, cols, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    splits = [s for s in (32, 64, 100, nsm) if s <= nsm]
    out = []
    for tokens in (256, 1024, 4096):
        X = torch.randn(tokens, cols, dtype=torch.bfloat16, device=dev)

        def seq():
            for i in range(nl):
                ep.decode_tensor_prepared(db, lut, ep.BF16, out=bufs[i % 2], stream=st)
                torch.matmul(X, bufs[i % 2].t())

        def gemm():
            for i in range(nl):
                torch.matmul(X, bufs[i % 2].t())

        r = {"tokens": tokens, "decode_then_gemm_us": per_layer(seq), "gemm_us": per_layer(gemm)}
        for s in splits:
            bs = [ep.DecodeBatch([(db, lut, bufs[k])], ep.BF16, num_ctas=s) for k in range(2)]

            def dec():
                for i in range(nl):
                    bs[i % 2].run(stream=st)

            def pipe():
                ev_dec = [torch.cuda.Event() for _ in range(nl)]
                ev_mm = [torch.cuda.Event() for _ in range(nl)]
                s_dec.wait_stream(st)
                for i in range(nl + 1):
                    if i < nl:
                        if i >= 2:
                            s_dec.wait_event(ev_mm[i - 2])  # the GEMM that last read this buffer
                        bs[i % 2].run(stream=s_dec)
                        ev_dec[i].record(s_dec)
                    j = i - 1
                    if j >= 0:
                        st.wait_event(ev_dec[j])
                        torch.matmul(X, bufs[j % 2].t())
                        ev_mm[j].record(st)
                st.wait_stream(s_dec)

            r[f"decode_on_{s}_us"] = per_layer(dec)
            r[f"pipelined_{s}_us"] = per_layer(pipe)
        if ep.decode_status() != 0:
            raise RuntimeError("decode reported a corrupt stream")
        out.append(r)
        print(json.dumps(r), flush=True)
    head = " | ".join([f"decode on {s}" for s in splits] + [f"pipelined, s = {s}" for s in splits])
    print(f"\n| tokens | decode then GEMM, one stream | GEMM alone | {head} |")
    print("|---" * (3 + 2 * len(splits)) + "|")
    for r in out:
        cells = [r[f"decode_on_{s}_us"] for s in splits] + [r[f"pipelined_{s}_us"] for s in splits]
        print(f"| {r['tokens']} | {r['decode_then_gemm_us']} | {r['gemm_us']} | " + " | ".join(map(str, cells)) + " |")


PROBE_CHAINS = [
    ("imad", "mad.lo.u32 (state update, addresses)"),
    ("lds32+imad", "32-bit shared load (lookup-table entry) + its address multiply-add"),
    ("lds16+imad", "16-bit shared load (payload word) + its address multiply-add"),
    ("vote+imad", "and + compare + vote.ballot, folded back with a multiply-add"),
    ("popc+imad", "popc, folded back with a multiply-add"),
    ("shfl", "shift + shfl.idx (source lane from the value)"),
    ("vote+and+popc+imad", "the renormalisation's word index"),
    ("vote+and+popc+imad+lds16", "the word index, then the word's shared load"),
    ("vote+and+popc+shfl+add", "the word index, then a shuffle instead of the address and load"),
    ("redux+imad", "redux.sync.add, folded back with a multiply-add"),
]


def run_chain(args):
    """The decode's chain latency and fixed cost: tensors of exactly one tile per SM (so one
    warp per SM, nothing to hide a step's latency behind), at four tile sizes; a straight line
    through (steps per tile, time) gives the fixed cost per call and the cycles per symbol step
    at the sampled SM clock.  Also times the 3840x10240 headline the same way (eager launches,
    four rotating copies).  Prints one JSON line."""
    import numpy as np
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build

    build.build()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rng = np.random.default_rng(0)

    def timed(db, outs, n):
        for i in range(5):
            ep.decode_tensor(db, ep.BF16, out=outs[i % len(outs)])
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(n):
            ep.decode_tensor(db, ep.BF16, out=outs[i % len(outs)])
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n * 1e3

    pts = []
    for V in (320, 640, 1280, 2560):
        W = (rng.standard_t(6, (sms * V // 128, 1024)) * 0.02).astype(np.float32)
        blob = ep.encode_tensor(W, TARGET, tile_vectors=V, prob_bits=11)
        assert blob.ntiles == sms
        db = ep.DeviceBlob(blob)
        outs = [torch.empty((blob.rows, blob.cols), dtype=torch.bfloat16, device="cuda")]
        pts.append((9 * ((V + 31) // 32), timed(db, outs, 30)))
    A = np.array([[1.0, s] for s, _ in pts])
    (fixed, per), *_ = np.linalg.lstsq(A, np.array([u for _, u in pts]), rcond=None)
    mhz = torch.cuda.clock_rate() if hasattr(torch.cuda, "clock_rate") else None
    hb = ep.encode_tensor(_make_weights(), TARGET)
    hdb = ep.DeviceBlob(hb)
    houts = [torch.empty((hb.rows, hb.cols), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    head = timed(hdb, houts, 50)
    print(json.dumps({"chain": {"fixed_us": round(float(fixed), 2), "us_per_step": round(float(per), 5),
                                "cycles_per_step_at_1965_mhz": round(float(per) * 1965, 1),
                                "points_steps_us": [(s, round(u, 2)) for s, u in pts], "sm_clock_query_mhz": mhz},
                      "headline_eager_us": round(head, 2)}), flush=True)


def run_knee(args):
    """Cycles per symbol step against the number of tiles each warp scheduler holds: for k = 1 ..
    6 (24 warps a CTA: 6 per sub-partition), tensors of exactly 4 k tiles per SM (k warps on each
    of its four sub-partitions, one tile each) at three tile sizes, with the packed b = 11 table
    and (k = 1, 3, 6) the two-level b = 12 one; the slope of time over steps per tile is the time per step with k
    chains interleaved on a sub-partition.  Against k x (warp instructions per step), it shows
    where the decode turns from chain-bound to issue-bound.  Eager launches, 4 rotating outputs,
    the SM clock taken as 1,965 MHz (the bench line records the clock it saw).  Prints JSON lines
    and a markdown table."""
    import numpy as np
    import torch

    import dit_weight_compression_ep_b200 as ep
    from dit_weight_compression_ep_b200 import build

    build.build()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rng = np.random.default_rng(0)

    def timed(db, outs, n=20):
        for i in range(4):
            ep.decode_tensor_prepared(db, lut, ep.BF16, out=outs[i % len(outs)])
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(n):
            ep.decode_tensor_prepared(db, lut, ep.BF16, out=outs[i % len(outs)])
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n * 1e3

    rows_out = []
    for b, k in [(11, k) for k in (1, 2, 3, 4, 5, 6)] + [(12, k) for k in (1, 3, 6)]:
        pts = []
        for V in (640, 1280, 2560):
            tiles = 4 * k * sms
            W = (rng.standard_t(6, (tiles * V // 128, 1024)) * 0.02).astype(np.float32)
            blob = ep.encode_tensor(W, TARGET, tile_vectors=V, prob_bits=b)
            assert blob.ntiles == tiles and blob.b == b
            db = ep.DeviceBlob(blob)
            lut = ep.prepare_lut(db)
            outs = [torch.empty((blob.rows, blob.cols), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
            pts.append((9 * ((V + 31) // 32), timed(db, outs)))
        A = np.array([[1.0, st] for st, _ in pts])
        (fixed, per), *_ = np.linalg.lstsq(A, np.array([u for _, u in pts]), rcond=None)
        r = {"b": b, "tiles_per_sub_partition": k, "cycles_per_step": round(float(per) * 1965, 1),
             "fixed_us": round(float(fixed), 2), "points_steps_us": [(st, round(u, 2)) for st, u in pts]}
        rows_out.append(r)
        print(json.dumps(r), flush=True)
        if ep.decode_status() != 0:
            raise RuntimeError("decode reported a corrupt stream")
    print("\n| b | tiles per sub-partition | cycles per symbol step | cycles per step per tile | fixed cost (µs) |")
    print("|---|---|---|---|---|")
    for r in rows_out:
        print(f"| {r['b']} | {r['tiles_per_sub_partition']} | {r['cycles_per_step']} | "
              f"{r['cycles_per_step'] / r['tiles_per_sub_partition']:.1f} | {r['fixed_us']} |")


def run_latency(args):
    """Latencies of the operations on the decode step's dependent chain on this GPU: one warp,
    dependent chains timed with clock64 (csrc/latency_probe.cu).  Prints a table and one JSON
    line; the single operations follow by subtracting the multiply-add chain."""
    import ctypes as C

    from dit_weight_compression_ep_b200 import build

    L = C.CDLL(build.build_probe())
    L.ep_probe_latencies.argtypes = [C.POINTER(C.c_double), C.c_int]
    L.ep_probe_latencies.restype = C.c_int
    out = (C.c_double * len(PROBE_CHAINS))()
    rc = L.ep_probe_latencies(out, len(PROBE_CHAINS))
    if rc:
        raise SystemExit(f"latency probe failed: CUDA error {rc}")
    cyc = {name: round(out[k], 1) for k, (name, _) in enumerate(PROBE_CHAINS)}
    imad = cyc["imad"]
    print("| chain | cycles per iteration |\n|---|---|")
    for name, what in PROBE_CHAINS:
        print(f"| {what} | {cyc[name]} |")
    derived = {"imad": imad, "lds32": round(cyc["lds32+imad"] - imad, 1), "lds16": round(cyc["lds16+imad"] - imad, 1),
               "popc": round(cyc["popc+imad"] - imad, 1), "vote_with_and_setp": round(cyc["vote+imad"] - imad, 1),
               "redux": round(cyc["redux+imad"] - imad, 1)}
    print(json.dumps({"latency_cycles": cyc, "derived": derived}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--sweep", action="store_true", help="every workload's decode throughput (one GPU)")
    ap.add_argument("--linear", action="store_true", help="decode-then-GEMM against a resident weight (one GPU)")
    ap.add_argument("--split", action="store_true", help="the decode on part of the GPU beside the GEMM (one GPU)")
    ap.add_argument("--gemv", action="store_true", help="the fused decode-GEMV on 1 to 8 tokens (one GPU)")
    ap.add_argument("--dit", action="store_true", help="the whole DiT stack: per layer, prepared, block batches")
    ap.add_argument("--encode", action="store_true", help="conversion speed: CPU packer and GPU encoder")
    ap.add_argument("--latency", action="store_true", help="latencies of the decode step's operations (one GPU)")
    ap.add_argument("--knee", action="store_true", help="cycles per step against tiles per sub-partition (one GPU)")
    ap.add_argument("--chain", action="store_true", help="decode chain latency and fixed cost per call (one GPU)")
    ap.add_argument("--workload", choices=["headline", *OTHER_WORKLOADS], default="headline",
                    help="time another workload with the default protocol (a measurement, not the benchmark)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    one_gpu_mode = (args.sweep or args.linear or args.split or args.gemv or args.dit or args.encode or args.latency
                    or args.chain or args.knee)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and not one_gpu_mode:
        # no launcher: start the N ranks here (one process per GPU) and pass on their status
        sys.exit(relaunch(args.gpus, os.path.abspath(__file__), sys.argv[1:]).returncode)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if not one_gpu_mode and world != args.gpus:
        ap.error(f"--gpus {args.gpus}, but the launcher started {world} rank(s)")

    if args.sweep:
        run_sweep(args)
        return
    if args.linear:
        run_linear(args)
        return
    if args.split:
        run_split(args)
        return
    if args.gemv:
        run_gemv(args)
        return
    if args.dit:
        run_dit(args)
        return
    if args.encode:
        run_encode(args)
        return
    if args.latency:
        run_latency(args)
        return
    if args.chain:
        run_chain(args)
        return
    if args.knee:
        run_knee(args)
        return
    if args.impl == "reference":
        if args.workload != "headline":
            ap.error("the reference arm runs the headline workload only")
        if rank != 0:
            return
        res = run_reference(args, world)
        print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
        if dist.get_world_size() != args.gpus:  # the ranks NCCL sees are the GPUs the line reports
            raise SystemExit(f"NCCL sees {dist.get_world_size()} ranks, --gpus {args.gpus}")
    try:
        res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
