#!/usr/bin/env python
"""Benchmark of the quantized linear layer on B200 (one JSON line on rank 0).

Headline workload: the per-token W8A8 GEMM, x int8 [4096,4096] x weight int8
[4096,4096] (nn.Linear layout) with per-token and per-channel fp32 scales,
bf16 out; metric int8-equivalent TOPS (2 ops per multiply-add).  One step is
one call of bq_gemm_i8_pertoken (one kernel launch) on inputs resident in
HBM; K steps are captured in one CUDA graph that cycles through 8 copies of
the inputs (268 MB, larger than the 126 MB L2) and timed with CUDA events on
the launching stream.  `e2e` times the same call through the Python API with
pinned host buffers, the host->device copies of every step's inputs and the
device->host copy of its output inside the timed region (consecutive steps
pipelined on three streams).

The other workloads of the benchmark set (BitLinear decode and prefill,
grouped INT4 decode, the tiny BitLinear) are timed the same way and reported
under "workloads", each against its own roofline.

Multi-GPU: every rank runs an independent replica (the layer needs no
exchange); the time is the max over ranks and `value` sums the work of all
ranks.  `--impl reference` times the oracle (plain C, row-parallel threads on
all host cores) on a bounded sample of the same workload instead.

`cpu_baseline` times the oracle, as it stands, on all host cores for every
workload of the set (threads split the output rows; each thread runs the
plain scalar oracle on its rows), on bounded row samples.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "int8-equiv TOPS (prefill) and weight GB/s (decode) vs B200 roofline"
HEAD = dict(M=4096, N=4096, K=4096)
HEAD_WORKLOAD = "per-token W8A8 GEMM: x int8 [4096,4096] x w int8 [4096,4096] (N,K), fp32 deqScale/perTokenScale, bf16 out"
L2_COPIES = 8

# DRAM traffic of one launch of the headline kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the hash of the
# kernel source it was taken on; stale once the source changes.  The capture
# flushes caches before the launch, not after it, so bf16 output still held in
# L2 when the kernel ends is not counted as written.
NCU_TRAFFIC = {
    # the ncu capture of the 4096^3 launch: 33.619712 MB read + 1.859840 MB written
    ("gemm_w8a8_4096", "d24aae2d5c2fdb35"): 35479552,
}
CPU_BUDGET_S = 4.0  # oracle wall time per workload in the CPU baseline


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10000)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-workloads", action="store_true", help="skip the secondary workloads")
    p.add_argument("--workloads", default="decode,w4,prefill,tiny,batched,w4a4,layernorm,conv,backward",
                   help="comma list of secondary workloads: decode, w4, prefill, tiny, batched, w4a4, layernorm, "
                        "conv, backward")
    p.add_argument("--workload-steps", type=int, default=200)
    p.add_argument("--decode-ms", default="1,4,16", help="token counts of the BitLinear decode workload")
    p.add_argument("--w4-ms", default="1,32", help="token counts of the grouped INT4 workload")
    p.add_argument("--no-head", action="store_true", help="skip the headline GEMM (profiling runs only)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=0, help="oracle sample rows of the headline (0 = calibrate)")
    p.add_argument("--cpu-budget", type=float, default=CPU_BUDGET_S, help="oracle seconds per workload")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "bit_quantized_linear_rmsnorm_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def gpu_id(device: int) -> str:
    """nvidia-smi -i argument naming the physical GPU behind torch device
    `device` (its PCI bus id; torch's index is relative to CUDA_VISIBLE_DEVICES)."""
    import torch
    props = torch.cuda.get_device_properties(device)
    dom, bus, dv = (getattr(props, a, None) for a in ("pci_domain_id", "pci_bus_id", "pci_device_id"))
    if None not in (dom, bus, dv):
        return f"{dom:08X}:{bus:02X}:{dv:02X}.0"
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    if vis:
        entries = [e.strip() for e in vis.split(",") if e.strip()]
        if device < len(entries):
            return entries[device]
    return str(device)


class Clocks:
    """SM clock, power and clock-event reasons of the GPU, sampled every few
    milliseconds (NVML, read-only queries) from a background thread while the
    warm-up replays and the timed region run; nvidia-smi at 200 ms where NVML
    is unavailable.  Every sample is taken under load (back-to-back replays)."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, device: int, period_s: float = 0.002):
        self.device = device
        self.period = period_s
        self.samples = []  # (t, sm_mhz, max_mhz, reason bits)
        self.marks = {}
        self._stop = None
        self._thread = None
        self._smi = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        gid = gpu_id(self.device)
        if ":" in gid:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(gid)
        if gid.startswith("GPU-"):
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(gid)
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(gid))

    def __enter__(self):
        import threading
        self.samples = []
        try:
            nv, h = self._handle()
        except Exception:
            nv = None
        if nv is None:
            try:
                self._smi = subprocess.Popen(
                    ["nvidia-smi", "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                     "--format=csv,noheader,nounits", "-i", gpu_id(self.device), "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self._smi = None
            return self
        self._stop = threading.Event()
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

        def run():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.perf_counter(), float(sm), float(mx), int(rs)))
                except Exception:
                    pass
                time.sleep(self.period)
        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def mark(self, name: str):
        self.marks[name] = time.perf_counter()

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._smi is not None:
            self._smi.terminate()
            try:
                out, _ = self._smi.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._smi.kill()
                out, _ = self._smi.communicate()
            now = time.perf_counter()
            for ln in out.splitlines():
                parts = [x.strip() for x in ln.split(",")]
                try:
                    self.samples.append((now, float(parts[0]), float(parts[1]), int(parts[2], 16)))
                except (ValueError, IndexError):
                    continue
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [x[1] for x in self.samples]
        bits = 0
        for x in self.samples:
            bits |= x[3]
        t0, t1 = self.marks.get("timed_start"), self.marks.get("timed_end")
        inside = [x[1] for x in self.samples if t0 is not None and t1 is not None and t0 <= x[0] <= t1]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[2] for x in self.samples),
                "reasons": sorted(n for n, b in self.REASONS if bits & b), "samples": len(sm),
                "samples_in_timed_region": len(inside),
                "sm_mhz_in_timed_region": statistics.median(inside) if inside else None,
                "source": "nvml" if self._smi is None else "nvidia-smi"}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class Dist:
    """Replica plumbing: a barrier and a max over ranks (NCCL on GPUs; gloo
    on CPU for the host-side tests).  No collective touches the data path."""

    def __init__(self, world, rank, local, backend: str = "nccl", timeout_s: int = 120):
        import torch
        self.world, self.rank, self.local = world, rank, local
        self.backend = backend
        self.pg = None
        if world > 1:
            import torch.distributed as td
            kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
            td.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.pg = td

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def aggregate(units_per_rank: float, ms_rank: float, dist) -> tuple:
    """Whole-job throughput of independent replicas: the units all ranks
    processed over the slowest rank's time.  Returns (units per second, max ms)."""
    ms_max = dist.max(ms_rank)
    return units_per_rank * dist.world / (ms_max * 1e-3), ms_max


def graph_time(fn_for_step, steps: int, warmup: int, dist=None, clocks=None, sustain_s: float = 0.0):
    """Captures `steps` calls fn_for_step(i) in one CUDA graph and times one
    replay with events on the capturing stream.  Returns (ms per step, ms of
    the replay, sustained ms per step or None).  `clocks` samples the GPU over
    the warm replays and the timed replay.  With sustain_s > 0 the graph is
    then replayed back to back for that long, under the power cap, and timed
    as a whole (the sustained figure)."""
    import torch
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for i in range(max(warmup, 1)):
            fn_for_step(i)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(steps):
            fn_for_step(i)
    # warm replays of the graph itself, for at least 50 ms so that the SM
    # clocks have left their idle level before the timed replay
    def replays(seconds):
        t_end = time.perf_counter() + seconds
        n = 0
        while True:
            g.replay()
            n += 1
            s.synchronize()
            if time.perf_counter() >= t_end:
                return n
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.__enter__()
    try:
        replays(0.05)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        if clocks is not None:
            clocks.mark("timed_start")
        with torch.cuda.stream(s):
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
        if clocks is not None:
            clocks.mark("timed_end")
        torch.cuda.synchronize()
    finally:
        if clocks is not None:
            clocks.__exit__(None, None, None)
    if dist is not None:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    sustained = None
    if sustain_s > 0:
        reps = max(1, int(sustain_s / max(ms * 1e-3, 1e-6)))
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(reps):
                g.replay()
            e1.record(s)
        s.synchronize()
        sustained = e0.elapsed_time(e1) / (reps * steps)
    del g
    return ms / steps, ms, sustained


# ---------------------------------------------------------------------------
# headline: per-token W8A8 GEMM
# ---------------------------------------------------------------------------
def headline(args, dist, pk):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    d = synth.gemm_w8a8(**HEAD)
    x0 = torch.from_numpy(d["x"]).cuda()
    w0 = torch.from_numpy(d["w"]).cuda()
    deq = torch.from_numpy(d["deq_scale"]).cuda()
    pts = torch.from_numpy(d["per_token_scale"]).cuda()
    xs = [x0.clone() for _ in range(L2_COPIES)]
    ws = [w0.clone() for _ in range(L2_COPIES)]
    outs = [torch.empty((HEAD["M"], HEAD["N"]), dtype=torch.bfloat16, device="cuda") for _ in range(L2_COPIES)]

    def step(i):
        j = i % L2_COPIES
        bq.bq_gemm_i8_pertoken(xs[j], ws[j], deq, pts, out=outs[j])

    clocks = Clocks(torch.cuda.current_device())
    ms_step, ms_total, ms_sust = graph_time(step, args.steps, args.warmup, dist, clocks, sustain_s=1.5)
    ops = 2.0 * HEAD["M"] * HEAD["N"] * HEAD["K"]
    tops_rank = ops / (ms_step * 1e-3) / 1e12
    ops_per_s, ms_step_max = aggregate(ops, ms_step, dist)
    value = ops_per_s / 1e12
    st, detail = bq.bq_device_status()
    if st != bq.BQ_OK:
        raise RuntimeError(f"device status {detail:#x} after the timed region")
    # int8 dense = 2x bf16 dense (nominal 4.5 vs 2.25 PF); a timed region of more than 0.2 s
    # runs under the power cap, which the sustained bf16 figure describes
    sustained = ms_total >= 200.0
    bf16_peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    peak_int8 = 2.0 * bf16_peak
    src = source_hash("gemm_tc.cu", "bq_common.cuh")
    traffic = NCU_TRAFFIC.get(("gemm_w8a8_4096", src))
    roof = {"bound": "tensor", "achieved": round(tops_rank, 2), "peak": round(peak_int8, 1), "unit": "TFLOP/s",
            "frac": round(tops_rank / peak_int8, 4), "traffic": traffic,
            "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch; the write count "
                            "misses the bf16 output still in L2 when the kernel ends",
            "kernel": "gemm_pair_kernel<bf16 out> (W8A8, K-major B, CTA pairs, tcgen05 cta_group::2)",
            "peak_note": f"{pk['source']} bf16 {'sustained' if sustained else 'burst'} {bf16_peak} TFLOP/s x 2 "
                         f"(nominal int8/bf16 ratio; timed region {ms_total:.0f} ms); "
                         "int8 ops counted like flops, 2 per multiply-add",
            "algorithmic_bytes_per_launch": 2 * 4096 * 4096 + 4096 * 4096 * 2 + 2 * 4096 * 4}
    if ms_sust is not None:
        sust_tops = ops / (ms_sust * 1e-3) / 1e12
        sust_peak = 2.0 * pk["bf16_tflops_sustained"]
        roof["sustained"] = {"us_per_step": round(ms_sust * 1e3, 3), "achieved": round(sust_tops, 2),
                             "peak": round(sust_peak, 1), "frac": round(sust_tops / sust_peak, 4),
                             "note": "the same graph replayed back to back for 1.5 s (power-capped clocks), "
                                     "against the sustained bf16 figure x 2"}
    # end to end through the public API with host buffers
    e2e = headline_e2e(args, d, dist)
    return {"value": value, "ms_per_step": ms_step_max, "roofline": roof, "clocks": clocks.summary(), "e2e": e2e,
            "gpu_launches": args.steps}, d


def headline_e2e(args, d, dist):
    """The headline call through the Python API from pinned host buffers: every
    step uploads its inputs (x, w, both scale vectors), runs the GEMM and reads
    its bf16 output back.  Consecutive steps are pipelined the way a serving loop
    would run them: uploads on one stream, the GEMM on a second, the read-back on
    a third, two sets of device buffers, so step i+1's upload and step i-1's
    read-back overlap step i's GEMM (PCIe carries both directions at once).  The
    timed region runs from before the first upload to after the last read-back."""
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    steps = max(2, min(args.steps, 100))
    xh = torch.from_numpy(d["x"]).pin_memory()
    wh = torch.from_numpy(d["w"]).pin_memory()
    dh = torch.from_numpy(d["deq_scale"]).pin_memory()
    ph = torch.from_numpy(d["per_token_scale"]).pin_memory()
    oh = [torch.empty((HEAD["M"], HEAD["N"]), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    bufs = [(torch.empty_like(xh, device="cuda"), torch.empty_like(wh, device="cuda"),
             torch.empty_like(dh, device="cuda"), torch.empty_like(ph, device="cuda"),
             torch.empty((HEAD["M"], HEAD["N"]), dtype=torch.bfloat16, device="cuda")) for _ in range(2)]
    up, comp, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    read_back = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            k = i & 1
            xd, wd, dd, pd, od = bufs[k]
            if i >= 2:
                up.wait_event(computed[k])       # the GEMM of step i-2 has read these inputs
            with torch.cuda.stream(up):
                xd.copy_(xh, non_blocking=True)
                wd.copy_(wh, non_blocking=True)
                dd.copy_(dh, non_blocking=True)
                pd.copy_(ph, non_blocking=True)
                uploaded[k].record(up)
            comp.wait_event(uploaded[k])
            if i >= 2:
                comp.wait_event(read_back[k])    # step i-2's output has been read back
            with torch.cuda.stream(comp):
                bq.bq_gemm_i8_pertoken(xd, wd, dd, pd, out=od, stream=comp)
                computed[k].record(comp)
            down.wait_event(computed[k])
            with torch.cuda.stream(down):
                oh[k].copy_(od, non_blocking=True)
                read_back[k].record(down)

    run(max(args.warmup, 2))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    e0.record(up)
    comp.wait_event(e0)
    down.wait_event(e0)
    run(steps)
    up.wait_stream(down)
    e1.record(up)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(e0.elapsed_time(e1) / steps)
    ops = 2.0 * HEAD["M"] * HEAD["N"] * HEAD["K"]
    h2d = xh.numel() + wh.numel() + 4 * (dh.numel() + ph.numel())
    d2h = 2 * oh[0].numel()
    return {"value": round(ops * dist.world / (ms * 1e-3) / 1e12, 3), "unit": "TOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": round(ms, 4),
            "pipelining": "upload / GEMM / read-back on three streams, two buffer sets"}


# ---------------------------------------------------------------------------
# secondary workloads
# ---------------------------------------------------------------------------
def workloads(args, pk):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    res = {}
    hbm = pk["hbm_gbs"]
    peak_int8 = 2.0 * pk["bf16_tflops"]
    steps = args.workload_steps
    want = set(args.workloads.split(","))
    if "decode" in want:
        _decode(res, steps, hbm, [int(m) for m in args.decode_ms.split(",")])
    if "w4" in want:
        _w4(res, steps, hbm, [int(m) for m in args.w4_ms.split(",")])
    if "prefill" in want:
        _prefill(res, max(steps // 4, 1), peak_int8, hbm)
    if "tiny" in want:
        _tiny(res, steps)
    if "batched" in want:
        _batched(res, steps, peak_int8)
    if "w4a4" in want:
        _w4a4(res, steps, peak_int8, hbm)
    if "layernorm" in want:
        _layernorm(res, steps, peak_int8, hbm)
    if "conv" in want:
        _conv(res, max(steps // 4, 1), peak_int8)
    if "backward" in want:
        _backward(res, max(steps // 8, 1), pk)
    st, detail = bq.bq_device_status()
    if st != bq.BQ_OK:
        raise RuntimeError(f"device status {detail:#x} after the workloads")
    return res


def _decode(res, steps, hbm, ms=(1, 4, 16)):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    N, K = 11008, 4096
    w = torch.from_numpy(synth.bitlinear_weight(N, K, 3)).cuda()
    wp, wsc = bq.bq_weight_quant_ternary_pack(w)
    del w
    copies = 24  # 24 x 11.3 MB = 270 MB > 2x L2
    wps = [wp.clone() for _ in range(copies)]
    for M in ms:
        d = synth.bitlinear_decode(M)
        x = torch.from_numpy(d["x_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K), dtype=torch.uint8, device="cuda")

        def step(i, x=x, out=out, work=work):
            bq.bq_bitlinear_w2a8(x, wps[i % copies], wsc, N, None, 1e-5, torch.bfloat16, out=out, workspace=work)

        ms, _, _ = graph_time(step, steps, 3)
        byts = N * K // 4 + 4 + 2 * M * K + 2 * M * N
        gbs = byts / (ms * 1e-3) / 1e9
        res[f"bitlinear_decode_M{M}"] = {"us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1),
                                         "frac_hbm": round(gbs / hbm, 4), "algorithmic_bytes": byts,
                                         "weight_GB/s": round((N * K // 4) / (ms * 1e-3) / 1e9, 1),
                                         "launches_per_step": 1,
                                         "config": f"x bf16 [{M},4096], W 2-bit [11008,4096]"}
    del wps


def _w4(res, steps, hbm, ms=(1, 32)):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # Grouped affine INT4, 4096 -> 14336, g = 128
    N, K, gs = 14336, 4096, 128
    wq = synth.linear_w4_weights()
    qw, qz = bq.bq_weight_pack_int4_grouped(torch.from_numpy(wq["q"]).cuda(), torch.from_numpy(wq["zeros"]).cuda(), gs)
    sc = torch.from_numpy(wq["scales_f16"].view(np.int16)).cuda()
    bias = torch.from_numpy(wq["bias"]).cuda()
    copies = 10  # 10 x 30.6 MB = 306 MB
    sets = [(qw.clone(), sc.clone(), qz.clone()) for _ in range(copies)]
    for M in ms:
        x = torch.from_numpy(synth.linear_w4_activations(M)).cuda()
        out = torch.empty((M, N), dtype=torch.float32, device="cuda")
        work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4_GROUPED, M, N, K, gs), dtype=torch.uint8,
                           device="cuda")

        def step(i, x=x, out=out, work=work):
            a, b, c = sets[i % copies]
            bq.bq_linear_w4_grouped(x, a, b, c, gs, bias, out=out, workspace=work)

        ms, _, _ = graph_time(step, steps, 3)
        byts = N * K // 2 + N * (K // gs) * 2 + N * ((K // gs + 7) // 8) * 4 + 4 * N + 4 * M * K + 4 * M * N
        gbs = byts / (ms * 1e-3) / 1e9
        res[f"linear_w4_M{M}"] = {"us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1),
                                  "frac_hbm": round(gbs / hbm, 4), "algorithmic_bytes": byts,
                                  "dequant_f32_bytes_elided": N * K * 4 - N * K // 2,
                                  "config": f"x fp32 [{M},4096], INT4 [14336,4096] g128"}
    del sets


def _prefill(res, steps, peak_int8, hbm):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # BitLinear prefill [8192, 4096] x [4096, 4096]
    d = synth.bitlinear_prefill()
    M, N, K = 8192, 4096, 4096
    x = torch.from_numpy(d["x_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    wp, wsc = bq.bq_weight_quant_ternary_pack(torch.from_numpy(d["w"]).cuda())
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K), dtype=torch.uint8, device="cuda")

    def step(i):
        bq.bq_bitlinear_w2a8(x, wp, wsc, N, None, 1e-5, torch.bfloat16, out=out, workspace=work)

    ms, _, _ = graph_time(step, steps, 3)
    ops = 2.0 * M * N * K
    tops = ops / (ms * 1e-3) / 1e12
    # the activation quantization alone, to split the step (three copies of x so
    # that two calls, 192 MB, separate reuses of one: each call reads x from HBM)
    xs = [x] + [x.clone() for _ in range(2)]
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sc = torch.empty(M, dtype=torch.float32, device="cuda")
    rs = torch.empty(M, dtype=torch.int32, device="cuda")

    def aq(i):
        bq.bq_act_quant_int8(xs[i % 3], 1e-5, xq=xq, act_scale=sc, rowsum=rs)

    ms_aq, _, _ = graph_time(aq, steps, 3)
    aq_bytes = 2 * M * K + M * K + 8 * M
    gemm_ms = max(ms - ms_aq, 1e-9)
    res["bitlinear_prefill"] = {"us_per_step": round(ms * 1e3, 2), "TOPS": round(tops, 1),
                                "frac_int8_peak": round(tops / peak_int8, 4),
                                "act_quant_us": round(ms_aq * 1e3, 2),
                                "act_quant_frac_hbm": round(aq_bytes / (ms_aq * 1e-3) / 1e9 / hbm, 4),
                                "gemm_us_derived": round(gemm_ms * 1e3, 2),
                                "gemm_TOPS_derived": round(ops / (gemm_ms * 1e-3) / 1e12, 1),
                                "config": "x bf16 [8192,4096] (1% outlier channels), W 2-bit [4096,4096]; "
                                          "act quant + tcgen05 GEMM per step (160 MB moved > L2); "
                                          "gemm_*_derived = step minus the separately timed act quant"}


def _tiny(res, steps):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # BitLinear tiny [8,256] x [128,256], fp32 out
    d = synth.bitlinear_tiny(0)
    x = torch.from_numpy(d["x"]).cuda()
    wp, wsc = bq.bq_weight_quant_ternary_pack(torch.from_numpy(d["w"]).cuda())
    out = torch.empty((8, 128), dtype=torch.float32, device="cuda")
    work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, 8, 128, 256), dtype=torch.uint8, device="cuda")

    def step(i):
        bq.bq_bitlinear_w2a8(x, wp, wsc, 128, None, 1e-5, torch.float32, out=out, workspace=work)

    ms, _, _ = graph_time(step, steps, 3)
    res["bitlinear_tiny"] = {"us_per_step": round(ms * 1e3, 3), "config": "x fp32 [8,256], W [128,256]"}


def _batched(res, steps, peak_int8):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # batched per-token W8A8: 8 x ([512,4096] x [4096,4096]) per-batch weights and scales,
    # and the 4096^3 product with x stored [K, M] (transposeA); 4 rotating copies (> L2)
    B, M, N, K = 8, 512, 4096, 4096
    g = synth.rng(31)
    x = torch.from_numpy(synth.int8_uniform(g, (B, M, K))).cuda()
    w = torch.from_numpy(synth.int8_uniform(g, (B, N, K))).cuda()
    deq = torch.from_numpy(synth.uniform_f32(g, (B, N), 0.001, 0.01)).cuda()
    pts = torch.from_numpy(synth.uniform_f32(g, (B, M), 0.001, 0.01)).cuda()
    sets = [(x.clone(), w.clone()) for _ in range(4)]
    out = torch.empty((B, M, N), dtype=torch.bfloat16, device="cuda")

    def step(i):
        a, b = sets[i % 4]
        bq.bq_gemm_i8_pertoken_batched(a, b, deq, pts, out=out)

    ms, _, _ = graph_time(step, steps, 3)
    ops = 2.0 * B * M * N * K
    res["gemm_batched_8x512"] = {"us_per_step": round(ms * 1e3, 2), "TOPS": round(ops / (ms * 1e-3) / 1e12, 1),
                                 "frac_int8_peak": round(ops / (ms * 1e-3) / 1e12 / peak_int8, 4),
                                 "config": "x int8 [8,512,4096] x w int8 [8,4096,4096] (N,K), per-batch scales, bf16 out"}
    del sets, x, w
    d = synth.gemm_w8a8()
    xt = torch.from_numpy(np.ascontiguousarray(d["x"].T)).cuda()[None]
    w1 = torch.from_numpy(d["w"]).cuda()[None]
    sets = [(xt.clone(), w1.clone()) for _ in range(4)]
    dq, pt = torch.from_numpy(d["deq_scale"]).cuda(), torch.from_numpy(d["per_token_scale"]).cuda()
    out1 = torch.empty((1, 4096, 4096), dtype=torch.bfloat16, device="cuda")

    def step_t(i):
        a, b = sets[i % 4]
        bq.bq_gemm_i8_pertoken_batched(a, b, dq, pt, trans_a=True, out=out1)

    ms, _, _ = graph_time(step_t, steps, 3)
    ops = 2.0 * 4096 ** 3
    res["gemm_transA_4096"] = {"us_per_step": round(ms * 1e3, 2), "TOPS": round(ops / (ms * 1e-3) / 1e12, 1),
                               "frac_int8_peak": round(ops / (ms * 1e-3) / 1e12 / peak_int8, 4),
                               "config": "x int8 stored [4096 (K), 4096 (M)] (transposeA) x w [4096,4096] (N,K), "
                                         "single-CTA tiles, bf16 out"}


def _w4a4(res, steps, peak_int8, hbm):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # 4-bit activations / 4-bit weights with given steps: prefill 4096^3 and one-token decode 11008 x 4096
    eps = 1e-6
    for (M, N, K, tag) in ((4096, 4096, 4096, "w4a4_prefill_4096"), (1, 11008, 4096, "w4a4_decode_M1")):
        g = synth.rng((41, M, N))
        x = torch.from_numpy(synth.f32_to_bf16_bits(synth.normal_f32(g, (M, K))).view(np.int16)).cuda().view(
            torch.bfloat16)
        w = torch.from_numpy(synth.normal_f32(g, (N, K), 0.02)).cuda()
        sa = torch.tensor([0.27], dtype=torch.float32, device="cuda")
        sw = (w.abs().amax(dim=1) / 7.5).contiguous()
        wp = bq.bq_weight_quant_int4_pack(w, sw, eps)
        del w
        copies = max(1, min(24, int(300e6 // (N * K // 2))))
        wps = [wp.clone() for _ in range(copies)]
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4A4, M, N, K), dtype=torch.uint8, device="cuda")

        def step(i, x=x, sa=sa, sw=sw, out=out, work=work, wps=wps):
            bq.bq_linear_w4a4(x, sa, wps[i % len(wps)], sw, N, eps, out=out, workspace=work)

        ms, _, _ = graph_time(step, steps if M == 1 else max(steps // 4, 1), 3)
        if M == 1:
            byts = N * K // 2 + 4 * N + 2 * K + 2 * N
            gbs = byts / (ms * 1e-3) / 1e9
            res[tag] = {"us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                        "algorithmic_bytes": byts, "config": "x bf16 [1,4096], W 4-bit [11008,4096], per-channel steps; "
                                                             "act quant + dp4a GEMV"}
        else:
            ops = 2.0 * M * N * K
            tops = ops / (ms * 1e-3) / 1e12
            res[tag] = {"us_per_step": round(ms * 1e3, 2), "TOPS": round(tops, 1),
                        "frac_int8_peak": round(tops / peak_int8, 4),
                        "config": "x bf16 [4096,4096], W 4-bit [4096,4096], per-channel steps; act quant + tcgen05 "
                                  "GEMM with the nibbles sign-extended in shared memory"}
        del wps


def _layernorm(res, steps, peak_int8, hbm):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # BitLinear with the LayerNorm normaliser: prefill 8192 x 4096 x 4096, one-token decode 11008 x 4096
    for (M, N, K, tag) in ((8192, 4096, 4096, "bitlinear_ln_prefill"), (1, 11008, 4096, "bitlinear_ln_decode_M1")):
        g = synth.rng((42, M, N))
        x = torch.from_numpy(synth.f32_to_bf16_bits(synth.normal_f32(g, (M, K)) + np.float32(0.75)).view(np.int16)
                             ).cuda().view(torch.bfloat16)
        lw = torch.from_numpy((1.0 + 0.2 * g.standard_normal(K)).astype(np.float32)).cuda()
        lb = torch.from_numpy((0.1 * g.standard_normal(K)).astype(np.float32)).cuda()
        wp, wsc = bq.bq_weight_quant_ternary_pack(torch.from_numpy(synth.bitlinear_weight(N, K, 6)).cuda())
        copies = max(1, min(24, int(300e6 // (N * K // 4))))
        wps = [wp.clone() for _ in range(copies)]
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K), dtype=torch.uint8, device="cuda")

        def step(i, x=x, out=out, work=work, wps=wps, wsc=wsc, lw=lw, lb=lb):
            bq.bq_bitlinear_w2a8_layernorm(x, wps[i % len(wps)], wsc, N, lw, lb, None, 1e-5, out=out, workspace=work)

        ms, _, _ = graph_time(step, steps if M == 1 else max(steps // 4, 1), 3)
        if M == 1:
            byts = N * K // 4 + 2 * K + 8 * K + 2 * N
            gbs = byts / (ms * 1e-3) / 1e9
            res[tag] = {"us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                        "algorithmic_bytes": byts, "config": "x bf16 [1,4096], affine LayerNorm, W 2-bit [11008,4096]; "
                                                             "binary64 LayerNorm quant + split GEMV"}
        else:
            ops = 2.0 * M * N * K
            tops = ops / (ms * 1e-3) / 1e12
            res[tag] = {"us_per_step": round(ms * 1e3, 2), "TOPS": round(tops, 1),
                        "frac_int8_peak": round(tops / peak_int8, 4),
                        "config": "x bf16 [8192,4096], affine LayerNorm, W 2-bit [4096,4096]; binary64 LayerNorm "
                                  "quant + tcgen05 GEMM"}
        del wps


def _conv(res, steps, peak_int8):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # BitConv1d: x (8, 1024, 1024) -> (8, 1024, 1024), kernel 3, padding 1
    B, C_in, L, C_out, KS = 8, 1024, 1024, 1024, 3
    g = synth.rng(43)
    x = torch.from_numpy(synth.f32_to_bf16_bits(synth.normal_f32(g, (B, C_in, L))).view(np.int16)).cuda().view(
        torch.bfloat16)
    wp, wsc = bq.bq_bitconv1d_weight_pack(torch.from_numpy(synth.normal_f32(g, (C_out, C_in, KS), 0.02)).cuda())
    out = torch.empty((B, C_out, L), dtype=torch.bfloat16, device="cuda")
    work = torch.empty(bq.lib().bq_bitconv1d_workspace_bytes(B, C_in, L, C_out, KS, 1, 1, 1), dtype=torch.uint8,
                       device="cuda")

    def step(i):
        bq.bq_bitconv1d(x, wp, wsc, C_out, KS, 1, 1, 1, out=out, workspace=work)

    ms, _, _ = graph_time(step, steps, 3)
    ops = 2.0 * B * L * C_out * C_in * KS
    tops = ops / (ms * 1e-3) / 1e12
    res["bitconv1d_8x1024x1024_k3"] = {"us_per_step": round(ms * 1e3, 2), "TOPS": round(tops, 1),
                                       "frac_int8_peak": round(tops / peak_int8, 4),
                                       "config": "x bf16 (8, 1024, 1024), W [1024, 1024, 3] ternary, padding 1; "
                                                 "transpose, LayerNorm quant, 3 x (gather + tcgen05 GEMM), tap sum"}


def _backward(res, steps, pk):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    # straight-through backward of BitLinear, M = N = K = 4096: dy and dW on the bf16 tensor cores
    M = N = K = 4096
    g = synth.rng(44)
    x = torch.from_numpy(synth.f32_to_bf16_bits(synth.normal_f32(g, (M, K))).view(np.int16)).cuda().view(
        torch.bfloat16)
    dout = torch.from_numpy(synth.f32_to_bf16_bits(synth.normal_f32(g, (M, N))).view(np.int16)).cuda().view(
        torch.bfloat16)
    wp, wsc = bq.bq_weight_quant_ternary_pack(torch.from_numpy(synth.bitlinear_weight(N, K, 7)).cuda())
    dx = torch.empty((M, K), dtype=torch.float32, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8_BACKWARD, M, N, K), dtype=torch.uint8,
                       device="cuda")

    def step(i):
        bq.bq_bitlinear_w2a8_backward(x, dout, wp, wsc, 1e-5, dx=dx, dw=dw, workspace=work)

    ms, _, _ = graph_time(step, steps, 3)
    flops = 2.0 * 2.0 * M * N * K  # the two contractions (the hi / lo split of dW is overhead, not counted)
    tf = flops / (ms * 1e-3) / 1e12
    res["bitlinear_backward_4096"] = {"us_per_step": round(ms * 1e3, 1), "TFLOP/s": round(tf, 1),
                                      "frac_bf16_peak": round(tf / pk["bf16_tflops"], 4),
                                      "config": "x bf16 [4096,4096], dout bf16 [4096,4096], W 2-bit [4096,4096]; "
                                                "act quant, operand prep, 2 x tcgen05 kind::f16 GEMM (dW with a "
                                                "hi/lo split: 2M contraction), RMSNorm backward"}
    del dx, dw, work

    # straight-through backward of the 4-bit activation / weight linear, one weight step, M = N = K = 4096
    wf = torch.from_numpy(synth.normal_f32(g, (N, K), 0.02)).cuda()
    sa = torch.tensor([0.27], dtype=torch.float32, device="cuda")
    sw = torch.tensor([0.006], dtype=torch.float32, device="cuda")
    dx = torch.empty((M, K), dtype=torch.float32, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ds = torch.empty(1, dtype=torch.float32, device="cuda")
    work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4A4_BACKWARD, M, N, K), dtype=torch.uint8,
                       device="cuda")

    def step4(i):
        bq.bq_linear_w4a4_backward(x, wf, dout, sa, sw, 1e-6, dx=dx, dw=dw, dscale_a=ds, workspace=work)

    ms, _, _ = graph_time(step4, steps, 3)
    tf = flops / (ms * 1e-3) / 1e12
    res["w4a4_backward_4096"] = {"us_per_step": round(ms * 1e3, 1), "TFLOP/s": round(tf, 1),
                                 "frac_bf16_peak": round(tf / pk["bf16_tflops"], 4),
                                 "config": "x bf16 [4096,4096], W fp32 [4096,4096] (4-bit codes, one step), dout bf16 "
                                           "[4096,4096]; codes, 2 x tcgen05 kind::f16 GEMM, range masks, binary64 "
                                           "dscale_a"}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on all host cores, every workload of the set
# ---------------------------------------------------------------------------
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _ranges(n: int, parts: int):
    parts = max(1, min(parts, n))
    step, extra = divmod(n, parts)
    lo = 0
    for i in range(parts):
        hi = lo + step + (1 if i < extra else 0)
        yield lo, hi
        lo = hi


def run_rows(fn, n: int, threads: int) -> float:
    """Wall time of fn(lo, hi) over rows [0, n) split across `threads` threads.
    The oracle's C routines run without the GIL (ctypes releases it), so the
    threads run in parallel; each runs the plain oracle on its own rows."""
    t0 = time.perf_counter()
    if threads <= 1:
        fn(0, n)
    else:
        with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
            for f in [ex.submit(fn, lo, hi) for lo, hi in _ranges(n, threads)]:
                f.result()
    return time.perf_counter() - t0


def sample_rows(fn, total: int, threads: int, budget_s: float, probe: int = 0) -> tuple:
    """Rows of a bounded sample (whole multiples of the thread count, capped at
    `total`) sized so fn over them takes about budget_s on `threads` threads.
    Returns (rows, seconds) of the timed sample (when the whole workload fits,
    the mean over repeated runs of it)."""
    probe = probe or min(total, threads)
    while True:
        t = run_rows(fn, probe, threads)
        if t >= 0.1 * budget_s or probe >= total:
            break
        probe = min(total, probe * 4)
    if probe >= total:
        # the whole workload fits the budget: repeat it for a stable mean
        reps = max(1, min(50, int(0.5 * budget_s / max(t, 1e-6))))
        if reps > 1:
            t = sum(run_rows(fn, total, threads) for _ in range(reps)) / reps
        return total, t
    per_round = t / max(1, -(-probe // threads))  # seconds per row per thread
    rows = int(budget_s / max(per_round, 1e-9)) * threads
    rows = max(threads, min(total, rows))
    return rows, run_rows(fn, rows, threads)


def _head_fn(d):
    import oracle

    def fn(lo, hi):
        oracle.gemm_i8_pertoken(d["x"][lo:hi], d["w"], d["deq_scale"], d["per_token_scale"][lo:hi])
    return fn


def cpu_baseline(d, args, pk) -> dict:
    """The oracle, as it stands, on the host cores for every workload; the
    headline's figure is the line's cpu_baseline.value."""
    import oracle
    import synth
    oracle.build()
    cores = host_cores()
    budget = args.cpu_budget
    res = {}
    # W8A8 GEMM 4096^3: rows of x
    M, N, K = HEAD["M"], HEAD["N"], HEAD["K"]
    if args.cpu_rows > 0:
        rows = min(M, args.cpu_rows)
        t = run_rows(_head_fn(d), rows, cores)
    else:
        rows, t = sample_rows(_head_fn(d), M, cores, budget)
    res["gemm_w8a8_4096"] = {"value": round(2.0 * rows * N * K / t / 1e12, 6), "unit": "TOPS", "cores": cores,
                             "sample": f"{rows} of {M} rows (all {N} columns), {t:.2f} s"}
    # BitLinear prefill 8192 x 4096 x 4096: act quant + integer linear on rows of x (weights quantized beforehand)
    dp = synth.bitlinear_prefill()
    tq = oracle.ternary_quant(dp["w"])

    def prefill(lo, hi):
        a = oracle.act_quant(dp["x"][lo:hi], dp["eps"])
        oracle.bitlinear_from_codes(a["xq"], a["act_scale"], tq["wq"], tq["gamma"])
    rows, t = sample_rows(prefill, 8192, cores, budget)
    res["bitlinear_prefill"] = {"value": round(2.0 * rows * 4096 * 4096 / t / 1e12, 6), "unit": "TOPS",
                                "cores": cores, "sample": f"{rows} of 8192 rows (all 4096 columns), {t:.2f} s"}
    # BitLinear decode, M in {1, 4, 16}: act quant of the tokens + integer linear over weight rows
    wd = synth.bitlinear_weight(11008, 4096, 3)
    td = oracle.ternary_quant(wd)
    for Md in (1, 4, 16):
        dd = synth.bitlinear_decode(Md)
        a = oracle.act_quant(dd["x"], dd["eps"])

        def decode(lo, hi, a=a, dd=dd):
            aa = oracle.act_quant(dd["x"], dd["eps"]) if lo == 0 else a
            oracle.bitlinear_from_codes(aa["xq"], aa["act_scale"], td["wq"][lo:hi], td["gamma"])
        rows, t = sample_rows(decode, 11008, cores, budget / 3)
        byts = (11008 * 4096 // 4 + 4 + 2 * Md * 4096 + 2 * Md * 11008) * rows / 11008
        res[f"bitlinear_decode_M{Md}"] = {"value": round(byts / t / 1e9, 4), "unit": "GB/s", "cores": cores,
                                          "sample": f"{rows} of 11008 weight rows, {t:.3f} s (bytes of the GPU "
                                                    "call's packed weights, scaled to the rows)"}
    # grouped INT4, M in {1, 32}: over weight rows
    w4 = synth.linear_w4_weights()
    qw, qz = oracle.int4_pack(w4["q"]), oracle.int4_pack(w4["zeros"])
    sb = w4["scales_f16"].view(np.uint16)
    Nw, Kw, gs = 14336, 4096, 128
    for Mw in (1, 32):
        xw = synth.linear_w4_activations(Mw)

        def w4f(lo, hi, xw=xw):
            oracle.linear_w4_grouped(xw, qw[lo:hi], sb[lo:hi], qz[lo:hi], w4["bias"][lo:hi], gs)
        rows, t = sample_rows(w4f, Nw, cores, budget / 2)
        byts = (Nw * Kw // 2 + Nw * (Kw // gs) * 2 + Nw * 4 * 4 + 4 * Nw + 4 * Mw * Kw + 4 * Mw * Nw) * rows / Nw
        res[f"linear_w4_M{Mw}"] = {"value": round(byts / t / 1e9, 4), "unit": "GB/s", "cores": cores,
                                   "sample": f"{rows} of {Nw} weight rows, {t:.3f} s (bytes of the GPU call, "
                                             "scaled to the rows)"}
    # BitLinear tiny 8 x 256 -> 128: whole forward from pre-quantized weights, one thread
    dt = synth.bitlinear_tiny(0)
    tt = oracle.ternary_quant(dt["w"])
    reps = 200
    t0 = time.perf_counter()
    for _ in range(reps):
        a = oracle.act_quant(dt["x"], dt["eps"])
        oracle.bitlinear_from_codes(a["xq"], a["act_scale"], tt["wq"], tt["gamma"])
    t = (time.perf_counter() - t0) / reps
    res["bitlinear_tiny"] = {"value": round(t * 1e6, 2), "unit": "us per call", "cores": 1,
                             "sample": f"whole workload, mean of {reps} calls"}
    head = res["gemm_w8a8_4096"]
    return {"value": head["value"], "unit": "TOPS", "cores": cores, "kind": "oracle", "host_cores": os.cpu_count(),
            "sample": f"W8A8 4096^3: {head['sample']}, plain C oracle on row-parallel threads",
            "workloads": res}


def reference_arm(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    import oracle
    import synth
    oracle.build()
    d = synth.gemm_w8a8(**HEAD)
    cores = host_cores()
    fn = _head_fn(d)
    if args.cpu_rows > 0:
        rows = args.cpu_rows
    else:
        # rows per step sized so that warm-up plus timed steps take about a minute
        t1 = run_rows(fn, cores, cores)
        rows = max(1, int(60.0 / max(args.steps + args.warmup, 1) / max(t1, 1e-6)) * cores)
        rows = min(rows, HEAD["M"])
    for _ in range(args.warmup):
        run_rows(fn, rows, cores)
    t = sum(run_rows(fn, rows, cores) for _ in range(args.steps))
    ops = 2.0 * rows * HEAD["N"] * HEAD["K"] * args.steps
    value = ops / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "config": {"workload": HEAD_WORKLOAD, **HEAD, "sample_rows_per_step": rows},
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": cores, "kind": "oracle",
                             "host_cores": os.cpu_count(),
                             "sample": f"{rows} rows x 4096 columns per step, plain C double/int64 loops on "
                                       f"{cores} row-parallel threads"},
            "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        reference_arm(args)
        return
    import torch
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    from bit_quantized_linear_rmsnorm_b200 import _build
    if rank == 0:
        _build.build()
    dist = Dist(world, rank, local)
    dist.barrier()
    import bit_quantized_linear_rmsnorm_b200 as bq
    bq.lib()
    pk = peaks()
    extra = {}
    if args.no_head:
        if rank == 0:
            print(json.dumps({"workloads": workloads(args, pk)}), flush=True)
        dist.close()
        return
    head, d = headline(args, dist, pk)
    if not args.no_workloads and rank == 0:
        extra = workloads(args, pk)
    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(d, args, pk)
    if rank == 0:
        line = {"metric": METRIC, "value": round(head["value"], 2), "unit": "TOPS", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(head["ms_per_step"], 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
                "data": "synthetic",
                "config": {"workload": HEAD_WORKLOAD, **HEAD, "parallelism": f"replicas x{world}",
                           "l2": f"{L2_COPIES} rotating input/output copies (268 MB of x+w > 126 MB L2)",
                           "timing": "one CUDA graph of `steps` launches, CUDA events on the launching stream"},
                "roofline": head["roofline"], "cpu_baseline": base, "e2e": head["e2e"],
                "gpu_launches": head["gpu_launches"], "clocks": head["clocks"], "workloads": extra}
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
