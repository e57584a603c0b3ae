#!/usr/bin/env python
"""Benchmark of the quantized linear layer on B200 (one JSON line on rank 0).

Headline workload: the per-token W8A8 GEMM, x int8 [4096,4096] x weight int8
[4096,4096] (nn.Linear layout) with per-token and per-channel fp32 scales,
bf16 out; metric int8-equivalent TOPS (2 ops per multiply-add).  One step is
one call of bq_gemm_i8_pertoken (one kernel launch) on inputs resident in
HBM; K steps are captured in one CUDA graph that cycles through 8 copies of
the inputs (268 MB, larger than the 126 MB L2) and timed with CUDA events on
the launching stream.  `e2e` times the same call through the Python API with
pinned host buffers, the host->device copies of the step's inputs and the
device->host copy of its output inside the timed region.

The other workloads of the benchmark set (BitLinear decode and prefill,
grouped INT4 decode, the tiny BitLinear) are timed the same way and reported
under "workloads", each against its own roofline.

Multi-GPU: every rank runs an independent replica (the layer needs no
exchange); the time is the max over ranks and `value` sums the work of all
ranks.  `--impl reference` times the oracle (plain C, one host core) on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
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
# kernel source it was taken on; stale once the source changes.
NCU_TRAFFIC = {
    # profiles/gemm_w8a8_4096.md: 33.620992 MB read + 3.274240 MB written
    ("gemm_w8a8_4096", "83d85f51941e8ecf"): 36895232,
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10000)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-workloads", action="store_true", help="skip the secondary workloads")
    p.add_argument("--workloads", default="decode,w4,prefill,tiny",
                   help="comma list of secondary workloads: decode, w4, prefill, tiny")
    p.add_argument("--workload-steps", type=int, default=200)
    p.add_argument("--no-head", action="store_true", help="skip the headline GEMM (profiling runs only)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=0, help="oracle sample rows (0 = calibrate to ~10 s)")
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


class Clocks:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class Dist:
    def __init__(self, world, rank, local):
        import torch
        self.world, self.rank, self.local = world, rank, local
        self.pg = None
        if world > 1:
            import torch.distributed as td
            td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                  device_id=torch.device("cuda", local))
            self.pg = td

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device="cuda")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def graph_time(fn_for_step, steps: int, warmup: int, dist=None, clocks=None):
    """Captures `steps` calls fn_for_step(i) in one CUDA graph and times one
    replay with events on the capturing stream.  Returns ms per step."""
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
    t_end = time.perf_counter() + 0.05
    while True:
        g.replay()
        s.synchronize()
        if time.perf_counter() >= t_end:
            break
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ctx = clocks if clocks is not None else _Null()
    with ctx:
        with torch.cuda.stream(s):
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    del g
    return ms / steps, ms


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


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
    ms_step, ms_total = graph_time(step, args.steps, args.warmup, dist, clocks)
    ms_step_max = dist.max(ms_step)
    ops = 2.0 * HEAD["M"] * HEAD["N"] * HEAD["K"]
    tops_rank = ops / (ms_step * 1e-3) / 1e12
    value = ops * dist.world / (ms_step_max * 1e-3) / 1e12
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
            "kernel": "gemm_pair_kernel<bf16 out> (W8A8, K-major B, CTA pairs, tcgen05 cta_group::2)",
            "peak_note": f"{pk['source']} bf16 {'sustained' if sustained else 'burst'} {bf16_peak} TFLOP/s x 2 "
                         f"(nominal int8/bf16 ratio; timed region {ms_total:.0f} ms); "
                         "int8 ops counted like flops, 2 per multiply-add",
            "algorithmic_bytes_per_launch": 2 * 4096 * 4096 + 4096 * 4096 * 2 + 2 * 4096 * 4}
    # end to end through the public API with host buffers
    e2e = headline_e2e(args, d, dist)
    return {"value": value, "ms_per_step": ms_step_max, "roofline": roof, "clocks": clocks.summary(), "e2e": e2e,
            "gpu_launches": args.steps}, d


def headline_e2e(args, d, dist):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    steps = max(1, min(args.steps, 100))
    xh = torch.from_numpy(d["x"]).pin_memory()
    wh = torch.from_numpy(d["w"]).pin_memory()
    dh = torch.from_numpy(d["deq_scale"]).pin_memory()
    ph = torch.from_numpy(d["per_token_scale"]).pin_memory()
    oh = torch.empty((HEAD["M"], HEAD["N"]), dtype=torch.bfloat16).pin_memory()
    xd, wd = torch.empty_like(xh, device="cuda"), torch.empty_like(wh, device="cuda")
    dd, pd = torch.empty_like(dh, device="cuda"), torch.empty_like(ph, device="cuda")
    od = torch.empty((HEAD["M"], HEAD["N"]), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()

    def one():
        xd.copy_(xh, non_blocking=True)
        wd.copy_(wh, non_blocking=True)
        dd.copy_(dh, non_blocking=True)
        pd.copy_(ph, non_blocking=True)
        bq.bq_gemm_i8_pertoken(xd, wd, dd, pd, out=od)
        oh.copy_(od, non_blocking=True)

    with torch.cuda.stream(s):
        for _ in range(max(args.warmup, 1)):
            one()
    s.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(steps):
            one()
        e1.record(s)
    s.synchronize()
    dist.barrier()
    ms = dist.max(e0.elapsed_time(e1) / steps)
    ops = 2.0 * HEAD["M"] * HEAD["N"] * HEAD["K"]
    h2d = xh.numel() + wh.numel() + 4 * (dh.numel() + ph.numel())
    d2h = 2 * oh.numel()
    return {"value": round(ops * dist.world / (ms * 1e-3) / 1e12, 3), "unit": "TOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": round(ms, 4)}


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
        _decode(res, steps, hbm)
    if "w4" in want:
        _w4(res, steps, hbm)
    if "prefill" in want:
        _prefill(res, max(steps // 4, 1), peak_int8, hbm)
    if "tiny" in want:
        _tiny(res, steps)
    st, detail = bq.bq_device_status()
    if st != bq.BQ_OK:
        raise RuntimeError(f"device status {detail:#x} after the workloads")
    return res


def _decode(res, steps, hbm):
    import torch

    import bit_quantized_linear_rmsnorm_b200 as bq
    import synth
    N, K = 11008, 4096
    w = torch.from_numpy(synth.bitlinear_weight(N, K, 3)).cuda()
    wp, wsc = bq.bq_weight_quant_ternary_pack(w)
    del w
    copies = 24  # 24 x 11.3 MB = 270 MB > 2x L2
    wps = [wp.clone() for _ in range(copies)]
    for M in (1, 4, 16):
        d = synth.bitlinear_decode(M)
        x = torch.from_numpy(d["x_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K), dtype=torch.uint8, device="cuda")

        def step(i, x=x, out=out, work=work):
            bq.bq_bitlinear_w2a8(x, wps[i % copies], wsc, N, None, 1e-5, torch.bfloat16, out=out, workspace=work)

        ms, _ = graph_time(step, steps, 3)
        byts = N * K // 4 + 4 + 2 * M * K + 2 * M * N
        gbs = byts / (ms * 1e-3) / 1e9
        res[f"bitlinear_decode_M{M}"] = {"us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1),
                                         "frac_hbm": round(gbs / hbm, 4), "algorithmic_bytes": byts,
                                         "weight_GB/s": round((N * K // 4) / (ms * 1e-3) / 1e9, 1),
                                         "launches_per_step": 1, "config": f"x bf16 [{M},4096], W 2-bit [11008,4096]"}
    del wps


def _w4(res, steps, hbm):
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
    for M in (1, 32):
        x = torch.from_numpy(synth.linear_w4_activations(M)).cuda()
        out = torch.empty((M, N), dtype=torch.float32, device="cuda")
        work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4_GROUPED, M, N, K, gs), dtype=torch.uint8,
                           device="cuda")

        def step(i, x=x, out=out, work=work):
            a, b, c = sets[i % copies]
            bq.bq_linear_w4_grouped(x, a, b, c, gs, bias, out=out, workspace=work)

        ms, _ = graph_time(step, steps, 3)
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

    ms, _ = graph_time(step, steps, 3)
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

    ms_aq, _ = graph_time(aq, steps, 3)
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

    ms, _ = graph_time(step, steps, 3)
    res["bitlinear_tiny"] = {"us_per_step": round(ms * 1e3, 3), "config": "x fp32 [8,256], W [128,256]"}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the headline workload
# ---------------------------------------------------------------------------
def oracle_sample(d, rows: int):
    import oracle
    sel = np.arange(rows)
    t0 = time.perf_counter()
    oracle.gemm_i8_pertoken(d["x"][sel], d["w"], d["deq_scale"], d["per_token_scale"][sel])
    return time.perf_counter() - t0


def cpu_baseline(d, rows: int = 0):
    import oracle
    oracle.build()
    if rows <= 0:
        t = oracle_sample(d, 2)
        rows = int(max(2, min(4096, round(2 * 10.0 / max(t, 1e-6)))))
    t = oracle_sample(d, rows)
    ops = 2.0 * rows * HEAD["N"] * HEAD["K"]
    return {"value": round(ops / t / 1e12, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
            "sample": f"{rows} of 4096 rows of the 4096^3 W8A8 GEMM (all 4096 columns), {t:.1f} s, one thread"}


def reference_arm(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    import oracle
    import synth
    oracle.build()
    d = synth.gemm_w8a8(**HEAD)
    rows = max(1, args.cpu_rows or 4)
    for _ in range(args.warmup):
        oracle_sample(d, rows)
    t = sum(oracle_sample(d, rows) for _ in range(args.steps))
    ops = 2.0 * rows * HEAD["N"] * HEAD["K"] * args.steps
    value = ops / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "config": {"workload": HEAD_WORKLOAD, **HEAD, "sample_rows_per_step": rows},
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
                             "sample": f"{rows} rows x 4096 columns per step, plain C double/int64 loops"},
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
        base = cpu_baseline(d, args.cpu_rows)
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
