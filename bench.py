#!/usr/bin/env python3
"""Throughput of the W4A16 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl w4|reference] [--workload NAME]

One step is one pass of the workload's kernels over one batch of its inputs.
The product workloads (decode, smallbatch, prefill) multiply every activation
batch by its packed weight (w4a16_gemm); their weights are quantized once,
before the timed region, as a model's weights are at load time, and the
GEMV-sized products are launched with W4_WEIGHTS_STATIC (the weight stream of
one product may start before the previous kernel on the stream finishes).
The quantizer workloads time the quantization itself.

  decode (default)  M=1, K=4096, N in {4096, 11008, 12288}, asymmetric INT4 g=128:
                    3 x w4a16_gemm (GEMV); value = algorithmic GB/s
  smallbatch        K=8192, N=28672, symmetric g=128: w4a16_gemm at M in {2,4,8,16,32}
  prefill           K=4096, N=14336, asymmetric g=128: w4a16_gemm at M in {512,2048,8192};
                    value = GEMM TFLOP/s over the step
  quantizer         w4_quant_pack of W[28672, 8192]: g in {32,64,128} x {sym, asym} + smoothing fold
  decodequant       w4_quant_pack of the decode weights (K=4096, N in {4096, 11008, 12288}, asym g=128)
  awq               the AWQ scale search over W[4096, 4096] with 128 calibration rows
  fp4quant          W[28672, 8192] to NVFP4 and to MXFP4: 2 x w4_fp4_quant per step
  mxdecode          the decode layers with MXFP4 weights and MXFP8 activations: per layer
                    w4_mxfp8_quant + w4_mx_gemm (block-scaled tcgen05); value = algorithmic GB/s

The K timed steps are captured in one CUDA graph (kernel nodes only) and
replayed once between CUDA events on the launching stream.  Inputs rotate over
enough copies that no kernel finds its inputs in the 126 MB L2 (one sweep of
the copies is more than 3x L2).
Each kernel's device time is measured the same way, live: the median (and min)
over five replays of a graph of max(K, 100) launches of that kernel alone over
enough copies of its inputs (one sweep > 3x L2) that every launch reads them
from HBM.  (An event-record node between kernels
inside the step graph would cost several microseconds per kernel.)

Under torchrun (N > 1) every rank runs its own replica with its own seeds
(weak scaling, no collective on the data path); the timed region is bracketed
by barriers and the reported time is the max over ranks.  With --shard n|k the
product workloads scale strongly instead: every layer is split over the ranks
(bit_gemm_quant_b200.shard), and a step includes the collective that
completes Y.  Rank 0 prints one
JSON line.  ``--impl reference`` times the CPU oracle on a bounded sample of
the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_gemm_quant_b200 import roofline, synth  # noqa: E402

METRIC = "W4A16 g128 GEMV HBM GB/s (% peak); GEMM TFLOPS (% peak); quant-pack GB/s"
KERNEL_SOURCES = {"w4_quant_pack": "quant_pack.cu", "w4a16_gemv": "gemv.cu", "w4a16_gemm_tc": "gemm_tc.cu",
                  "w4_fp4_quant": "fp4_quant.cu", "w4_mx_gemm": "mx_gemm.cu", "w4_mxfp8_quant": "mx_quant.cu"}
THROTTLE_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["w4", "reference"], default="w4")
    ap.add_argument("--workload", choices=["decode", "smallbatch", "prefill", "quantizer", "decodequant", "awq", "fp4quant",
                                               "mxdecode"],
                    default="decode")
    ap.add_argument("--shard", choices=["none", "n", "k"], default="none",
                    help="strong scaling of the product workloads: split every layer over the ranks by rows of W "
                         "(n, all-gather of Y) or by columns (k, all-reduce of fp32 partials); default: replicas")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- ranks --

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def aggregate(local_ms: float, local_units: float, device=None):
    """Max of the timed milliseconds and sum of the work units over all ranks."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return local_ms, local_units
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    u = torch.tensor([float(local_units)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------ workloads --

def problems_for(workload: str):
    """Problems of a workload and how their weights are shared.

    Returns a list of (weight_key, Problem); problems with the same key use one
    quantization of one weight matrix per step."""
    probs = synth.workload(workload)
    if workload == "decode":
        return [(p.name, p) for p in probs]
    if workload in ("smallbatch", "prefill"):
        return [(workload + "_W", p) for p in probs]
    return [(p.name, p) for p in probs]


WORKLOAD_DESC = {
    "decode": "decode GEMV: M=1, K=4096, N in {4096,11008,12288}, asymmetric INT4 g=128, fp16 scales, uint4 zero-points; "
              "step = 3 w4a16_gemm (GEMV, W4_WEIGHTS_STATIC), weights quantized once before timing",
    "smallbatch": "small-batch decode: K=8192, N=28672, symmetric INT4 g=128, M in {2,4,8,16,32}; "
                  "step = 5 w4a16_gemm (W4_WEIGHTS_STATIC where M <= 16), weights quantized once before timing",
    "prefill": "prefill GEMM: K=4096, N=14336, asymmetric INT4 g=128, M in {512,2048,8192}; step = 3 w4a16_gemm "
               "(tensor cores), weights quantized once before timing",
    "quantizer": "quantizer sweep: W[28672,8192], g in {32,64,128} x {sym,asym} + smoothing fold; step = 7 w4_quant_pack",
    "decodequant": "quantizer on the decode weights: W[N,4096] bf16, N in {4096,11008,12288}, asymmetric INT4 g=128; "
                   "step = 3 w4_quant_pack",
    "fp4quant": "block-scaled FP4 weight quantization: W[28672,8192] bf16 to NVFP4 (E2M1, E4M3 scale per 16) and "
                "to MXFP4 (E2M1, E8M0 scale per 32); step = 2 w4_fp4_quant",
    "mxdecode": "MX decode: M=1, K=4096, N in {4096,11008,12288}, MXFP4 weights (E2M1, E8M0 scale per 32) x MXFP8 "
                "activations (E4M3, E8M0 scale per 32); step = per layer w4_mxfp8_quant + w4_mx_gemm "
                "(tcgen05.mma kind::mxf8f6f4, W4_WEIGHTS_STATIC), weights quantized once before timing",
}


def awq_desc(M, N, K, g, na):
    return ("AWQ scale search: W[%d,%d] bf16, X[%d,%d] calibration rows with 1%% outlier channels x20, "
            "asymmetric INT4 g=%d, %d alphas; step = one whole search" % (N, K, M, K, g, na))


def kernel_name(M: int) -> str:
    return "w4a16_gemv" if M <= 16 else "w4a16_gemm_tc"


class Launch:
    def __init__(self, name, work_bytes, flops, label):
        self.name, self.bytes, self.flops, self.label = name, work_bytes, flops, label


# ------------------------------------------------------------ clocks ----

class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.t_begin = self.t_end = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="w4clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def mark_begin(self):
        self.t_begin = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvidia-smi unavailable"}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        os.unlink(self.path)
        win = [r for r in rows if self.t_begin is not None and self.t_begin - 1 <= r[0] <= self.t_end + 1] or rows
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in win for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in win), "sm_max_mhz": max(r[2] for r in win),
                "reasons": reasons, "samples": len(win), "window": "sustained load before and during the timed replay"}


def smi_gpu_id(local_rank: int) -> str:
    """nvidia-smi index of this rank's device (honours CUDA_VISIBLE_DEVICES)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------ traffic ---

def traffic_table() -> dict:
    """DRAM bytes per launch from the committed ncu summary, keyed by
    (kernel, problem); entries whose kernel source changed since are dropped."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    out = {}
    if not os.path.exists(path):
        return out
    shas = {}
    for k, src in KERNEL_SOURCES.items():
        p = os.path.join(ROOT, "bit_gemm_quant_b200", "csrc", src)
        if os.path.exists(p):
            shas[k] = hashlib.sha256(open(p, "rb").read()).hexdigest()[:12]
    for line in open(path):
        parts = line.split()
        if len(parts) != 4 or parts[0].startswith("#"):
            continue
        kern, label, sha, nbytes = parts
        if shas.get(kern) == sha:
            out[(kern, label)] = float(nbytes)
    return out


# ------------------------------------------------------------- our arm ---

QUANT_WORKLOADS = ("quantizer", "decodequant")


def run_w4(args, rank, world, local_rank):
    import torch
    import bit_gemm_quant_b200 as w4

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    w4.lib()
    pk = roofline.peaks(ROOT)
    plist = problems_for(args.workload)
    quant_step = args.workload in QUANT_WORKLOADS
    rank_seed = 1000 * rank
    L2_BYTES = 126 << 20

    # ---- inputs (host bits, then device) ----
    keys = list(dict.fromkeys(k for k, _ in plist))
    first = {k: p for k, p in reversed(plist)}
    qp = {k: first[k] for k in keys}              # the quantization problem of each weight key
    host_W = {k: [synth.weights(qp[k].seed + rank_seed, qp[k].N, qp[k].K, qp[k].w_std, *qp[k].w_outlier)]
              for k in keys}
    host_s = {k: qp[k].s() for k in keys}
    host_X = {p.name: [synth.activations(p.seed + rank_seed, p.M, p.K, *p.x_outlier, fixed_channels=p.x_fixed)]
              for _, p in plist if p.M > 0}

    def dev_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)

    W_d = {k: dev_bf16(host_W[k][0]) for k in keys}
    s_d = {k: (torch.from_numpy(host_s[k]).to(device) if host_s[k] is not None else None) for k in keys}
    X_d = {n: dev_bf16(v[0]) for n, v in host_X.items()}

    def copies_for(nbytes):
        return max(2, -(-3 * L2_BYTES // max(nbytes, 1)) + 1)   # reuse distance of one copy > 3x L2

    def packed_bytes(p):
        qs, ss, zs = w4.packed_shapes(p.N, p.K, p.group)
        return qs[0] * qs[1] * 4 + ss[0] * ss[1] * 2 + (zs[0] * zs[1] * 4 if p.mode == w4.ASYM else 0)

    launches = []
    if quant_step:
        # the quantizer reads each weight from one of several copies of W
        W_pool = {k: [W_d[k]] + [W_d[k].clone() for _ in range(copies_for(W_d[k].numel() * 2) - 1)] for k in keys}
        packed_out = {k: w4.quant_pack(W_d[k], qp[k].group, qp[k].mode, s=s_d[k]) for k in keys}
        for k in keys:
            p = qp[k]
            launches.append(Launch("w4_quant_pack", roofline.quant_pack_bytes(p.N, p.K, p.group, p.mode, p.smooth), 0, k))
    else:
        # weights quantized once, as at model load; each product of a step takes
        # the next of several copies of its packed weight
        packed0 = {k: w4.quant_pack(W_d[k], qp[k].group, qp[k].mode, s=s_d[k]) for k in keys}
        uses = {k: sum(1 for key, pp in plist if key == k and pp.M > 0) for k in keys}
        P_pool = {}
        for k in keys:
            n = max(copies_for(packed_bytes(qp[k]) * uses[k]), uses[k] + 1)
            P_pool[k] = [packed0[k]] + [tuple(None if t is None else t.clone() for t in packed0[k]) for _ in range(n - 1)]
        Y_d, ws_d = {}, {}
        for key, p in plist:
            if p.M > 0:
                Y_d[p.name] = torch.empty((p.M, p.N), dtype=torch.bfloat16, device=device)
                need = w4.w4a16_workspace_bytes(p.M, p.N, p.K, p.group)
                ws_d[p.name] = torch.zeros(max(need, 256), dtype=torch.uint8, device=device)
                launches.append(Launch(kernel_name(p.M), roofline.gemm_bytes(p.M, p.N, p.K, p.group, p.mode),
                                       roofline.gemm_flops(p.M, p.N, p.K), p.name))
    torch.cuda.synchronize()

    use_count = {k: 0 for k in keys}

    def step(si):
        if quant_step:
            for k in keys:
                p = qp[k]
                pool = W_pool[k]
                w4.quant_pack(pool[si % len(pool)], p.group, p.mode, s=s_d[k], out=packed_out[k])
            return
        for key, pp in plist:
            if pp.M > 0:
                pool = P_pool[key]
                q, sc, z = pool[use_count[key] % len(pool)]
                use_count[key] += 1
                w4.gemm(X_d[pp.name], q, sc, z, pp.group, pp.mode, N=pp.N, workspace=ws_d[pp.name],
                        out=Y_d[pp.name], weights_static=pp.M <= 16)

    per_step = len(launches)
    # ---- eager warm-up ----
    for si in range(max(3, args.warmup)):
        step(si)
    torch.cuda.synchronize()

    # ---- capture the K timed steps: kernels only, no nodes between them ----
    # (an event-record node inside a graph costs several microseconds, so the
    # per-kernel durations are taken from separate graphs below)
    K = args.steps
    graph = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream(device)
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cap_stream):
        for si in range(K):
            step(si)
    torch.cuda.synchronize()

    # ---- sustained load (untimed) so the clock samples cover a steady state ----
    sampler = ClockSampler(smi_gpu_id(local_rank))
    sampler.start()
    sampler.mark_begin()
    t_end = time.time() + 1.5
    replays = 0
    while time.time() < t_end or replays < 2:
        graph.replay()
        replays += 1
        torch.cuda.synchronize()

    def timed():
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        e1.synchronize()
        barrier()
        return e0.elapsed_time(e1)

    local_ms = timed()
    sampler.mark_end()
    clocks = sampler.stop()
    if any(r in clocks.get("reasons", []) for r in THROTTLE_REASONS):
        sampler = ClockSampler(sampler.gpu_id)
        sampler.start()
        sampler.mark_begin()
        local_ms = timed()
        sampler.mark_end()
        clocks = sampler.stop()
        clocks["remeasured"] = True
    del graph

    # ---- per-kernel device time: each launch of the step alone, KL times in one
    # graph, over enough copies of its inputs (> 3x L2) that every launch reads
    # them from HBM; CUDA events on the launching stream around the replay ----
    KL = max(K, 100)                             # launches per per-kernel graph
    REPLAYS = 5

    def kernel_graph_ms(fns):
        """Median and min over REPLAYS replays of the per-launch time of a graph
        of KL launches cycling over fns."""
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(device)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=cs):
            for i in range(KL):
                fns[i % len(fns)]()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        per = []
        for _ in range(REPLAYS):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(cs):
                e0.record(cs)
                g.replay()
                e1.record(cs)
            e1.synchronize()
            per.append(e0.elapsed_time(e1) / KL)
        del g
        return statistics.median(per), min(per)

    kt = {}
    RP_pool = {}
    for L in launches:
        if quant_step:
            p = qp[L.label]
            fns = [(lambda Wc=Wc, p=p, k=L.label: w4.quant_pack(Wc, p.group, p.mode, s=s_d[k], out=packed_out[k]))
                   for Wc in W_pool[L.label]]
            kt[(L.name, L.label)] = kernel_graph_ms(fns)
            continue
        pp = next(p for _, p in plist if p.name == L.label)
        key = next(k for k, p in plist if p.name == L.label)
        pool = P_pool[key]
        for static in ((True, False) if pp.M <= 16 else (False,)):
            fns = [(lambda Pc=Pc, pp=pp, static=static: w4.gemm(X_d[pp.name], Pc[0], Pc[1], Pc[2], pp.group, pp.mode,
                                                                 N=pp.N, workspace=ws_d[pp.name], out=Y_d[pp.name],
                                                                 weights_static=static))
                   for Pc in pool]
            kt[(L.name, L.label, static)] = kernel_graph_ms(fns)
        kt[(L.name, L.label)] = kt[(L.name, L.label, pp.M <= 16)]
        if pp.M <= 16 and pp.K % 256 == 0:
            # the same product on codes in the GEMV's box order (w4_repack, done offline)
            if key not in RP_pool:
                RP_pool[key] = [w4.repack(Pc[0], pp.N, pp.K) for Pc in pool]
            fns = [(lambda Pc=Pc, Rq=Rq, pp=pp: w4.gemm(X_d[pp.name], Rq, Pc[1], Pc[2], pp.group, pp.mode, N=pp.N,
                                                       out=Y_d[pp.name], weights_static=True, repacked=True))
                   for Pc, Rq in zip(pool, RP_pool[key])]
            kt[(L.name, L.label, "repacked")] = kernel_graph_ms(fns)
    torch.cuda.synchronize()

    step_bytes = sum(L.bytes for L in launches)
    step_flops = sum(L.flops for L in launches)
    work = K * (step_flops if args.workload == "prefill" else step_bytes)
    max_ms, total_work = aggregate(local_ms, work, device)

    if args.workload == "prefill":
        value, unit = total_work / (max_ms * 1e-3) / 1e12, "TFLOP/s"
    else:
        value, unit = total_work / (max_ms * 1e-3) / 1e9, "GB/s"

    # ---- per-kernel roofline ----
    traffic = traffic_table()

    def tensor_peak(avg_ms):
        """The measured cuBLAS bf16 peak that matches how the kernel was timed:
        the sustained (power-capped) figure when one replay of its timing graph
        ran for at least 50 ms of back-to-back launches, else the burst figure."""
        return pk["bf16_tflops_sustained"] if KL * avg_ms >= 50.0 else pk["bf16_tflops"]

    kernels = {}
    by_name = {}

    def entry(L, avg, mn):
        ent = {"launches": KL * REPLAYS, "avg_us": round(avg * 1e3, 3), "min_us": round(mn * 1e3, 3),
               "bytes": L.bytes,
               "gbs": round(L.bytes / (avg * 1e-3) / 1e9, 1),
               "hbm_frac": round(L.bytes / (avg * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        if L.flops:
            tf = L.flops / (avg * 1e-3) / 1e12
            peak_t = tensor_peak(avg)
            ent.update({"flops": L.flops, "tflops": round(tf, 1), "tensor_frac": round(tf / peak_t, 4),
                        "tensor_frac_burst": round(tf / pk["bf16_tflops"], 4)})
        return ent

    for L in launches:
        avg, mn = kt[(L.name, L.label)]
        kernels["%s[%s]" % (L.name, L.label)] = entry(L, avg, mn)
        if (L.name, L.label, False) in kt and (L.name, L.label, True) in kt:
            # the same launch without W4_WEIGHTS_STATIC: the weight stream waits
            # for the previous kernel to finish
            kernels["%s[%s]" % (L.name, L.label)]["weights_static"] = True
            a2, m2 = kt[(L.name, L.label, False)]
            e2 = entry(L, a2, m2)
            e2["weights_static"] = False
            kernels["%s_plain[%s]" % (L.name, L.label)] = e2
        if (L.name, L.label, "repacked") in kt:
            a3, m3 = kt[(L.name, L.label, "repacked")]
            e3 = entry(L, a3, m3)
            e3["weights_static"] = True
            e3["codes"] = "w4_repack layout (16-channel x 256-k boxes contiguous)"
            kernels["%s_repacked[%s]" % (L.name, L.label)] = e3
        by_name.setdefault(L.name, []).append((L, [avg] * KL))

    dom = max(by_name, key=lambda n: sum(sum(ts) for _, ts in by_name[n]))
    dom_launches = by_name[dom]
    tot_time = sum(sum(ts) for _, ts in dom_launches) * 1e-3
    nlaunch = sum(len(ts) for _, ts in dom_launches)
    if dom == "w4a16_gemm_tc":
        per_launch = sum(L.flops * len(ts) for L, ts in dom_launches) / nlaunch
        avg_launch_ms = tot_time * 1e3 / nlaunch
        # sustained only if every launch of the kernel was timed in that regime
        peak = max(tensor_peak(kt[(L.name, L.label)][0]) for L, _ in dom_launches)
        achieved = per_launch / (tot_time / nlaunch) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "frac_of_burst": round(achieved / pk["bf16_tflops"], 4),
                "peak_regime": "sustained" if peak == pk["bf16_tflops_sustained"] else "burst",
                "avg_launch_ms": round(avg_launch_ms, 4)}
    else:
        per_launch = sum(L.bytes * len(ts) for L, ts in dom_launches) / nlaunch
        achieved = per_launch / (tot_time / nlaunch) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4)}
    if dom == "w4a16_gemv":
        roof["weights_static"] = True
        plain = [kt[(L.name, L.label, False)][0] for L, _ in dom_launches]
        roof["frac_plain"] = round(per_launch / (sum(plain) / len(plain) * 1e-3) / 1e9 / pk["hbm_gbs"], 4)
        rep = [kt.get((L.name, L.label, "repacked")) for L, _ in dom_launches]
        if all(r is not None for r in rep):
            roof["frac_repacked"] = round(per_launch / (sum(r[0] for r in rep) / len(rep) * 1e-3) / 1e9
                                          / pk["hbm_gbs"], 4)
    tr = [traffic.get((dom, L.label)) for L, _ in dom_launches]
    roof["traffic"] = (sum(tr) / len(tr)) if tr and all(t is not None for t in tr) else None
    roof["kernel"] = dom
    roof["peak_source"] = "%s (%s)" % (pk["source"], "MEASURED_PEAKS.json" if pk["source"] == "measured" else "recipe")
    roof["algorithmic_per_launch"] = per_launch

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(w4, torch, device, plist, keys, qp, host_W, host_X, host_s, min(args.steps, 10), quant_step)
        e2e_ms, e2e_work = aggregate(e2e["ms"], e2e["work"] if args.workload != "prefill" else e2e["flops"], device)
        e2e = {"value": round(e2e_work / (e2e_ms * 1e-3) / (1e12 if args.workload == "prefill" else 1e9), 2),
               "unit": unit, "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
               "steps": e2e["steps"], "what": e2e["what"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, plist, keys, qp, host_W, host_X, host_s, args.cpu_budget, quant_step)

    if rank == 0:
        wl_desc = WORKLOAD_DESC[args.workload]
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": round(max_ms / K, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl_desc, "codes": "int4 packed 8 per uint32", "accumulate": "fp32",
                       "l2": "every launch reads its weight from one of several copies whose reuse distance exceeds 3x L2",
                       "timing": "K steps captured in one CUDA graph (kernels only), replayed between CUDA events on the launching stream after %d untimed replays; max over ranks; per-kernel durations: median (and min) over 5 replays of a graph of max(K, 100) launches of that kernel alone over rotating input copies (one sweep > 3x L2), between CUDA events on its stream" % replays,
                       "parallelism": "replicas (dp%d), no data-path collective" % world},
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": K * per_step * world, "clocks": clocks,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(w4, torch, device, plist, keys, qp, host_W, host_X, host_s, steps, quant_step):
    """The step through the tensor API with pinned host buffers, all timed.
    Quantizer workloads: host->device copies of W (and s), the quantization and
    device->host copies of the packed weight.  Product workloads: the weights
    are quantized once, untimed (model state); each step copies the
    activations host->device, multiplies, and copies Y device->host."""
    pin = lambda a: torch.from_numpy(a.view(np.int16)).pin_memory()
    h2d = d2h = 0
    if quant_step:
        hW = {k: pin(host_W[k][0]) for k in keys}
        hs = {k: (torch.from_numpy(host_s[k]).pin_memory() if host_s[k] is not None else None) for k in keys}
        outs_q = {}
        for k in keys:
            p = qp[k]
            qs, ss, zs = w4.packed_shapes(p.N, p.K, p.group)
            outs_q[k] = (torch.empty(qs, dtype=torch.int32).pin_memory(),
                         torch.empty(ss, dtype=torch.float16).pin_memory(),
                         torch.empty(zs, dtype=torch.int32).pin_memory() if p.mode == 1 else None)
            h2d += hW[k].numel() * 2 + (hs[k].numel() * 4 if hs[k] is not None else 0)
            d2h += sum(t.numel() * t.element_size() for t in outs_q[k] if t is not None)
        work = sum(roofline.quant_pack_bytes(qp[k].N, qp[k].K, qp[k].group, qp[k].mode, qp[k].smooth) for k in keys)
        flops = 0

        def one():
            for k in keys:
                p = qp[k]
                Wd = hW[k].to(device, non_blocking=True).view(torch.bfloat16)
                sd = hs[k].to(device, non_blocking=True) if hs[k] is not None else None
                for t_h, t_d in zip(outs_q[k], w4.quant_pack(Wd, p.group, p.mode, s=sd)):
                    if t_h is not None:
                        t_h.copy_(t_d, non_blocking=True)
        what = "H2D of W (and s), w4_quant_pack, D2H of the packed weight"
    else:
        packed = {}
        for k in keys:
            p = qp[k]
            Wd = torch.from_numpy(host_W[k][0].view(np.int16)).to(device).view(torch.bfloat16)
            sd = torch.from_numpy(host_s[k]).to(device) if host_s[k] is not None else None
            packed[k] = w4.quant_pack(Wd, p.group, p.mode, s=sd)
        hX = {n: pin(v[0]) for n, v in host_X.items()}
        outs_y = {}
        for key, p in plist:
            if p.M > 0:
                outs_y[p.name] = torch.empty((p.M, p.N), dtype=torch.bfloat16).pin_memory()
                h2d += hX[p.name].numel() * 2
                d2h += p.M * p.N * 2
        work = sum(roofline.gemm_bytes(p.M, p.N, p.K, p.group, p.mode) for _, p in plist if p.M > 0)
        flops = sum(roofline.gemm_flops(p.M, p.N, p.K) for _, p in plist if p.M > 0)

        def one():
            for key, pp in plist:
                if pp.M > 0:
                    q, sc, z = packed[key]
                    Xd = hX[pp.name].to(device, non_blocking=True).view(torch.bfloat16)
                    Y = w4.gemm(Xd, q, sc, z, pp.group, pp.mode, N=pp.N)
                    outs_y[pp.name].copy_(Y, non_blocking=True)
        what = "H2D of X, w4a16_gemm, D2H of Y (packed weights resident, quantized once before timing)"

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    e1.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    return {"ms": ms, "work": work * steps, "flops": flops * steps, "h2d": h2d, "d2h": d2h, "steps": steps,
            "what": what}


# ------------------------------------------------------- oracle (CPU) ---

def oracle_prepare(oracle, keys, qp, host_W, host_s, rows_per_weight: int, offset: int = 0, threads: int = 1):
    """Quantize rows [offset, offset + r) of each weight with the oracle and
    dequantize them (the product workloads' model state, not timed)."""
    out = {}
    for k in keys:
        p = qp[k]
        r0 = offset % p.N
        r1 = min(p.N, r0 + rows_per_weight)
        q, sc, z = oracle.quant_pack(host_W[k][0], p.group, p.mode, s=host_s[k], rows=(r0, r1), threads=threads)
        out[k] = oracle.dequant(q, sc, z, p.K, p.group, p.mode, rows=(r0, r1), threads=threads), r1 - r0
    return out


def oracle_sample(oracle, plist, keys, qp, host_W, host_X, host_s, rows_per_weight: int, offset: int = 0,
                  threads: int = 1, quant_step: bool = False, prepared=None):
    """The oracle's share of one step on rows [offset, offset + r) of each
    weight: quantize and pack them (quantizer workloads), or the fp64 product
    of the activations with those output channels of the dequantized weight
    (product workloads; ``prepared`` from oracle_prepare).  Returns the
    algorithmic bytes (or flops) processed."""
    nbytes = 0
    nflops = 0
    for k in keys:
        p = qp[k]
        if quant_step:
            r0 = offset % p.N
            r1 = min(p.N, r0 + rows_per_weight)
            oracle.quant_pack(host_W[k][0], p.group, p.mode, s=host_s[k], rows=(r0, r1), threads=threads)
            nbytes += roofline.quant_pack_bytes(r1 - r0, p.K, p.group, p.mode, p.smooth)
            continue
        what, nr = prepared[k]
        for pp in (pp for key, pp in plist if key == k and pp.M > 0):
            oracle.gemm_f64(host_X[pp.name][0], what, threads=threads)
            nbytes += roofline.gemm_bytes(pp.M, nr, pp.K, pp.group, pp.mode)
            nflops += roofline.gemm_flops(pp.M, nr, pp.K)
    return nbytes, nflops


def cpu_baseline(workload, plist, keys, qp, host_W, host_X, host_s, budget_s, quant_step):
    import oracle
    oracle.build()
    rate = lambda nb, nf, t: nf / t / 1e12 if workload == "prefill" else nb / t / 1e9
    unit = "TFLOP/s" if workload == "prefill" else "GB/s"
    maxrows = max(p.N for p in qp.values())

    def timed(rows, threads):
        prep = None if quant_step else oracle_prepare(oracle, keys, qp, host_W, host_s, rows, threads=threads)
        t0 = time.perf_counter()
        nb, nf = oracle_sample(oracle, plist, keys, qp, host_W, host_X, host_s, rows, threads=threads,
                               quant_step=quant_step, prepared=prep)
        return nb, nf, time.perf_counter() - t0

    _, _, dt = timed(4, 1)
    rows = min(maxrows, max(4, int(4 * budget_s / max(dt, 1e-3))))
    nbytes, nflops, dt = timed(rows, 1)
    what = ("oracle fold+quantize+pack" if quant_step else
            "oracle fp64 product of the activations with those output channels of the dequantized weight "
            "(quantized by the oracle beforehand, untimed)")
    out = {"value": rate(nbytes, nflops, dt), "unit": unit, "cores": 1, "kind": "oracle", "seconds": round(dt, 2),
           "sample": "first %d rows of each weight of the workload: %s, single thread" % (rows, what)}
    cores = os.cpu_count() or 1
    if cores > 1:
        # the same oracle with its row slices spread over every host core
        rows_mc = min(rows * cores, maxrows)
        nb_mc, nf_mc, dt_mc = timed(rows_mc, cores)
        out["all_cores"] = {"value": rate(nb_mc, nf_mc, dt_mc), "unit": unit, "cores": cores,
                            "seconds": round(dt_mc, 2),
                            "sample": "first %d rows of each weight, the oracle's row slices on %d threads"
                                      % (rows_mc, cores)}
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    oracle.build()
    if args.workload == "awq":
        return run_reference_awq(args, world)
    if args.workload == "fp4quant":
        return run_reference_fp4(args, world)
    if args.workload in MX_WORKLOADS:
        return run_reference_mx(args, world)
    plist = problems_for(args.workload)
    keys = list(dict.fromkeys(k for k, _ in plist))
    first = {k: p for k, p in reversed(plist)}
    qp = {k: first[k] for k in keys}
    quant_step = args.workload in QUANT_WORKLOADS
    host_W = {k: [synth.weights(qp[k].seed, qp[k].N, qp[k].K, qp[k].w_std, *qp[k].w_outlier)] for k in keys}
    host_s = {k: qp[k].s() for k in keys}
    host_X = {p.name: [p.X()] for _, p in plist if p.M > 0}
    rows = 8
    steps_total = max(3, args.warmup) + args.steps
    # the product workloads' model state: every sampled row quantized and
    # dequantized by the oracle before timing
    prep = {} if quant_step else {
        si: oracle_prepare(oracle, keys, qp, host_W, host_s, rows, si * rows) for si in range(steps_total)}
    for si in range(max(3, args.warmup)):
        oracle_sample(oracle, plist, keys, qp, host_W, host_X, host_s, rows, si * rows, quant_step=quant_step,
                      prepared=prep.get(si))
    nb = nf = 0
    t0 = time.perf_counter()
    for j in range(args.steps):
        si = max(3, args.warmup) + j
        b, f = oracle_sample(oracle, plist, keys, qp, host_W, host_X, host_s, rows, si * rows, quant_step=quant_step,
                             prepared=prep.get(si))
        nb, nf = nb + b, nf + f
    dt = time.perf_counter() - t0
    if args.workload == "prefill":
        val, unit = nf / dt / 1e12, "TFLOP/s"
    else:
        val, unit = nb / dt / 1e9, "GB/s"
    what = ("oracle fold+quantize+pack" if quant_step else
            "oracle fp64 product with those output channels of the dequantized weight (quantized by the oracle "
            "before timing)")
    sample = "%d rows of each weight per step (rotating): %s, single thread" % (rows, what)
    print_reference(args, world, val, unit, dt * 1e3 / args.steps, WORKLOAD_DESC[args.workload], sample)


def print_reference(args, world, val, unit, ms_per_step, desc, sample):
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": unit, "n_gpus": world,
           "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64",
           "data": "synthetic", "config": {"workload": desc, "kind": "CPU oracle on a bounded sample"},
           "cpu_baseline": {"value": val, "unit": unit, "cores": 1, "kind": "oracle", "sample": sample},
           "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_reference_awq(args, world):
    """The oracle's AWQ search over the first `rows` output channels of the
    bench's layer (all 20 alphas, all calibration rows), single thread; the
    algorithmic bytes are those of a search over that many channels."""
    import oracle.awq as oawq
    sh = AWQ_SHAPE
    M, N, K, g, mode, na = sh["M"], sh["N"], sh["K"], sh["group"], sh["mode"], sh["n_alpha"]
    rows = 8
    W = synth.weights(21, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(22, M, K, 0.01, 20.0)
    for si in range(max(3, args.warmup)):
        oawq.awq_losses(W[(si * rows) % N:(si * rows) % N + rows], X, g, mode, na)
    t0 = time.perf_counter()
    for si in range(args.steps):
        r0 = (si * rows) % N
        oawq.awq_losses(W[r0:r0 + rows], X, g, mode, na)
    dt = time.perf_counter() - t0
    val = args.steps * awq_bytes(M, rows, K, g, mode, na) / dt / 1e9
    sample = ("the search over %d output channels per step (rotating), all %d calibration rows and %d alphas: "
              "oracle fold+quantize+pack, dequantize, fp64 products and losses, single thread" % (rows, M, na))
    print_reference(args, world, val, "GB/s", dt * 1e3 / args.steps, awq_desc(M, N, K, g, na), sample)


def run_reference_fp4(args, world):
    """The oracle's NVFP4 and MXFP4 quantizers on `rows` rows of the bench's
    weight per step (rotating), single thread."""
    import oracle
    N, K = FP4_SHAPE["N"], FP4_SHAPE["K"]
    rows = 16
    W = fp4_weight(0)
    for si in range(max(3, args.warmup)):
        oracle_fp4_sample(oracle, W, rows, si * rows)
    nb = 0
    t0 = time.perf_counter()
    for si in range(args.steps):
        nb += oracle_fp4_sample(oracle, W, rows, si * rows)
    dt = time.perf_counter() - t0
    sample = "%d rows of W[%d,%d] per step (rotating), NVFP4 and MXFP4, oracle, single thread" % (rows, N, K)
    print_reference(args, world, nb / dt / 1e9, "GB/s", dt * 1e3 / args.steps, WORKLOAD_DESC["fp4quant"], sample)


# ------------------------------------------------------------ awq search --

AWQ_SHAPE = dict(M=128, N=4096, K=4096, group=128, mode=1, n_alpha=20)


def awq_bytes(M, N, K, group, mode, n_alpha):
    """Algorithmic bytes of one search: per alpha a folded quantization and a
    W4A16 product (plus X/s), once the reference product W X^T."""
    per_alpha = (roofline.quant_pack_bytes(N, K, group, mode, True) + roofline.gemm_bytes(M, N, K, group, mode)
                 + 4 * M * K + 6 * M * N)
    return n_alpha * per_alpha + 2 * M * K + 2 * N * K + 4 * M * N


def run_awq(args, rank, world, local_rank):
    """The AWQ scale search (page 2, AWQ section) over a decode-sized layer and
    128 calibration rows with 1% outlier input channels; one step is one whole
    search (20 alphas)."""
    import torch
    import bit_gemm_quant_b200 as w4

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    w4.lib()
    pk = roofline.peaks(ROOT)
    sh = AWQ_SHAPE
    M, N, K, g, mode, na = sh["M"], sh["N"], sh["K"], sh["group"], sh["mode"], sh["n_alpha"]
    W = torch.from_numpy(synth.weights(21 + 1000 * rank, N, K, 0.02, 0.01, 5.0).view(np.int16)).to(device)
    X = torch.from_numpy(synth.activations(22 + 1000 * rank, M, K, 0.01, 20.0).view(np.int16)).to(device)
    W, X = W.view(torch.bfloat16), X.view(torch.bfloat16)
    need = w4.w4_awq_workspace_bytes(M, N, K, g, mode, na)
    ws = torch.empty(need, dtype=torch.uint8, device=device)
    losses = torch.empty(na, dtype=torch.float64, device=device)
    best = torch.empty(1, dtype=torch.int32, device=device)
    s_best = torch.empty(K, dtype=torch.float32, device=device)

    def step():
        st = w4.w4_awq_search(w4._ptr(W), w4._ptr(X), N, K, M, g, mode, na, w4._ptr(losses), w4._ptr(best),
                              w4._ptr(s_best), w4._ptr(ws), need, w4._stream_handle(None))
        if st != w4.W4_OK:
            raise w4.W4Error(st, "w4_awq_search")

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    K_steps = args.steps
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(device)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cs):
        for _ in range(K_steps):
            step()
    torch.cuda.synchronize()
    sampler = ClockSampler(smi_gpu_id(local_rank))
    sampler.start()
    sampler.mark_begin()
    t_end = time.time() + 1.5
    while time.time() < t_end:
        graph.replay()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    e1.synchronize()
    barrier()
    local_ms = e0.elapsed_time(e1)
    sampler.mark_end()
    clocks = sampler.stop()
    del graph
    work = K_steps * awq_bytes(M, N, K, g, mode, na)
    max_ms, total = aggregate(local_ms, work, device)
    value = total / (max_ms * 1e-3) / 1e9
    per_search_s = max_ms * 1e-3 / K_steps
    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K_steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(max_ms / K_steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": awq_desc(M, N, K, g, na),
                       "timing": "K searches captured in one CUDA graph, replayed between CUDA events after 1.5 s "
                                 "of untimed replays; max over ranks",
                       "parallelism": "replicas (dp%d), no data-path collective" % world},
            "roofline": {"bound": "hbm", "achieved": round(value / world, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(value / world / pk["hbm_gbs"], 4), "traffic": None,
                         "kernel": "w4_awq_search (whole search)",
                         "algorithmic_per_launch": awq_bytes(M, N, K, g, mode, na)},
            "searches_per_s": round(world / per_search_s, 2),
            "best_alpha_index": int(best.cpu().numpy()[0]),
            "cpu_baseline": None, "e2e": None,
            "gpu_launches": K_steps * (4 + na * 3 + 2) * world, "clocks": clocks,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------- FP4 quantization --

FP4_SHAPE = dict(N=28672, K=8192)
FP4_KINDS = (("nvfp4", 0, 16), ("mxfp4", 1, 32))


def fp4_weight(rank_seed: int) -> np.ndarray:
    """The quantizer sweep's weight: W[28672, 8192] ~ N(0, 0.02^2), bf16 bits."""
    return synth.weights(4 + rank_seed, FP4_SHAPE["N"], FP4_SHAPE["K"], 0.02)


def fp4_step_bytes() -> int:
    N, K = FP4_SHAPE["N"], FP4_SHAPE["K"]
    return sum(roofline.fp4_quant_bytes(N, K, B) for _, _, B in FP4_KINDS)


def oracle_fp4_sample(oracle, W, rows: int, offset: int) -> int:
    """Both oracle quantizers on rows [offset, offset + rows) of W; returns the
    algorithmic bytes processed."""
    N, K = W.shape
    r0 = offset % N
    r1 = min(N, r0 + rows)
    nb = 0
    for _, kind, B in FP4_KINDS:
        oracle.fp4_quant(W[r0:r1], kind)
        nb += roofline.fp4_quant_bytes(r1 - r0, K, B)
    return nb


def run_fp4(args, rank, world, local_rank):
    """Block-scaled FP4 weight quantization of the quantizer sweep's weight
    (W[28672, 8192], 470 MB, larger than L2, so every launch reads it from
    HBM): one step is its NVFP4 and its MXFP4 quantization."""
    import torch
    import bit_gemm_quant_b200 as w4

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    w4.lib()
    pk = roofline.peaks(ROOT)
    N, K = FP4_SHAPE["N"], FP4_SHAPE["K"]
    host_W = fp4_weight(1000 * rank)
    W = torch.from_numpy(host_W.view(np.int16)).to(device).view(torch.bfloat16)
    outs = {name: w4.fp4_quant(W, kind) for name, kind, _ in FP4_KINDS}

    def step():
        for name, kind, _ in FP4_KINDS:
            w4.fp4_quant(W, kind, out=outs[name])

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    K_steps = args.steps
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(device)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cs):
        for _ in range(K_steps):
            step()
    torch.cuda.synchronize()
    sampler = ClockSampler(smi_gpu_id(local_rank))
    sampler.start()
    sampler.mark_begin()
    t_end = time.time() + 1.5
    replays = 0
    while time.time() < t_end or replays < 2:
        graph.replay()
        replays += 1
        torch.cuda.synchronize()

    def timed():
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(cs):
            e0.record(cs)
            graph.replay()
            e1.record(cs)
        e1.synchronize()
        barrier()
        return e0.elapsed_time(e1)

    local_ms = timed()
    sampler.mark_end()
    clocks = sampler.stop()
    if any(r in clocks.get("reasons", []) for r in THROTTLE_REASONS):
        sampler = ClockSampler(sampler.gpu_id)
        sampler.start()
        sampler.mark_begin()
        local_ms = timed()
        sampler.mark_end()
        clocks = sampler.stop()
        clocks["remeasured"] = True
    del graph

    # each kind alone: a graph of KL launches between CUDA events on its stream,
    # median and min over 5 replays (W is 470 MB, so every launch reads it from HBM)
    KL = max(K_steps, 20)
    kernels = {}
    for name, kind, B in FP4_KINDS:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            for _ in range(KL):
                w4.fp4_quant(W, kind, out=outs[name])
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        per = []
        for _ in range(5):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(cs):
                e0.record(cs)
                g.replay()
                e1.record(cs)
            e1.synchronize()
            per.append(e0.elapsed_time(e1) / KL)
        del g
        avg, mn = statistics.median(per), min(per)
        nbytes = roofline.fp4_quant_bytes(N, K, B)
        kernels["w4_fp4_quant[%s]" % name] = {
            "launches": KL * 5, "avg_us": round(avg * 1e3, 3), "min_us": round(mn * 1e3, 3), "bytes": nbytes,
            "gbs": round(nbytes / (avg * 1e-3) / 1e9, 1),
            "hbm_frac": round(nbytes / (avg * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}

    work = K_steps * fp4_step_bytes()
    max_ms, total = aggregate(local_ms, work, device)
    value = total / (max_ms * 1e-3) / 1e9
    # the roofline entry is the kernel over both kinds: bytes per launch averaged
    # over the two launches of a step, divided by their average duration
    tot_us = sum(v["avg_us"] for v in kernels.values())
    per_launch = fp4_step_bytes() / len(FP4_KINDS)
    achieved = per_launch / (tot_us * 1e-6 / len(FP4_KINDS)) / 1e9
    traffic = traffic_table()
    tr = [traffic.get(("w4_fp4_quant", name)) for name, _, _ in FP4_KINDS]
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4),
            "traffic": (sum(tr) / len(tr)) if all(t is not None for t in tr) else None,
            "kernel": "w4_fp4_quant", "algorithmic_per_launch": per_launch,
            "peak_source": "%s (%s)" % (pk["source"], "MEASURED_PEAKS.json" if pk["source"] == "measured"
                                        else "recipe")}

    e2e = None
    if not args.no_e2e:
        e2e = fp4_e2e(w4, torch, device, host_W, min(K_steps, 5))
        e_ms, e_work = aggregate(e2e["ms"], e2e["work"], device)
        e2e = {"value": round(e_work / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["steps"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_fp4(host_W, args.cpu_budget)

    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K_steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(max_ms / K_steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC["fp4quant"],
                       "l2": "the 470 MB weight is larger than L2; every launch reads it from HBM",
                       "timing": "K steps captured in one CUDA graph, replayed between CUDA events on the launching "
                                 "stream after %d untimed replays; max over ranks" % replays,
                       "parallelism": "replicas (dp%d), no data-path collective" % world},
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": K_steps * len(FP4_KINDS) * world, "clocks": clocks,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def cpu_baseline_fp4(host_W, budget_s):
    """Both oracle quantizers on the first rows of the weight, single thread,
    sized to about ``budget_s`` seconds."""
    import oracle
    oracle.build()
    N, K = host_W.shape
    t0 = time.perf_counter()
    oracle_fp4_sample(oracle, host_W, 16, 0)
    dt = time.perf_counter() - t0
    rows = min(N, max(16, int(16 * budget_s / max(dt, 1e-3))))
    t0 = time.perf_counter()
    nb = oracle_fp4_sample(oracle, host_W, rows, 0)
    dt = time.perf_counter() - t0
    return {"value": nb / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle", "seconds": round(dt, 2),
            "sample": "first %d rows of W[%d,%d], NVFP4 and MXFP4, oracle, single thread" % (rows, N, K)}


def fp4_e2e(w4, torch, device, host_W, steps):
    """Both quantizations through the tensor API from a pinned host weight:
    the host->device copy of W, the two calls and the device->host copies of
    the codes and scales, all timed."""
    hW = torch.from_numpy(host_W.view(np.int16)).pin_memory()
    N, K = host_W.shape
    h_out = {name: (torch.empty((N, K // 2), dtype=torch.uint8).pin_memory(),
                    torch.empty((N, K // B), dtype=torch.uint8).pin_memory()) for name, _, B in FP4_KINDS}
    d2h = sum(c.numel() + s.numel() for c, s in h_out.values())

    def one():
        Wd = hW.to(device, non_blocking=True).view(torch.bfloat16)
        for name, kind, _ in FP4_KINDS:
            c, s = w4.fp4_quant(Wd, kind)
            h_out[name][0].copy_(c, non_blocking=True)
            h_out[name][1].copy_(s, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    e1.synchronize()
    barrier()
    return {"ms": e0.elapsed_time(e1), "work": fp4_step_bytes() * steps, "h2d": hW.numel() * 2, "d2h": d2h,
            "steps": steps}


# ------------------------------------------------------------ MX product --

MX_WORKLOADS = ("mxdecode",)
MXFP4_KIND = 1


def mx_step_bytes(probs) -> int:
    return sum(roofline.mxfp8_quant_bytes(p.M, p.K) + roofline.mx_gemm_bytes(p.M, p.N, p.K) for p in probs)


def graph_launch_ms(torch, device, fns, KL, replays=5):
    """Median and min per-launch time of a CUDA graph of KL launches cycling
    over fns, between CUDA events on the graph's stream."""
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(device)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cs):
        for i in range(KL):
            fns[i % len(fns)]()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    per = []
    for _ in range(replays):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(cs):
            e0.record(cs)
            g.replay()
            e1.record(cs)
        e1.synchronize()
        per.append(e0.elapsed_time(e1) / KL)
    del g
    return statistics.median(per), min(per)


def run_mx(args, rank, world, local_rank):
    """The decode layers with MXFP4 weights and MXFP8 activations (page 3
    section 4.3): per layer, the activation quantization and the block-scaled
    tensor-core product.  The weights are quantized and their scales laid out
    once before timing (model state); each step reads them from one of
    several copies whose reuse distance exceeds 3x L2."""
    import torch
    import bit_gemm_quant_b200 as w4

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    w4.lib()
    pk = roofline.peaks(ROOT)
    probs = synth.workload(args.workload)
    rank_seed = 1000 * rank
    host_W = [synth.weights(p.seed + rank_seed, p.N, p.K, p.w_std, *p.w_outlier) for p in probs]
    host_X = [synth.activations(p.seed + rank_seed, p.M, p.K, *p.x_outlier) for p in probs]
    dev = lambda bits: torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)

    state = []
    for p, hw in zip(probs, host_W):
        Wd = dev(hw)
        c, s_rows = w4.fp4_quant(Wd, w4.MXFP4)
        state.append((c, w4.mx_scale_layout(s_rows, p.K)))
        del Wd, s_rows
    wbytes = sum(c.numel() + s.numel() for c, s in state)
    copies = max(2, -(-3 * (126 << 20) // wbytes) + 1)
    pools = [[st] + [(st[0].clone(), st[1].clone()) for _ in range(copies - 1)] for st in state]
    X_d = [dev(hx) for hx in host_X]
    xq = [w4.mxfp8_quant(x, w4.MX_SCALES_MMA) for x in X_d]
    Y_d = [torch.empty((p.M, p.N), dtype=torch.bfloat16, device=device) for p in probs]
    torch.cuda.synchronize()

    def layer(i, copy):
        c, s = pools[i][copy % copies]
        w4.mxfp8_quant(X_d[i], w4.MX_SCALES_MMA, out=xq[i])
        w4.mx_gemm(xq[i][0], xq[i][1], c, s, out=Y_d[i], weights_static=True)

    def step(si):
        for i in range(len(probs)):
            layer(i, si)

    for si in range(max(3, args.warmup)):
        step(si)
    torch.cuda.synchronize()
    K_steps = args.steps
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(device)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cs):
        for si in range(K_steps):
            step(si)
    torch.cuda.synchronize()
    sampler = ClockSampler(smi_gpu_id(local_rank))
    sampler.start()
    sampler.mark_begin()
    t_end = time.time() + 1.5
    replays = 0
    while time.time() < t_end or replays < 2:
        graph.replay()
        replays += 1
        torch.cuda.synchronize()

    def timed():
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(cs):
            e0.record(cs)
            graph.replay()
            e1.record(cs)
        e1.synchronize()
        barrier()
        return e0.elapsed_time(e1)

    local_ms = timed()
    sampler.mark_end()
    clocks = sampler.stop()
    if any(r in clocks.get("reasons", []) for r in THROTTLE_REASONS):
        sampler = ClockSampler(sampler.gpu_id)
        sampler.start()
        sampler.mark_begin()
        local_ms = timed()
        sampler.mark_end()
        clocks = sampler.stop()
        clocks["remeasured"] = True
    del graph

    # each kernel of each layer alone (the product over the rotating weight
    # copies, with W4_WEIGHTS_STATIC as in the step and without it)
    KL = max(K_steps, 100)
    kernels = {}
    gemm_times = []
    gemm_plain = []
    for i, p in enumerate(probs):
        nb = roofline.mx_gemm_bytes(p.M, p.N, p.K)
        for static in (True, False):
            fns = [(lambda i=i, j=j, st=static: w4.mx_gemm(xq[i][0], xq[i][1], pools[i][j][0], pools[i][j][1],
                                                          out=Y_d[i], weights_static=st)) for j in range(copies)]
            avg, mn = graph_launch_ms(torch, device, fns, KL)
            (gemm_times if static else gemm_plain).append((nb, avg))
            kernels["w4_mx_gemm%s[%s]" % ("" if static else "_plain", p.name)] = {
                "launches": KL * 5, "avg_us": round(avg * 1e3, 3), "min_us": round(mn * 1e3, 3), "bytes": nb,
                "gbs": round(nb / (avg * 1e-3) / 1e9, 1), "hbm_frac": round(nb / (avg * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                "weights_static": static}
        avg, mn = graph_launch_ms(torch, device, [lambda i=i: w4.mxfp8_quant(X_d[i], w4.MX_SCALES_MMA, out=xq[i])], KL)
        nb = roofline.mxfp8_quant_bytes(p.M, p.K)
        kernels["w4_mxfp8_quant[%s]" % p.name] = {
            "launches": KL * 5, "avg_us": round(avg * 1e3, 3), "min_us": round(mn * 1e3, 3), "bytes": nb,
            "gbs": round(nb / (avg * 1e-3) / 1e9, 1)}
    torch.cuda.synchronize()

    work = K_steps * mx_step_bytes(probs)
    max_ms, total = aggregate(local_ms, work, device)
    value = total / (max_ms * 1e-3) / 1e9
    per_launch = sum(nb for nb, _ in gemm_times) / len(gemm_times)
    avg_ms = sum(t for _, t in gemm_times) / len(gemm_times)
    achieved = per_launch / (avg_ms * 1e-3) / 1e9
    traffic = traffic_table()
    tr = [traffic.get(("w4_mx_gemm", p.name)) for p in probs]
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4),
            "traffic": (sum(tr) / len(tr)) if all(t is not None for t in tr) else None,
            "kernel": "w4_mx_gemm", "algorithmic_per_launch": per_launch, "weights_static": True,
            "frac_plain": round(per_launch / (sum(t for _, t in gemm_plain) / len(gemm_plain) * 1e-3) / 1e9
                                / pk["hbm_gbs"], 4),
            "peak_source": "%s (%s)" % (pk["source"], "MEASURED_PEAKS.json" if pk["source"] == "measured"
                                        else "recipe")}

    e2e = None
    if not args.no_e2e:
        e2e = mx_e2e(w4, torch, device, probs, state, host_X, min(K_steps, 10))
        e_ms, e_work = aggregate(e2e["ms"], e2e["work"], device)
        e2e = {"value": round(e_work / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["steps"],
               "what": e2e["what"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_mx(probs, host_W, host_X, args.cpu_budget)

    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K_steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(max_ms / K_steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e2m1 x e4m3 (E8M0 scales), fp32 accumulate",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC[args.workload],
                       "l2": "every product reads its weight from one of %d copies (reuse distance > 3x L2)" % copies,
                       "timing": "K steps captured in one CUDA graph, replayed between CUDA events on the launching "
                                 "stream after %d untimed replays; max over ranks; per-kernel durations: median (and "
                                 "min) over 5 replays of a graph of max(K, 100) launches of that kernel alone" % replays,
                       "parallelism": "replicas (dp%d), no data-path collective" % world},
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": K_steps * 2 * len(probs) * world, "clocks": clocks,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def mx_e2e(w4, torch, device, probs, state, host_X, steps):
    """Through the tensor API with pinned host buffers, all timed: per layer the
    host->device copy of X, its MXFP8 quantization, the product and the
    device->host copy of Y (the quantized weights resident)."""
    hX = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in host_X]
    hY = [torch.empty((p.M, p.N), dtype=torch.bfloat16).pin_memory() for p in probs]

    def one():
        for i, p in enumerate(probs):
            Xd = hX[i].to(device, non_blocking=True).view(torch.bfloat16)
            xc, xs = w4.mxfp8_quant(Xd, w4.MX_SCALES_MMA)
            hY[i].copy_(w4.mx_gemm(xc, xs, state[i][0], state[i][1], weights_static=True), non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    e1.synchronize()
    barrier()
    return {"ms": e0.elapsed_time(e1), "work": mx_step_bytes(probs) * steps,
            "h2d": sum(x.numel() * 2 for x in hX), "d2h": sum(y.numel() * 2 for y in hY), "steps": steps,
            "what": "H2D of X, w4_mxfp8_quant, w4_mx_gemm, D2H of Y (MXFP4 weights resident)"}


def oracle_mx_prepare(oracle, probs, host_W, rows: int, offset: int = 0):
    """Rows [offset, offset + rows) of each weight quantized to MXFP4 by the
    oracle (model state, untimed)."""
    out = []
    for p, W in zip(probs, host_W):
        r0 = offset % p.N
        r1 = min(p.N, r0 + rows)
        out.append(oracle.fp4_quant(np.ascontiguousarray(W[r0:r1]), MXFP4_KIND))
    return out


def oracle_mx_sample(oracle, probs, host_X, prepared) -> int:
    """The oracle's share of one step: each layer's activations quantized to
    MXFP8 and their fp64 product with the prepared weight rows.  Returns the
    algorithmic bytes processed."""
    nb = 0
    for p, X, (wc, ws) in zip(probs, host_X, prepared):
        xc, xs = oracle.mxfp8_quant(X)
        oracle.mx_reference(xc, xs, wc, ws)
        nb += roofline.mxfp8_quant_bytes(p.M, p.K) + roofline.mx_gemm_bytes(p.M, wc.shape[0], p.K)
    return nb


def cpu_baseline_mx(probs, host_W, host_X, budget_s):
    import oracle
    oracle.build()
    rows = 16
    prep = oracle_mx_prepare(oracle, probs, host_W, rows)
    t0 = time.perf_counter()
    oracle_mx_sample(oracle, probs, host_X, prep)
    dt = time.perf_counter() - t0
    rows = min(max(p.N for p in probs), max(16, int(16 * budget_s / max(dt, 1e-3))))
    prep = oracle_mx_prepare(oracle, probs, host_W, rows)
    t0 = time.perf_counter()
    nb = oracle_mx_sample(oracle, probs, host_X, prep)
    dt = time.perf_counter() - t0
    return {"value": nb / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle", "seconds": round(dt, 2),
            "sample": "first %d rows of each decode weight: oracle MXFP8 quantization of X and the fp64 product "
                      "with those rows of the MXFP4 weight (quantized by the oracle beforehand, untimed), "
                      "single thread" % rows}


def run_reference_mx(args, world):
    """The oracle on `rows` rows of each layer's weight per step (rotating)."""
    import oracle
    probs = synth.workload(args.workload)
    host_W = [p.W() for p in probs]
    host_X = [p.X() for p in probs]
    rows = 16
    steps_total = max(3, args.warmup) + args.steps
    prep = {si: oracle_mx_prepare(oracle, probs, host_W, rows, si * rows) for si in range(steps_total)}
    for si in range(max(3, args.warmup)):
        oracle_mx_sample(oracle, probs, host_X, prep[si])
    nb = 0
    t0 = time.perf_counter()
    for j in range(args.steps):
        nb += oracle_mx_sample(oracle, probs, host_X, prep[max(3, args.warmup) + j])
    dt = time.perf_counter() - t0
    sample = ("%d rows of each weight per step (rotating): oracle MXFP8 quantization of X and the fp64 product "
              "(weights quantized by the oracle before timing), single thread" % rows)
    print_reference(args, world, nb / dt / 1e9, "GB/s", dt * 1e3 / args.steps, WORKLOAD_DESC[args.workload], sample)


# ------------------------------------------------ strong scaling (sharded) --

def run_sharded(args, rank, world, local_rank):
    """Every layer of a product workload split over the ranks: rows of W
    (column-parallel, all-gather of Y) or columns of W and X (row-parallel,
    all-reduce of the fp32 partials, then the bf16 rounding).  All ranks hold
    shares of the same layers (same seeds); value = the unsharded layers'
    algorithmic bytes (FLOPs for prefill) per step / the max-over-ranks time."""
    import torch
    import bit_gemm_quant_b200 as w4
    from bit_gemm_quant_b200 import shard

    if args.workload not in ("decode", "smallbatch", "prefill"):
        raise SystemExit("--shard applies to the product workloads (decode, smallbatch, prefill)")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    pg_ok = world > 1
    if pg_ok:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    w4.lib()
    pk = roofline.peaks(ROOT)
    split = args.shard
    plist = problems_for(args.workload)
    keys = list(dict.fromkeys(k for k, _ in plist))
    first = {k: p for k, p in reversed(plist)}
    qp = {k: first[k] for k in keys}
    dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)
    layers = {}
    for k in keys:
        p = qp[k]
        W = synth.weights(p.seed, p.N, p.K, p.w_std, *p.w_outlier)
        layers[k] = shard.ShardedW4Linear(dev(shard.local_weight(W, split, world, rank, p.group)), p.N, p.K, p.group,
                                          p.mode, split, world, rank)
    host_X = {p.name: shard.local_activations(p.X(), split, world, rank, p.group) for _, p in plist}
    X_d = {n: dev(x) for n, x in host_X.items()}
    torch.cuda.synchronize()

    def step():
        for key, p in plist:
            layers[key].forward(X_d[p.name])

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(smi_gpu_id(local_rank))
    sampler.start()
    sampler.mark_begin()
    t_end = time.time() + 1.0
    while time.time() < t_end:
        step()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    e1.synchronize()
    barrier()
    local_ms = e0.elapsed_time(e1)
    sampler.mark_end()
    clocks = sampler.stop()

    prefill = args.workload == "prefill"
    per_step = sum((roofline.gemm_flops(p.M, p.N, p.K) if prefill else roofline.gemm_bytes(p.M, p.N, p.K, p.group, p.mode))
                   for _, p in plist)
    # strong scaling: the work is the unsharded layers', counted once (not per rank)
    max_ms, _ = aggregate(local_ms, 0.0, device)
    value = args.steps * per_step / (max_ms * 1e-3) / (1e12 if prefill else 1e9)

    # the local product alone (no collective): its algorithmic bytes over its time
    KL = max(args.steps, 50)
    loc = []
    for key, p in plist:
        lay = layers[key]
        n_loc, k_loc = lay.n1 - lay.n0, lay.k1 - lay.k0
        f = (lambda lay=lay, x=X_d[p.name], n=n_loc: lay.ops.gemm(x, lay.packed, lay.group, lay.mode,
                                                                   n, out_f32=lay.split == "k"))
        avg, _ = graph_launch_ms(torch, device, [f], KL)
        loc.append((roofline.gemm_bytes(p.M, n_loc, k_loc, p.group, p.mode), roofline.gemm_flops(p.M, n_loc, k_loc),
                    avg))
    nb = sum(b for b, _, _ in loc) / len(loc)
    nf = sum(f for _, f, _ in loc) / len(loc)
    avg_ms = sum(t for _, _, t in loc) / len(loc)
    if prefill:
        ach = nf / (avg_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(ach / pk["bf16_tflops"], 4)}
    else:
        ach = nb / (avg_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4)}
    roof.update({"traffic": None, "kernel": "w4a16_gemm on this rank's shard (collective excluded)",
                 "algorithmic_per_launch": nf if prefill else nb,
                 "peak_source": "%s (%s)" % (pk["source"], "MEASURED_PEAKS.json" if pk["source"] == "measured"
                                             else "recipe")})

    e2e = None
    if not args.no_e2e:
        hX = {n: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).pin_memory() for n, x in host_X.items()}
        hY = {p.name: torch.empty((p.M, p.N), dtype=torch.bfloat16).pin_memory() for _, p in plist}

        def one():
            for key, p in plist:
                Y = layers[key].forward(hX[p.name].to(device, non_blocking=True).view(torch.bfloat16))
                hY[p.name].copy_(Y, non_blocking=True)

        one()
        torch.cuda.synchronize()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps_e = min(args.steps, 10)
        a0.record()
        for _ in range(steps_e):
            one()
        a1.record()
        a1.synchronize()
        barrier()
        e_ms, _ = aggregate(a0.elapsed_time(a1), 0.0, device)
        e2e = {"value": round(steps_e * per_step / (e_ms * 1e-3) / (1e12 if prefill else 1e9), 2),
               "unit": "TFLOP/s" if prefill else "GB/s",
               "h2d_bytes_per_step": sum(x.numel() * 2 for x in hX.values()),
               "d2h_bytes_per_step": sum(y.numel() * 2 for y in hY.values()), "steps": steps_e,
               "what": "per rank: H2D of its activations, the sharded layer (product + collective), D2H of Y"}

    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s" if prefill else "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(max_ms / args.steps, 5),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC[args.workload],
                       "shard": "%s-split over %d ranks: %s" % (split, world, "rows of W, all-gather of Y" if split == "n"
                                                                else "columns of W and X, all-reduce of fp32 partials, "
                                                                     "then w4_f32_to_bf16"),
                       "timing": "K eager steps between CUDA events on the current stream, barrier and synchronize "
                                 "on both sides, max over ranks",
                       "parallelism": "tp%d (%s-split)" % (world, split)},
            "roofline": roof, "cpu_baseline": None, "e2e": e2e,
            "gpu_launches": args.steps * len(plist) * (2 if split == "k" else 1) * world, "clocks": clocks,
        }
        print(json.dumps(out), flush=True)
    if pg_ok:
        import torch.distributed as dist
        dist.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    if args.workload == "awq":
        run_awq(args, rank, world, local_rank)
        return 0
    if args.workload == "fp4quant":
        run_fp4(args, rank, world, local_rank)
        return 0
    if args.workload in MX_WORKLOADS:
        run_mx(args, rank, world, local_rank)
        return 0
    if args.shard != "none":
        run_sharded(args, rank, world, local_rank)
        return 0
    run_w4(args, rank, world, local_rank)
    return 0


if __name__ == "__main__":
    sys.exit(main())
