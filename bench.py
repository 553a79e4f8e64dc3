"""Benchmark of the binary-weight decode GEMV (one JSON line on rank 0).

Default workload: the Llama-7B attention projection, 4096x4096 with two binary
bases and bf16 row/column scales, batch M=1. One step = one replay of a CUDA
graph holding S back-to-back GEMVs over S distinct weight copies whose total
size exceeds 3x the L2 cache, so every GEMV streams its weights from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bisco|reference]
                    [--workload attn4096|mlp_gate_up|mlp_down|lowrank5120|cfg1|decoder7b|
                                fluxbin4096_g128|fluxbin4096_s16] [--M m]

Workload decoder7b is the 32-layer Llama-7B-shaped decoder weight stream (per layer
q, k, v, o 4096x4096, gate and up 4096->11008, down 11008->4096; 2 bases and a
rank-256 binary correction each): one step replays a graph of all 224 GEMVs, in
layer order, over 1.71 GB of distinct weights. Workloads fluxbin4096_* are the same
4096x4096 projection in FluxBin's own configurations (2b-g128: grouped row scales; 2b-s16-g128:
plus two binary refinement bases over 16 salient columns of every group).

Metric: effective HBM GB/s of the M=1 binary GEMV (algorithmic bytes: packed
sign bits, scales, correction signs and coefficients, salient payload, X read
and Y written, over device time); the microseconds per GEMV are reported too.
Multi-GPU runs are weak-scaling replicas: every rank streams its own layers,
there is no data-path collective, and the time is the max over ranks.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import make_activations, make_layer  # noqa: E402
from synth.configs import SEED, build  # noqa: E402

WORKLOADS = {
    # name: (config, spec index, default M, description)
    "attn4096": (2, 0, 1, "Llama-7B attention projection 4096x4096, 2 binary bases, bf16 scales"),
    "mlp_gate_up": (3, 0, 1, "Llama-7B MLP gate/up 4096->11008, 2 bases, 1% salient int8 columns"),
    "mlp_down": (3, 1, 1, "Llama-7B MLP down 11008->4096, 2 bases, 1% salient int8 columns"),
    "lowrank5120": (4, 0, 1, "5120x5120, 2 bases + rank-512 binary correction, 0.1% outliers x20"),
    "cfg1": (1, 0, 1, "256x512, 1 base, fp32 scales, rank-8 correction"),
    "decoder7b": (5, None, 1, "32-layer Llama-7B decoder weight stream: q/k/v/o 4096^2, gate/up 4096->11008, "
                              "down 11008->4096, 2 bases + rank-256 binary correction each (224 GEMVs)"),
    "fluxbin4096_g128": (2, 0, 1, "4096x4096 FluxBin 2b-g128: 2 bases, bf16 row scales per 128-column group"),
    "fluxbin4096_s16": (2, 0, 1, "4096x4096 FluxBin 2b-s16-g128: 2 bases, bf16 row scales per 128-column group, "
                                 "2 binary refinement bases over 16 salient columns per group"),
}
# FluxBin layers ("FluxBin", Sec. 4, Kb-sS-gG): workload -> (group size, (Ks, s) or None)
FLUXBIN = {"fluxbin4096_g128": (128, None), "fluxbin4096_s16": (128, (2, 16))}
DECODER_LAYERS = 32
DECODER_MATRICES = 7  # q, k, v, o, gate, up, down


def base_matrices(workload, M):
    """(layer, X) pairs of the distinct matrices of a workload: one for the single-layer
    workloads, the seven matrix shapes of a decoder layer for decoder7b (every decoder
    layer streams its own device copy of them)."""
    cfg, spec, _, _ = WORKLOADS[workload]
    if spec is None:
        return [build(cfg, i, M) for i in range(DECODER_MATRICES)]
    if workload in FLUXBIN:
        g, ref = FLUXBIN[workload]
        L = make_layer(SEED, (870, 4096, 4096), 4096, 4096, 2, "bf16", group=g, refine=ref, name=workload)
        return [(L, make_activations(SEED, (870, 4096, 1000 + M), M, 4096, "bf16"))]
    return [build(cfg, spec, M)]

MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_per_launch.json")
FALLBACK_HBM_GBS = 6650.0


def sources_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "binary_weight_decode_b200", "csrc")
    for n in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        with open(MEASURED_PEAKS) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0


def tensor_peak():
    """Measured dense bf16 tensor throughput (burst: a kernel timed alone), TFLOP/s."""
    try:
        with open(MEASURED_PEAKS) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def algorithmic_flops(L, M):
    """Multiply-adds of one GEMV x 2: the K binary bases, both correction factors and
    the salient columns, for M batch rows."""
    return 2.0 * M * (L.K * L.out * L.in_ + L.rank * (L.in_ + L.out) + L.out * L.n_sal)


def traffic_for(workload, M):
    """dram bytes per launch of the dominant kernel from a committed ncu capture (plus the
    refinement launch of the same GEMV where the workload has one), or None if there is
    none for this workload or the kernel sources changed."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        e, r = t.get(f"{workload}_M{M}"), t.get(f"{workload}_M{M}_refine")
        if e and e.get("sources") == sources_digest():
            if r is None:
                return e["dram_bytes_per_launch"]
            if r.get("sources") == e["sources"]:
                return e["dram_bytes_per_launch"] + r["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def max_over_ranks(value, dist, device):
    """The largest of `value` over all ranks (the job is as slow as its slowest rank);
    `value` itself when there is no process group."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_baseline(workload, M, budget_s=12.0):
    """The fp64 oracle, as it stands, on this host's cores over a bounded sample."""
    import oracle
    from threadpoolctl import threadpool_info
    cfg, spec, _, _ = WORKLOADS[workload]
    L, X = base_matrices(workload, M)[0] if spec is not None else build(cfg, 0, M)  # decoder7b: its q projection
    xdt = "f32" if cfg == 1 else "bf16"
    nbytes = oracle.algorithmic_bytes(L, M, xdt, "bf16")
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.gemv(L, X, xdt)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 200:
            break
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    # the same oracle on one thread, over a shorter sample
    from threadpoolctl import threadpool_limits
    n1, t1 = 0, time.perf_counter()
    with threadpool_limits(limits=1):
        while True:
            oracle.gemv(L, X, xdt)
            n1 += 1
            el1 = time.perf_counter() - t1
            if el1 >= budget_s / 4 or n1 >= 50:
                break
    return {"value": round(n * nbytes / el / 1e9, 4), "unit": "GB/s", "cores": int(threads),
            "value_1thread": round(n1 * nbytes / el1 / 1e9, 4),
            "kind": "oracle", "us_per_gemv": el / n * 1e6,
            "sample": f"{n} full fp64 oracle GEMVs of the {workload} layer{' q projection' if spec is None else ''} "
                      f"(M={M}) in {el:.1f} s on {os.cpu_count()} host cores"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cb = cpu_baseline(args.workload, args.M, budget_s=max(5.0, 3.0 * args.steps))
    cfg, spec, _, desc = WORKLOADS[args.workload]
    line = {"metric": "M=1 binary-GEMV effective HBM GB/s", "value": cb["value"], "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": cb["us_per_gemv"] / 1000.0, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"{args.workload}: {desc}", "M": args.M},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def algorithmic_bytes(L, M, x_bytes, y_bytes):
    """Bytes one GEMV must move (same accounting as the oracle's, restated for the
    product path so that the bench does not depend on the oracle)."""
    sb = 2 if L.scale_dtype == "bf16" else 4
    g = getattr(L, "group", 0) or 0
    ng = -(-L.in_ // g) if g else 1  # row scales per row
    n = L.K * L.out * L.in_ / 8.0 + L.K * (L.out * ng + L.in_) * sb
    if L.rank:
        n += L.rank * (L.out + L.in_) / 8.0 + 4 * L.rank
    if L.n_sal:
        n += L.out * L.n_sal + 8 * L.n_sal
    ks = getattr(L, "ref_K", 0) or 0
    if ks:  # refinement signs, row scales per group, column scales, int32 indices
        nr = len(L.ref_idx)
        n += ks * L.out * nr / 8.0 + ks * (L.out * ng + nr) * sb + 4 * nr
    n += M * L.in_ * x_bytes + M * L.out * y_bytes
    return int(round(n))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="bisco", choices=["bisco", "reference"])
    ap.add_argument("--workload", default="attn4096", choices=sorted(WORKLOADS))
    ap.add_argument("--M", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-group", action="store_true",
                    help="decoder7b: one bisco_gemv per matrix instead of one bisco_gemv_group for q/k/v and gate/up")
    ap.add_argument("--calls", type=int, default=0,
                    help="profiling case: run this many plain bisco_gemv calls on one weight copy and exit")
    args = ap.parse_args()
    cfg, spec, m_default, desc = WORKLOADS[args.workload]
    args.M = args.M or m_default
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import binary_weight_decode_b200 as bw

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    M = args.M
    mats = base_matrices(args.workload, M)
    xdt = "f32" if cfg == 1 else "bf16"

    def dev_x(X):
        Xh = torch.from_numpy(X.view(np.int16) if xdt == "bf16" else X)
        return Xh, (Xh.to("cuda").view(torch.bfloat16) if xdt == "bf16" else Xh.to("cuda"))

    if args.calls:  # small case for ncu captures: no graph, no timing
        L, X = mats[0]
        dl = bw.DeviceLayer(L)
        Xd = dev_x(X)[1]
        Yd = torch.empty((M, L.out), dtype=torch.bfloat16, device="cuda")
        ws = bw.alloc_workspace([dl], M)
        for _ in range(args.calls):
            bw.bisco_gemv(dl, Xd, Yd, ws)
            torch.cuda.synchronize()
        st = bw.bisco_sync_status(ws)
        if st != bw.BISCO_OK:
            raise SystemExit(f"device status {bw.bisco_status_string(st)}")
        return
    x_bytes = 4 if xdt == "f32" else 2
    y_dtype = torch.bfloat16
    nbytes_b = [algorithmic_bytes(L, M, x_bytes, 2) for (L, _) in mats]
    props = torch.cuda.get_device_properties(local)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    if WORKLOADS[args.workload][1] is None:
        S = DECODER_LAYERS  # the decoder stream: one copy per layer (1.7 GB, far above L2)
    else:
        S = max(4, math.ceil(3 * l2 / nbytes_b[0]))
    nbytes = sum(nbytes_b)  # one pass over the distinct matrices

    # S distinct device copies of every base matrix: same values, separate HBM buffers
    first = [bw.DeviceLayer(L) for (L, _) in mats]
    dls = [[d] + [d.clone() for _ in range(S - 1)] for d in first]
    grouped = WORKLOADS[args.workload][1] is None and not args.no_group
    if grouped:  # q/k/v read one x, gate/up another (as in a decoder layer)
        mats = [(L, mats[0][1]) if b in (1, 2) else (L, mats[4][1]) if b == 5 else (L, X)
                for b, (L, X) in enumerate(mats)]
    xs = [dev_x(X) for (_, X) in mats]
    Yd = [torch.empty((S, M, L.out), dtype=y_dtype, device="cuda") for (L, _) in mats]
    groups = [[0, 1, 2], [3], [4, 5], [6]] if grouped else [[b] for b in range(len(mats))]
    need = [bw.bisco_workspace_size(d, M) for d in first]
    need += [bw.bisco_group_workspace_size([first[b] for b in g], M) for g in groups if len(g) > 1]
    ws = torch.empty(max(need), dtype=torch.uint8, device="cuda")
    bw.bisco_workspace_init(ws)
    ws_bytes = ws.numel() * ws.element_size()
    xcode = bw.BISCO_BF16 if xdt == "bf16" else bw.BISCO_F32
    kinds = [bw.bisco_plan_group_kernels([first[b] for b in g], M, xcode, ws_bytes) if len(g) > 1
             else bw.bisco_plan_kernels(first[g[0]], M, xcode, ws_bytes) for g in groups]

    def stream_once(stream):
        for i in range(S):
            for g in groups:
                if len(g) == 1:
                    bw.bisco_gemv(dls[g[0]][i], xs[g[0]][1], Yd[g[0]][i], ws, stream=stream)
                else:
                    bw.bisco_gemv_group([dls[b][i] for b in g], xs[g[0]][1], [Yd[b][i] for b in g], ws, stream=stream)

    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        stream_once(stream)  # eager warm-up run (also sets kernel attributes before capture)
    stream.synchronize()
    st = bw.bisco_sync_status(ws)
    if st != bw.BISCO_OK:
        raise SystemExit(f"device status {bw.bisco_status_string(st)}")
    with torch.cuda.graph(graph, stream=stream):
        stream_once(stream)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # graph replays and events all go to `stream` (CUDAGraph.replay uses the current stream)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    barrier()
    ms = e0.elapsed_time(e1)
    clocks = sampler.stop()
    ms = max_over_ranks(ms, dist, "cuda")
    gemvs = args.steps * S * len(mats)
    us_per_gemv = ms * 1000.0 / gemvs
    value = world * args.steps * S * nbytes / (ms / 1000.0) / 1e9

    # end to end through the public API: pinned host X in, host Y out, every step
    Xpins = [xh.pin_memory() for (xh, _) in xs]
    Xraws = [xd.view(torch.int16) if xdt == "bf16" else xd for (_, xd) in xs]
    Ypins = [torch.empty(y.shape, dtype=torch.int16).pin_memory() for y in Yd]
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, args.steps // 2)
    barrier()
    e2.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(e2e_steps):
            for xr, xp in zip(Xraws, Xpins):
                xr.copy_(xp, non_blocking=True)
            graph.replay()
            for yp, y in zip(Ypins, Yd):
                yp.copy_(y.view(torch.int16), non_blocking=True)
    e3.record(stream)
    barrier()
    ms_e2e = e2.elapsed_time(e3)
    ms_e2e = max_over_ranks(ms_e2e, dist, "cuda")
    e2e_value = world * e2e_steps * S * nbytes / (ms_e2e / 1000.0) / 1e9
    L = mats[0][0]
    peak, peak_kind = hbm_peak()
    us_per_pass = ms * 1000.0 / (args.steps * S)  # one GEMV of every distinct matrix
    achieved = nbytes / (us_per_pass * 1e-6) / 1e9
    # batch chunks of 32+ rows run on the tensor cores (bf16 scales): a dense contraction
    on_tensor = M >= 32 and (L.K == 0 or L.scale_dtype == "bf16")
    if on_tensor:
        tpeak, tpeak_kind = tensor_peak()
        flops = sum(algorithmic_flops(Lb, M) for (Lb, _) in mats)
        tflops = flops / (us_per_pass * 1e-6) / 1e12
        roofline = {"bound": "tensor", "achieved": round(tflops, 2), "peak": tpeak, "unit": "TFLOP/s",
                    "frac": round(tflops / tpeak, 4), "peak_kind": f"{tpeak_kind} dense bf16 (burst)",
                    "flops_per_gemv": flops / len(mats), "traffic": traffic_for(args.workload, M)}
    else:
        roofline = {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                    "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
                    "frac_of_8000": round(achieved / 8000.0, 4), "traffic": traffic_for(args.workload, M)}
    line = {
        "metric": "M=1 binary-GEMV effective HBM GB/s", "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if on_tensor else "f32",
        "data": "synthetic",
        "impl": "bisco",
        "config": {"workload": f"{args.workload}: {desc}", "M": M, "gemvs_per_step": S * len(mats),
                   "algorithmic_bytes_per_gemv": nbytes if len(mats) == 1 else round(nbytes / len(mats)),
                   "algorithmic_bytes_per_step": S * nbytes, "y_dtype": "bf16",
                   "l2": f"inputs larger than L2: each step streams {S * len(mats)} distinct weight copies "
                         f"({S * nbytes / 2 ** 20:.0f} MiB > 3x L2)",
                   "kernels_per_gemv": kinds if len(mats) > 1 else kinds[0],
                   "grouped_calls": [[["q", "k", "v", "o", "gate", "up", "down"][b] for b in g] for g in groups]
                   if len(mats) > 1 else None,
                   "parallelism": f"replicas x{world} (no collective)"},
        "us_per_gemv": round(us_per_gemv, 4),
        "us_per_step": round(ms * 1000.0 / args.steps, 2),
        "roofline": roofline,
        "clocks": clocks,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in Xpins)),
                "d2h_bytes_per_step": int(sum(y.numel() * 2 for y in Ypins))},
        "gpu_launches": int(args.steps * S * sum(len(k) for k in kinds)),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, M)
    del graph
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
