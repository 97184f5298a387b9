"""Throughput of the SVDQuant W4A4 (NVFP4) linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload flux_qkv] [--sets 4] [--no-e2e] [--no-cpu-baseline]

One step = one pass of the whole hot path over one batch: the activation
kernel (smoothing, NVFP4 quantization, fused low-rank down-projection) and
the 4-bit GEMM kernel (fused up-projection, bias, bf16 store) of one
Flux-shaped linear.  Default workload: the fused QKV projection, M = 4608
tokens, K = 3072, N = 9216, rank 32, synthetic seeded data.

With N > 1 (launched by torchrun) every rank runs its own batch of tokens
through a replica of the layer (weak scaling, no data-path collective); the
time is the max over ranks.  Rank 0 prints one JSON line.

--impl reference runs the CPU oracle (the test reference implementation)
on the host cores instead, on a bounded sample of rows per step.
"""
from __future__ import annotations

import argparse
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

import svdq_inputs as SI  # noqa: E402

METRIC = "svdq W4A4 linear effective TFLOPS & % of dense NVFP4 peak; µs/layer @M=4608"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0            # nominal dense ratio 9 / 2.25 PFLOP/s
CSRC = "w4a4_rank_corrected_b200/csrc/"
# the sources each kernel is compiled from (its header, the headers it
# includes, the PTX wrappers): a committed ncu figure counts only while these
# are unchanged
KERNEL_SOURCES = {
    "w4a4_gemm": ["w4a4_gemm.cuh", "gelu.cuh", "row_scales.cuh", "ptx.cuh"],
    "quantize_act": ["quantize_act.cuh", "row_scales.cuh", "ptx.cuh"],
    "quantize_act64": ["quantize_act64.cuh", "row_scales.cuh", "ptx.cuh"],
    "awq_gemv": ["awq_gemv.cuh", "ptx.cuh"],
}


def act_kernel_for(M: int) -> str:
    """The activation kernel the library runs for M rows (the same rule as
    launch_quantize on a 148-SM B200)."""
    return "quantize_act" if (M + 127) // 128 >= 120 else "quantize_act64"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="flux_qkv")
    ap.add_argument("--layer", type=int, default=0, help="which layer of the workload to time")
    ap.add_argument("--sets", type=int, default=4, help="rotating input/weight/output sets")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step from a CUDA graph (small layers are launch-bound)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--awq", type=int, default=0, metavar="M",
                    help="time the AWQ W4A16 modulation linear (3072 -> 18432) at batch M instead")
    ap.add_argument("--pair", action="store_true",
                    help="time the MLP pair of the workload (fc1 -> GELU -> fc2) as one step")
    ap.add_argument("--kernel-seconds", type=float, default=1.0,
                    help="device time of the per-kernel timing batches (each kernel alone)")
    ap.add_argument("--kernel-launches", type=int, default=1000,
                    help="minimum launches of the per-kernel timing batches; 0 with "
                         "--kernel-seconds 0 leaves them out (profiler runs)")
    return ap.parse_args()


# ----------------------------------------------------------- helpers ----

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_activations(spec, rank: int, M: int, K: int) -> np.ndarray:
    """Rank 0 uses the workload's own draw; rank r > 0 its own batch of
    tokens with the same value model (independent seed)."""
    if rank == 0:
        return SI.make_workload(spec.name, M=M).X_bf16
    rng = np.random.default_rng(spec.seed * 1000003 + rank)
    return SI.draw_activations(rng, M, K, spec.x_dist, spec.x_outliers, spec.x_scale)


def layer_setup(spec, layer: int, rank: int = 0):
    """(layer spec, W, bias, X) of layer `layer` of a workload.  Layer 0 takes
    the workload's own input draw; a later layer (whose real input is the
    previous layer's output) takes a seeded draw of its own shape with the
    same value model, which is what its timing needs."""
    wl = SI.make_workload(spec.name)
    lt = wl.layers[layer]
    ls = lt.spec
    if layer == 0:
        X0 = wl.X_bf16 if rank == 0 else rank_activations(spec, rank, ls.M, ls.K)
    else:
        rng = np.random.default_rng(spec.seed * 7919 + 100 * layer + rank)
        X0 = SI.draw_activations(rng, ls.M, ls.K, spec.x_dist, min(spec.x_outliers, ls.K),
                                 spec.x_scale)
    return ls, lt.W, lt.bias_bf16, X0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, CSRC + rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of `kernel`,
    or None when there is none or the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha") != kernel_source_hash(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons in the
    background while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"svdq_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "10", "-i", str(self.gpu)], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi needs a moment to start: wait (bounded) for its first line
        t0 = time.time()
        while time.time() - t0 < 5.0:
            try:
                if os.path.getsize(self.path) > 0:
                    break
            except OSError:
                pass
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "util": float(parts[4]),
                             "hw": parts[6], "hwt": parts[7], "swt": parts[8], "pc": parts[9]})
            except ValueError:
                continue
        os.unlink(self.path)
        load = [r for r in rows if r["util"] > 0] or rows
        if not load:
            return {"samples": 0}
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pc", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in load), "reasons": sorted(reasons),
                "samples": len(load)}


# --------------------------------------------------------------- ours ----

def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    import w4a4_rank_corrected_b200 as S

    spec = SI.workload_specs()[args.workload]
    ls, W, bias, X0 = layer_setup(spec, args.layer, rank)
    M, K, N, r = ls.M, ls.K, ls.N, ls.r
    cx = SI.channel_absmax(X0)
    packed = S.svdq_pack_weight(W, cx, r)

    nsets = max(1, args.sets)
    weights = [packed.to_device(dev, bias) for _ in range(nsets)]
    Xs = [torch.from_numpy(X0.view(np.int16)).to(dev).view(torch.bfloat16) for _ in range(nsets)]
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(nsets)]
    klr = ((2 * r + 63) // 64) * 64
    sf_bytes = ((M + 127) // 128) * 128 * (K // 16)
    codes = [torch.empty((M, K // 2), dtype=torch.uint8, device=dev) for _ in range(nsets)]
    sfs = [torch.empty(sf_bytes, dtype=torch.uint8, device=dev) for _ in range(nsets)]
    xl1s = [torch.empty((M, klr), dtype=torch.bfloat16, device=dev) if r else None
            for _ in range(nsets)]
    stream = torch.cuda.current_stream(dev)
    # few output tiles (small M): the GEMM splits K across CTA pairs, with
    # its partial sums in a workspace of its own per buffer set
    split_need = S.svdq_gemm_workspace_bytes(M, N, K)
    split_ws = [torch.empty(split_need, dtype=torch.uint8, device=dev) for _ in range(nsets)] \
        if split_need else None

    def gemm(j, stream=None):
        if split_ws:
            S.svdq_gemm_splitk(weights[j], codes[j], sfs[j], xl1s[j], M, Ys[j], split_ws[j],
                               stream)
        else:
            S.svdq_gemm(weights[j], codes[j], sfs[j], xl1s[j], M, Ys[j], stream)

    def step(i):
        j = i % nsets
        S.svdq_quantize_act(weights[j], Xs[j], codes[j], sfs[j], xl1s[j], stream)
        gemm(j, stream)

    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
    sampler.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)

    # With --graph each step (activation kernel + GEMM, the two launches of
    # svdq_linear_forward) is captured once per buffer set into a CUDA graph
    # and replayed, so the timed loop measures the GPU rather than per-call
    # host work (TMA descriptor encoding, Python marshalling), which
    # dominates at small M.  By default the launches are issued one by one
    # (at large M they overlap through programmatic dependent launch).
    graphs = None
    if args.graph:
        try:
            graphs = []
            for j in range(nsets):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    S.svdq_quantize_act(weights[j], Xs[j], codes[j], sfs[j], xl1s[j])
                    gemm(j)
                graphs.append(g)
            for j in range(nsets):
                graphs[j].replay()
            torch.cuda.synchronize(dev)
        except Exception as ex:  # capture not available: time the launches directly
            print(f"graph capture failed ({type(ex).__name__}: {ex}); timing direct launches",
                  file=sys.stderr)
            graphs = None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)

    K_steps = args.steps
    ev_start = torch.cuda.Event(enable_timing=True)
    ev_end = torch.cuda.Event(enable_timing=True)
    ev_start.record(stream)
    if graphs is not None:
        for i in range(K_steps):
            graphs[i % nsets].replay()
    else:
        for i in range(K_steps):
            step(i)
    ev_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    elapsed_ms = max_over_ranks(ev_start.elapsed_time(ev_end), world, dev)

    # Per-kernel times, right after the timed region and under the same clock
    # sampling: each kernel alone, launched back to back from a CUDA graph of
    # `per_graph` launches over the rotating buffer sets (so host launch cost
    # does not hide the kernel), replayed until at least `min_launches`
    # launches and `min_seconds` of device time; CUDA events on the
    # launching stream around all replays.
    def kernel_time_ms(launch, min_launches=1000, min_seconds=1.0, per_graph=200):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(per_graph):
                launch(i)
        g.replay()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        est = a.elapsed_time(b) / per_graph
        reps = max(-(-min_launches // per_graph), int(min_seconds * 1e3 / (est * per_graph)) + 1)
        cur = torch.cuda.current_stream(dev)
        a.record(cur)
        for _ in range(reps):
            g.replay()
        b.record(cur)
        torch.cuda.synchronize(dev)
        del g
        return a.elapsed_time(b) / (reps * per_graph), reps * per_graph

    if args.kernel_seconds > 0 or args.kernel_launches > 0:
        kt = dict(min_launches=max(1, args.kernel_launches), min_seconds=args.kernel_seconds)
        q_ms, q_n = kernel_time_ms(lambda i: S.svdq_quantize_act(
            weights[i % nsets], Xs[i % nsets], codes[i % nsets], sfs[i % nsets], xl1s[i % nsets]),
            **kt)
        g_ms, g_n = kernel_time_ms(lambda i: gemm(i % nsets), **kt)
    else:                      # profiler runs: per-kernel times come from the profiler
        q_ms = g_ms = float("nan")
        q_n = g_n = 0
    clocks = sampler.stop()
    err = S.svdq_device_error(stream)
    if err:
        raise SystemExit(f"device error code {err:#x}")
    ms_per_step = elapsed_ms / K_steps
    flops = 2.0 * M * N * K
    value = world * flops * K_steps / (elapsed_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    fp4_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * FP4_OVER_BF16
    fp4_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP4_OVER_BF16
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gemm_tflops = flops / (g_ms * 1e-3) / 1e12
    q_bytes = M * K * 2 + M * K // 2 + M * K // 16 + (M * klr * 2 + 2 * r * K * 2 if r else 0) + K * 4
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9
    traffic = profiled_traffic("w4a4_gemm", args.workload)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world,
        "steps": K_steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
        "data": "synthetic",
        "config": {
            "workload": f"{spec.name}: {spec.description}", "layer": ls.name, "M": M, "K": K, "N": N, "r": r,
            "global_batch": M * world, "parallelism": f"dp{world} (independent replicas, no collective)",
            "launch": "CUDA graph replay per step" if graphs is not None else "direct launches",
            "gemm": (f"split-K over CTA pairs ({split_need / 1e6:.1f} MB partials workspace)"
                     if split_ws else "whole-K tiles"),
            "l2": f"{nsets} rotating input/weight/output sets (~{nsets * (M * K * 2 + M * N * 2 + N * K // 2) / 1e6:.0f} MB > 126 MB L2)",
            "us_per_layer": round(ms_per_step * 1e3, 2),
            "us_quantize_act": round(q_ms * 1e3, 2), "us_gemm": round(g_ms * 1e3, 2),
            "gemm_tflops": round(gemm_tflops, 1),
            "pct_fp4_peak_sustained": round(100 * gemm_tflops / fp4_sust, 1),
            "pct_fp4_peak_burst": round(100 * gemm_tflops / fp4_burst, 1),
            "pct_fp4_datasheet_9pf": round(100 * gemm_tflops / 9000.0, 1),
            "quantize_act_gbs": round(q_gbs, 1), "quantize_act_pct_hbm": round(100 * q_gbs / hbm, 1),
            "per_kernel_timing": "each kernel alone after the timed region, >= 1000 launches and >= 1 s from CUDA graphs",
            "layer_roofline_frac": round(max(flops / (fp4_sust * 1e12), (q_bytes + M * N * 2) / (hbm * 1e9)) / (ms_per_step * 1e-3), 3),
        },
        "roofline": {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(fp4_burst, 1),
                     "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_burst, 4), "traffic": traffic,
                     "kernel": "w4a4_gemm_kernel",
                     "peak_source": f"{peak_src} bf16_tflops (burst) x {FP4_OVER_BF16:g} (nominal FP4/BF16 dense ratio); the kernel is timed alone",
                     "frac_sustained": round(gemm_tflops / fp4_sust, 4),
                     "peak_sustained": round(fp4_sust, 1),
                     "timing": f"{g_n} back-to-back launches from a CUDA graph, CUDA events on the launching stream"},
        "roofline_quantize_act": {"bound": "hbm", "achieved": round(q_gbs, 1), "peak": round(hbm, 1),
                                  "unit": "GB/s", "frac": round(q_gbs / hbm, 4),
                                  "traffic": profiled_traffic(act_kernel_for(M), args.workload),
                                  "kernel": act_kernel_for(M) + "_kernel",
                                  "algorithmic_bytes": int(q_bytes),
                                  "timing": f"{q_n} back-to-back launches from a CUDA graph"},
        "gpu_launches": 2 * K_steps,
        "clocks": clocks,
    }

    if not args.no_e2e:
        out["e2e"] = e2e_leg(S, weights[0], X0, M, K, N, r, dev, stream, args.e2e_steps, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(spec, W, bias, X0, packed, r, budget_s=15.0)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def e2e_leg(S, w, X0, M, K, N, r, dev, stream, steps, world):
    """The same metric through the public host-buffer call
    (svdq_linear_forward_host, via HostStreamer): every step uploads X from
    pinned host memory, runs the layer and downloads Y into pinned host
    memory, one C call on one stream; consecutive steps alternate between
    two streams, so one step's download overlaps the next step's upload."""
    import torch
    Xh = torch.from_numpy(X0.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hs = S.HostStreamer(w, M, dev)
    for i in range(3):
        hs.submit(Xh, Yh[i & 1])
    hs.synchronize()
    torch.cuda.synchronize(dev)
    cur = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(cur)
    for st in hs.streams:
        st.wait_stream(cur)
    for i in range(steps):
        hs.submit(Xh, Yh[i & 1])
    for st in hs.streams:
        cur.wait_stream(st)
    b.record(cur)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(a.elapsed_time(b), world, dev) / steps
    return {"value": round(world * 2.0 * M * N * K / (ms * 1e-3) / 1e12, 3), "unit": "TFLOPS",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": M * K * 2,
            "d2h_bytes_per_step": M * N * 2,
            "path": "svdq_linear_forward_host (C ABI): H2D copy, both kernels, D2H copy per step; "
                    "steps alternate between two streams"}


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def _oracle_setup(W, X0, packed, r):
    """The oracle's pack of this layer (taking the library's stored low-rank
    factors, which the SVD leaves non-unique) and its dequantized weight.
    Setup, not timed: the timed work per row is the activation NVFP4, the
    float64 dequantized GEMM, the low-rank branch and the bias."""
    from oracle import svdq as O
    cx = SI.channel_absmax(X0)
    op = O.pack(W, cx, r, L1=packed.l1, L2=packed.l2) if r else O.pack(W, cx, 0)
    return op, O.nvfp4_dequantize(op.codes_w, op.sf_w)


def _rows_for_budget(run, budget_s, M):
    """Rows per call so that one call takes about budget_s (fitted from
    two timed calls: fixed cost plus cost per row)."""
    t0 = time.perf_counter()
    run(np.arange(4))
    t4 = time.perf_counter() - t0
    t0 = time.perf_counter()
    run(np.arange(32))
    t32 = time.perf_counter() - t0
    per_row = max((t32 - t4) / 28, 1e-7)
    fixed = max(t4 - 4 * per_row, 0.0)
    return int(max(1, min(M, (budget_s - fixed) / per_row)))


def cpu_baseline(spec, W, bias, X0, packed, r, budget_s=15.0):
    """The oracle as it stands, on a bounded sample of rows of the same
    workload, timed on the host cores; scaled to effective TFLOPS."""
    from oracle import svdq as O
    op, deq_w = _oracle_setup(W, X0, packed, r)
    M, K = X0.shape
    N = W.shape[0]

    def run(idx):
        O.linear_reference(X0, op, bias, rows=idx, deq_w=deq_w)

    rows = _rows_for_budget(run, budget_s, M)
    idx = np.arange(rows)
    t0 = time.perf_counter()
    run(idx)
    dt = time.perf_counter() - t0
    return {"value": round(2.0 * rows * N * K / dt / 1e12, 6), "unit": "TFLOPS",
            "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"first {rows} of {M} rows of {spec.name} (activation NVFP4 + float64 dequantized GEMM + low-rank branch + bias; weight dequantized once, untimed), {dt:.2f} s"}


# ---------------------------------------------------------- reference ----

def run_reference(args):
    """The oracle alone, on the host cores (the reference implementation of
    this path): its own pack (LAPACK SVD, untimed setup), then per step the
    activation NVFP4, the float64 dequantized GEMM, the low-rank branch and
    the bias on a bounded sample of rows.  Nothing of the CUDA library is
    loaded."""
    rank, world, local = dist_env()
    if rank != 0:
        return
    from oracle import svdq as O
    spec = SI.workload_specs()[args.workload]
    ls, W, bias, X0 = layer_setup(spec, args.layer)
    M, K, N, r = ls.M, ls.K, ls.N, ls.r
    op = O.pack(W, SI.channel_absmax(X0), r)
    deq_w = O.nvfp4_dequantize(op.codes_w, op.sf_w)

    def run(idx):
        O.linear_reference(X0, op, bias, rows=idx, deq_w=deq_w)

    total_budget = 120.0
    rows = _rows_for_budget(run, total_budget / max(1, args.steps + args.warmup), M)
    for i in range(args.warmup):
        run((np.arange(rows) + i * rows) % M)
    t0 = time.perf_counter()
    for i in range(args.steps):
        run((np.arange(rows) + i * rows) % M)
    dt = time.perf_counter() - t0
    value = 2.0 * rows * N * K * args.steps / dt / 1e12
    cores = _oracle_threads()
    out = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOPS", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "impl": "reference",
           "config": {"workload": f"{spec.name}: {spec.description}", "layer": ls.name, "M": M, "K": K, "N": N,
                      "r": r, "rows_per_step": rows},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": cores,
                            "kind": "oracle",
                            "sample": f"{rows} rows of {M} per step (activation NVFP4 + float64 dequantized GEMM + low-rank branch + bias; the oracle's own pack and weight dequantization, untimed)"},
           "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_pair(args):
    """One step = the whole MLP pair of the workload (flux_mlp, or the fc1/fc2
    layers of flux_block): svdq_mlp_forward, i.e. fc1's activation kernel,
    fc1's GEMM with the GELU epilogue, fc2's activation kernel on H, fc2's
    GEMM.  Reported beside it: the same pair with GELU as a separate pass
    (torch, bf16) between the layers."""
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    import w4a4_rank_corrected_b200 as S
    spec = SI.workload_specs()[args.workload]
    wl = SI.make_workload(spec.name)
    names = [l.spec.name for l in wl.layers]
    i1 = names.index("fc1")
    l1, l2 = wl.layers[i1], wl.layers[i1 + 1]
    M, K1, N1, N2 = l1.spec.M, l1.spec.K, l1.spec.N, l2.spec.N
    X0 = wl.X_bf16 if i1 == 0 else SI.draw_activations(
        np.random.default_rng(spec.seed * 7919 + rank), M, K1, spec.x_dist, spec.x_outliers,
        spec.x_scale)
    if rank > 0 and i1 == 0:
        X0 = rank_activations(spec, rank, M, K1)
    p1 = S.svdq_pack_weight(l1.W, SI.channel_absmax(X0), l1.spec.r, bias_bf16=l1.bias_bf16)
    w1 = p1.to_device(dev)
    Xd = torch.from_numpy(X0.view(np.int16)).to(dev).view(torch.bfloat16)
    # fc2 is calibrated on the pair's own GELU output
    Hcal = S.svdq_debug_gelu(S.svdq_linear_forward(w1, Xd))
    hbits = Hcal.view(torch.int16).cpu().numpy().view(np.uint16)
    p2 = S.svdq_pack_weight(l2.W, SI.channel_absmax(hbits), l2.spec.r, bias_bf16=l2.bias_bf16)
    nsets = max(1, min(args.sets, 2))
    W1 = [p1.to_device(dev) for _ in range(nsets)]
    W2 = [p2.to_device(dev) for _ in range(nsets)]
    Xs = [Xd.clone() for _ in range(nsets)]
    Hs = [torch.empty((M, N1), dtype=torch.bfloat16, device=dev) for _ in range(nsets)]
    Ys = [torch.empty((M, N2), dtype=torch.bfloat16, device=dev) for _ in range(nsets)]
    wss = [S.new_mlp_workspace(M, W1[j], W2[j], dev) for j in range(nsets)]

    def fused(i):
        j = i % nsets
        S.svdq_mlp_forward(W1[j], W2[j], Xs[j], Hs[j], Ys[j], wss[j])

    def unfused(i):
        j = i % nsets
        Y1 = S.svdq_linear_forward(W1[j], Xs[j], Hs[j], wss[j])
        G = torch.nn.functional.gelu(Y1, approximate="tanh")
        S.svdq_linear_forward(W2[j], G, Ys[j], wss[j])

    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        fused(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(args.steps):
        fused(i)
    b.record()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(a.elapsed_time(b), world, dev) / args.steps
    for i in range(args.warmup):
        unfused(i)
    torch.cuda.synchronize(dev)
    a.record()
    for i in range(args.steps):
        unfused(i)
    b.record()
    torch.cuda.synchronize(dev)
    ms_unfused = max_over_ranks(a.elapsed_time(b), world, dev) / args.steps
    clocks = sampler.stop()
    err = S.svdq_device_error()
    if err:
        raise SystemExit(f"device error code {err:#x}")
    flops = 2.0 * M * (N1 * K1 + N2 * N1)
    out = {"metric": METRIC, "value": round(world * flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOPS",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
           "config": {"workload": f"{spec.name}: MLP pair fc1 {K1}->{N1}, GELU, fc2 {N1}->{N2}",
                      "M": M, "r": l1.spec.r,
                      "us_per_pair": round(ms * 1e3, 2),
                      "us_per_pair_unfused_gelu": round(ms_unfused * 1e3, 2),
                      "path": "svdq_mlp_forward: fc1 activation kernel, fc1 GEMM with the GELU "
                              "epilogue, fc2 activation kernel, fc2 GEMM; the unfused figure runs "
                              "torch's bf16 tanh GELU between the layers instead",
                      "l2": f"{nsets} rotating sets"},
           "gpu_launches": 4 * args.steps, "clocks": clocks}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_awq(args):
    """The AWQ W4A16 linear of a Flux modulation projection (adanorm_zero:
    hidden 3072 -> 6 x 3072), batch M = args.awq conditioning vectors,
    synthetic weights N(0, 0.02^2) and inputs N(0, 1).  Memory-bound: the
    roofline is the weight stream at the measured copy bandwidth."""
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import w4a4_rank_corrected_b200 as S
    M, K, N, group = args.awq, 3072, 6 * 3072, 128
    rng = np.random.default_rng(5 + rank)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    b = SI.f32_to_bf16_bits((rng.standard_normal(N) * 0.01).astype(np.float32))
    X0 = SI.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    nsets = 8     # 8 x 28 MB of weights > L2
    ws = [S.svdq_awq_pack(W, group, bias_bf16=b).to_device(dev) for _ in range(1)]
    ws = ws + [S.AwqWeight(N, K, group, ws[0].q, ws[0].zeros, ws[0].scales, b).to_device(dev)
               for _ in range(nsets - 1)]
    Xd = torch.from_numpy(X0.view(np.int16)).to(dev).view(torch.bfloat16)
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(nsets)]
    sampler = ClockSampler(local)
    sampler.start()
    for i in range(max(3, args.warmup)):
        S.svdq_awq_linear(ws[i % nsets], Xd, Ys[i % nsets])
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(200):
            S.svdq_awq_linear(ws[i % nsets], Xd, Ys[i % nsets])
    g.replay()
    torch.cuda.synchronize(dev)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(1, args.steps // 200)
    a.record()
    for _ in range(reps):
        g.replay()
    e.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    us = a.elapsed_time(e) / (reps * 200) * 1e3
    byts = N * K // 2 + N * (K // group) * 3 + M * K * 2 + M * N * 2 + N * 2
    peaks, src = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    out = {"metric": "AWQ W4A16 linear GB/s (weight stream) and us/layer", "value": round(byts / us / 1e3, 1),
           "unit": "GB/s", "n_gpus": 1, "steps": reps * 200, "warmup": args.warmup,
           "ms_per_step": round(us / 1e3, 6), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "int4 weights x bf16", "data": "synthetic",
           "config": {"workload": f"awq_w4a16 modulation linear K={K} N={N} group={group}, M={M}",
                      "us_per_layer": round(us, 2)},
           "roofline": {"bound": "hbm", "achieved": round(byts / us / 1e3, 1), "peak": hbm,
                        "unit": "GB/s", "frac": round(byts / us / 1e3 / hbm, 4),
                        "algorithmic_bytes": byts, "peak_source": src},
           "gpu_launches": reps * 200, "clocks": clocks}
    print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.awq:
        run_awq(args)
    elif args.pair:
        run_pair(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
