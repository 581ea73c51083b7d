#!/usr/bin/env python
"""Throughput of the fused SVDQuant W4A4 + low-rank linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    (N > 1: one rank per GPU under torch.distributed.run; started as a plain
    process, the script starts those N ranks itself)

One step = one pass of the whole hot path over one batch: kernel 1
(smoothing, NVFP4 quantization of X, down projection X_hat L1) and kernel 2
(block-scaled NVFP4 GEMM with the up projection folded into the same
accumulator, bias epilogue).  The weights are prepared once, outside the
timed region, as a model load would.

Workload: the attention-projection layer M = 4096 tokens, K = N = 3072,
rank 32, bf16 bias, Student-t(4) activations with 1 % outlier channels x 50,
N(0, 0.02) weights with 0.5 % outlier columns x 20 (synthetic, seeded).

Timing: each step is a CUDA graph (so host launch cost cannot bound the
GPU); steps rotate over buffer sets (X, activation buffer, Y and a copy of
the prepared layer) whose total exceeds the 126 MB L2, so every step reads
its operands from HBM.  CUDA events on the launching stream, max over ranks.
value = 2 M N K / step time, summed over ranks (weak scaling: every rank
runs its own batch; the layer has no cross-GPU exchange, so ranks are
replicas).  The roofline of each kernel counts its algorithmic bytes or
flops per launch (the formulas are in layer_flops and run_ours).
"""

import argparse
import datetime
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
METRIC = "fused W4A4+low-rank linear TFLOPS"
UNIT = "TFLOP/s"


# ----------------------------------------------------------------- workload
def workload_spec(name):
    from bit_w4a4_quantized_b200 import workloads as WL

    table = {"cfg1": WL.CFG1, "cfg2": WL.CFG2, "cfg3_fc1": WL.CFG3_FC1, "cfg3_fc2": WL.CFG3_FC2, "cfg4": WL.CFG4}
    if name in table:
        return table[name]
    if name.startswith("sweep:"):
        _, m, kn, r = name.split(":")
        return WL.sweep_spec(int(m), int(kn), int(r))
    raise SystemExit(f"unknown workload {name}")


def qkv_shape(N, head_dim=128):
    """True when N splits into Q | K | V of whole heads (the fused QKV epilogue applies)."""
    return N % 3 == 0 and (N // 3) % head_dim == 0


def layer_flops(spec, r_tot):
    """(FP4 GEMM flops, bf16 low-rank flops) of one forward of the layer."""
    fp4 = 2 * spec.M * spec.N * spec.K
    lowrank = 2 * spec.M * spec.K * r_tot + 2 * spec.M * spec.N * r_tot
    return fp4, lowrank


# ------------------------------------------------------------ multi-rank
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def rank_seed(base_seed, rank):
    """Each rank draws its own batch (weak scaling); rank 0 keeps the workload's seed."""
    return base_seed if rank == 0 else base_seed * 1000 + rank


def reduce_max(value, device=None):
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units, world, seconds_max):
    """Whole-job throughput: units of every rank over the slowest rank's time."""
    return per_rank_units * world / seconds_max


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region.

    All GPUs are sampled; rows are kept for the one whose UUID matches the
    benchmarked device (the first GPU if the UUID is unknown)."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = None if uuid is None else str(uuid).lower().replace("gpu-", "")
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self, load_mhz_floor=500):
        rows = [[x.strip() for x in l.split(",")] for l in self.lines]
        rows = [r for r in rows if len(r) >= 9]
        if self.uuid is not None and any(self.uuid in r[0].lower() for r in rows):
            rows = [r for r in rows if self.uuid in r[0].lower()]
        elif rows:
            first = rows[0][0]
            rows = [r for r in rows if r[0] == first]
        sm, mx, reasons = [], None, set()
        for r in rows:
            try:
                mhz, mx = float(r[1]), float(r[2])
            except ValueError:
                continue
            if mhz >= load_mhz_floor:
                sm.append(mhz)
                for n, v in zip(self.REASONS, r[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(sm)}


FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}  # an earlier measurement on the same B200 pool
FALLBACK_BF16_SUSTAINED = 1400.0  # the same GEMM back to back under the 1000 W cap (about 1.3 GHz)


def measured_peaks():
    """(bf16 TFLOP/s, HBM GB/s, origin) from MEASURED_PEAKS.json; a value that is
    missing, unreadable or not positive is replaced by the fallback, and the
    origin then says so."""
    d = {}
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        d = {}
    out, fell_back = [], []
    for key in ("bf16_tflops", "hbm_gbs"):
        v = d.get(key) if isinstance(d, dict) else None
        if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
            out.append(float(v))
        else:
            out.append(FALLBACK_PEAKS[key])
            fell_back.append(key)
    if not fell_back:
        origin = "measured"
    elif len(fell_back) == 2:
        origin = "fallback"
    else:
        origin = "measured, fallback for " + ", ".join(fell_back)
    return out[0], out[1], origin


def sustained_bf16_peak():
    """(bf16 TFLOP/s, origin) of a GEMM kept busy for seconds under the power cap, from
    MEASURED_PEAKS.json (`bf16_tflops_sustained`), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            v = json.load(fh).get("bf16_tflops_sustained")
    except (OSError, ValueError, AttributeError):
        v = None
    if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
        return float(v), "measured"
    return FALLBACK_BF16_SUSTAINED, "fallback"


def power_capped(clocks):
    """True when the clock samples of the timed region show the power cap holding the SM clock
    below its maximum: the kernels then run at the sustained rate, not the burst one."""
    if not clocks or "sw_power_cap" not in clocks.get("reasons", []):
        return False
    mhz, top = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    return mhz is not None and top is not None and mhz < top - 15


KERNEL_SOURCES = {
    "gemm_kernel": ("gemm.cu", "ptx.cuh", "layout.h", "kernels.h"),
    "act_quant_kernel": ("act_quant.cu", "ptx.cuh", "layout.h", "kernels.h"),
}
PROFILE_FILES = {
    "gemm_kernel": "gemm_kernel_attention_projection.md",
    "act_quant_kernel": "act_quant_kernel_attention_projection.md",
}


def kernel_source_hash(kernel):
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "bit_w4a4_quantized_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from the committed ncu summary,
    or None if the summary is for another workload or the kernel's source changed since the capture."""
    if workload != "attn_proj_M4096_K3072_N3072_r32":
        return None
    path = os.path.join(ROOT, "profiles", PROFILE_FILES[kernel])
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if "=" in line:
            k, _, v = line.strip().partition("=")
            fields[k.strip()] = v.strip()
    if fields.get("source_sha256_16") != kernel_source_hash(kernel):
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# -------------------------------------------------------------- CPU oracle
def oracle_throughput(spec, budget_s, min_steps=1, max_rows=None, steps=None, warmup=0):
    """Time the CPU oracle (quantize_act + linear) on a bounded sample of the workload.

    Returns (value TFLOP/s, seconds, steps, rows per step, threads)."""
    import threadpoolctl

    from oracle import svdquant as S

    X = spec.x(min(spec.M, 256)).astype(np.float32)
    W = spec.w().astype(np.float32)
    amax = np.max(np.abs(X), axis=0)
    b = spec.b()
    layer = S.prepare(W, amax, spec.rank, bias=None if b is None else b.astype(np.float64))
    _ = layer.deq_w  # weights are dequantized once per layer
    epi = S.EPI_GELU_TANH if spec.gelu else S.EPI_NONE
    # size the per-step sample from one calibration step
    t0 = time.perf_counter()
    S.linear(layer, S.quantize_act(layer, X[:1]), epi)
    t_row = max(time.perf_counter() - t0, 1e-4)
    n_steps = steps if steps is not None else max(min_steps, 1)
    rows = int(max(1, min(X.shape[0], max_rows or X.shape[0], budget_s / (n_steps + warmup) / t_row)))
    xs = X[:rows]
    for _ in range(warmup):
        S.linear(layer, S.quantize_act(layer, xs), epi)
    t0 = time.perf_counter()
    done = 0
    while True:
        S.linear(layer, S.quantize_act(layer, xs), epi)
        done += 1
        el = time.perf_counter() - t0
        if steps is not None:
            if done >= steps:
                break
        elif el >= budget_s and done >= min_steps:
            break
    el = time.perf_counter() - t0
    info = threadpoolctl.threadpool_info()
    threads = max([i.get("num_threads", 1) for i in info] or [1])
    flops = 2 * rows * spec.N * spec.K * done
    return flops / el / 1e12, el, done, rows, threads


# --------------------------------------------------------------- our arm
def flux_layer_point(spec, device, steps):
    """Kernel 1 and kernel 2 times of one FLUX-sized layer (its rank plus any LoRA rank), graph-timed over
    rotating buffer sets larger than L2, with kernel 2's fraction of the FP4 roofline: the extra keys of
    the bench line that carry the larger layers next to the headline one."""
    import torch

    from bit_w4a4_quantized_b200 import svdq
    from bit_w4a4_quantized_b200 import workloads as WL

    M, K, N = spec.M, spec.K, spec.N
    X = WL.make_x(M, K, spec.seed, spec.x_dist, spec.x_outliers, spec.x_outlier_scale)
    amax = svdq.calibrate_amax(X)
    r = spec.rank + (spec.lora_rank or 0)  # an adapter only adds ranks to the branch
    L0 = svdq.Layer(spec.w(), amax, r, bias=spec.b(), device=device)
    epi = svdq.EPI_GELU_TANH if spec.gelu else svdq.EPI_NONE
    Xd = torch.from_numpy(X.view(np.uint16).astype(np.int16)).view(torch.bfloat16).to(device)
    per_set = L0.device_bytes + L0.act_buffer_bytes(M) + 2 * M * K + 2 * M * N
    nsets = int(min(8, max(2, math.ceil(3 * L2_BYTES / per_set))))
    layers = [L0] + [L0.clone(device=device) for _ in range(nsets - 1)]
    Xs = [Xd] + [Xd.clone() for _ in range(nsets - 1)]
    acts = [L.new_act_buffer(M) for L in layers]
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(nsets):
            layers[i].quantize_act(Xs[i], acts[i])
            layers[i].linear(acts[i], M, out=Ys[i], epilogue=epi)
        stream.synchronize()
    k1 = _capture([lambda i=i: layers[i].quantize_act(Xs[i], acts[i]) for i in range(nsets)], stream)
    k2 = _capture([lambda i=i: layers[i].linear(acts[i], M, out=Ys[i], epilogue=epi) for i in range(nsets)], stream)
    t1 = _graph_seconds(k1, nsets, steps, stream, device)
    t2 = _graph_seconds(k2, nsets, steps, stream, device)
    for L in layers:
        L.poll_status()
    bf16_peak, _, peak_src = measured_peaks()
    fp4 = 2 * M * N * K
    roof_s = fp4 / (4.0 * bf16_peak * 1e12) + 2 * M * N * r / (bf16_peak * 1e12)
    out = {"M": M, "K": K, "N": N, "rank_total": r, "act_quant_us": round(t1 * 1e6, 3),
           "gemm_us": round(t2 * 1e6, 3), "gemm_TFLOPs": round(fp4 / t2 / 1e12, 1),
           "gemm_frac_of_roofline": round(roof_s / t2, 4), "peak_basis": f"{peak_src} bf16 x 4 (FP4)"}
    del k1, k2
    for L in layers:
        L.close()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    from bit_w4a4_quantized_b200 import svdq
    from bit_w4a4_quantized_b200 import workloads as WL

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    spec = workload_spec(args.workload)
    seed = rank_seed(spec.seed, rank)
    X = WL.make_x(spec.M, spec.K, seed, spec.x_dist, spec.x_outliers, spec.x_outlier_scale)
    W = spec.w()
    bias = spec.b()
    amax = svdq.calibrate_amax(X)  # calibrated on the batch it runs, like the parity tests
    t_prep = time.perf_counter()
    layer0 = svdq.Layer(W, amax, spec.rank, bias=bias, device=device)
    t_prep = time.perf_counter() - t_prep
    r_tot = layer0.info().rank_total
    lora_note = None
    if spec.lora_rank:
        layer0 = svdq.Layer(W, amax, spec.rank, rank_capacity=spec.rank + spec.lora_rank, bias=bias,
                            factors=(layer0.export(svdq.EXPORT_L1), layer0.export(svdq.EXPORT_L2)), device=device)
        A, B = spec.lora()
        to_dev = lambda a: torch.from_numpy(a.view(np.uint16).astype(np.int16)).view(torch.bfloat16).to(device)
        lora_dev = (to_dev(A), to_dev(B))
        layer0.lora_swap(*lora_dev)
        r_tot = layer0.info().rank_total
        lora_note = f"LoRA rank {spec.lora_rank} attached"
    epi = svdq.EPI_GELU_TANH if spec.gelu else svdq.EPI_NONE
    M, N, K = spec.M, spec.N, spec.K

    # buffer sets: (layer copy, X, act, Y); total > 3x L2 so each step misses L2
    Xd = torch.from_numpy(X.view(np.uint16).astype(np.int16)).view(torch.bfloat16).to(device)
    act_bytes = layer0.act_buffer_bytes(M)
    per_set = layer0.device_bytes + act_bytes + 2 * M * K + 2 * M * N
    nsets = int(min(16, max(2, math.ceil(3 * L2_BYTES / per_set))))
    layers = [layer0]
    for _ in range(nsets - 1):  # device copies of the same prepared layer
        L = layer0.clone(device=device)
        if spec.lora_rank:
            L.lora_swap(*lora_dev)
        layers.append(L)
    Xs = [Xd] + [Xd.clone() for _ in range(nsets - 1)]
    acts = [L.new_act_buffer(M) for L in layers]
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]

    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize(device)

    def q(i):
        layers[i].quantize_act(Xs[i], acts[i])

    def g(i):
        layers[i].linear(acts[i], M, out=Ys[i], epilogue=epi)

    with torch.cuda.stream(stream):
        for i in range(nsets):  # eager warm-up: sets function attributes, loads modules
            q(i)
            g(i)
        stream.synchronize()
        for L in layers:
            L.poll_status()

    def capture(fn):
        """One graph running fn over every buffer set in turn (launch cost amortised over nsets
        steps), and one graph per set for a remainder."""
        whole = torch.cuda.CUDAGraph()
        with torch.cuda.graph(whole, stream=stream, capture_error_mode="thread_local"):
            for i in range(nsets):
                fn(i)
        singles = []
        for i in range(nsets):
            cg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(cg, stream=stream, capture_error_mode="thread_local"):
                fn(i)
            singles.append(cg)
        return whole, singles

    step_graphs = capture(lambda i: (q(i), g(i)))
    k1_graphs = capture(q)
    k2_graphs = capture(g)

    def replay(graphs, steps):
        whole, singles = graphs
        for _ in range(steps // nsets):
            whole.replay()
        for i in range(steps % nsets):
            singles[i].replay()

    def timed(graphs, steps):
        """Seconds for exactly `steps` steps, CUDA events on the launching stream."""
        with torch.cuda.stream(stream):
            barrier(device)
            torch.cuda.synchronize(device)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            replay(graphs, steps)
            e1.record(stream)
            torch.cuda.synchronize(device)
            barrier(device)
        return e0.elapsed_time(e1) / 1e3

    with torch.cuda.stream(stream):
        replay(step_graphs, args.warmup)
    props = torch.cuda.get_device_properties(device)
    with ClockSampler(getattr(props, "uuid", None)) as clk:
        t_step = timed(step_graphs, args.steps)
    t_step_max = reduce_max(t_step, device)
    t_k1 = reduce_max(timed(k1_graphs, args.steps), device)
    t_k2 = reduce_max(timed(k2_graphs, args.steps), device)
    for L in layers:
        L.poll_status()

    # end to end through the public API with host buffers (pinned): every step copies its X in
    # and its Y out inside the timed region, double-buffered so both directions of the link and
    # the kernels overlap (svdq.HostPipeline)
    e2e_steps = max(3, min(args.steps, 100))  # the first copy in and the last copy out are not overlapped
    pipe = svdq.HostPipeline(layers[0], M, epilogue=epi)
    Xh = [Xd.cpu().pin_memory() for _ in range(2)]
    Yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    pipe.run([Xh[i % 2] for i in range(4)], [Yh[i % 2] for i in range(4)])  # warm-up
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    pipe.run([Xh[i % 2] for i in range(e2e_steps)], [Yh[i % 2] for i in range(e2e_steps)])
    pipe.s_in.wait_event(pipe.done_event())
    e1.record(pipe.s_in)
    torch.cuda.synchronize(device)
    barrier(device)
    t_e2e = reduce_max(e0.elapsed_time(e1) / 1e3, device)

    fp4, lowrank = layer_flops(spec, r_tot)
    value = aggregate(2 * M * N * K * args.steps, world, t_step_max) / 1e12
    e2e_value = aggregate(2 * M * N * K * e2e_steps, world, t_e2e) / 1e12

    # roofline of the dominant kernel: the burst bf16 peak, or the sustained one when the power
    # cap held the clock down during the timed region
    bf16_peak, hbm_peak, peak_src = measured_peaks()
    bf16_src = f"{peak_src} burst"
    clocks = clk.summary()
    if power_capped(clocks):
        bf16_peak, src = sustained_bf16_peak()
        bf16_src = f"{src} sustained"
    fp4_peak = bf16_peak * 4.0  # dense FP4 / BF16 nominal ratio (9 / 2.25 PFLOP/s)
    per_k2 = t_k2 / args.steps
    per_k1 = t_k1 / args.steps
    k2_flops = fp4 + 2 * M * N * r_tot
    k2_roof_s = fp4 / (fp4_peak * 1e12) + 2 * M * N * r_tot / (bf16_peak * 1e12)
    k1_bytes = 2 * M * K + M * K // 2 + M * K // 16 + 2 * M * r_tot + 2 * K * r_tot + 4 * K
    if per_k2 >= per_k1:
        roof = {"kernel": "svdq_gemm (kernel 2)", "bound": "tensor", "achieved": k2_flops / per_k2 / 1e12,
                "peak": k2_flops / k2_roof_s / 1e12, "unit": "TFLOP/s",
                "traffic": profiled_traffic("gemm_kernel", spec.name),
                "traffic_source": "dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture "
                                  "(profiles/gemm_kernel_attention_projection.md); Y stays in L2 during the kernel"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["peak_basis"] = (f"{bf16_src} bf16 {bf16_peak} TF/s x 4 (nominal FP4:BF16) for the FP4 flops, "
                              f"bf16 {bf16_peak} TF/s for the fold")
    else:
        roof = {"kernel": "act_quant (kernel 1)", "bound": "hbm", "achieved": k1_bytes / per_k1 / 1e9,
                "peak": hbm_peak, "unit": "GB/s", "traffic": profiled_traffic("act_quant_kernel", spec.name),
                "peak_basis": f"{peak_src} HBM copy"}
        roof["frac"] = roof["achieved"] / roof["peak"]

    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_step_max / args.steps * 1e3, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4(e2m1,e4m3 scales)+bf16 low-rank, fp32 acc",
        "data": "synthetic (seeded; stands in for FLUX.1 projection inputs)",
        "config": {"workload": spec.name, "M": M, "K": K, "N": N, "rank": spec.rank, "rank_total": r_tot,
                   "bias": bias is not None, "epilogue": "gelu_tanh" if spec.gelu else "none",
                   "lora": lora_note, "parallelism": f"replicas x{world} (no collective on the data path)",
                   "l2": f"rotating {nsets} buffer sets of {per_set / 2**20:.1f} MiB (X, act, Y, layer copy): "
                         f"{nsets * per_set / 2**20:.0f} MiB > L2",
                   "timing": f"CUDA graphs of {nsets} steps (one per buffer set), CUDA events"},
        "kernels": {"act_quant_us": round(per_k1 * 1e6, 3), "gemm_us": round(per_k2 * 1e6, 3),
                    "act_quant_GBps": round(k1_bytes / per_k1 / 1e9, 1),
                    "gemm_TFLOPs": round(k2_flops / per_k2 / 1e12, 1), "flops_fp4": fp4,
                    "flops_lowrank": lowrank, "prepare_s": round(t_prep, 3)},
        "roofline": {k: (round(v, 4) if isinstance(v, float) else v) for k, v in roof.items()},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": pipe.h2d_bytes,
                "d2h_bytes_per_step": pipe.d2h_bytes,
                "how": f"{e2e_steps} steps of svdq.HostPipeline: pinned host X in, both kernels, host Y out, "
                       "double-buffered over three streams"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_flux_layers:
        # kernel 2 on the larger FLUX layers too (outside the timed region)
        del step_graphs, k1_graphs, k2_graphs
        step_graphs = k1_graphs = k2_graphs = None
        torch.cuda.empty_cache()
        out["flux_layers"] = {s.name: flux_layer_point(s, device, 30)
                              for s in (WL.CFG3_FC1, WL.CFG3_FC2, WL.CFG4)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, el, done, rows, threads = oracle_throughput(spec, args.cpu_budget)
        out["cpu_baseline"] = {"value": round(v, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                               "sample": f"{rows} rows x {done} calls of the CPU oracle (quantize_act + linear, "
                                         f"float64 NumPy/BLAS) on the same layer, {el:.1f} s; "
                                         f"host has {os.cpu_count()} logical cores"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    del step_graphs, k1_graphs, k2_graphs
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ sweep
def _graph_seconds(graph, launches, steps, stream, device):
    """Mean seconds per launch: `graph` holds `launches` launches (one per buffer set) and is
    replayed until about `steps` launches ran; CUDA events on `stream`."""
    import torch

    reps = max(1, steps // launches)
    with torch.cuda.stream(stream):
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / 1e3 / (reps * launches)


def _capture(fns, stream):
    """One CUDA graph running every fn in turn."""
    import torch

    cg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cg, stream=stream, capture_error_mode="thread_local"):
        for fn in fns:
            fn()
    return cg


def sweep_point(spec, device, steps, factors_cache):
    """Kernel times of one shape at its rank and at rank 0, next to a bf16 cuBLAS linear.

    Low-rank factors come from one library SVD per (K, N) at the largest rank
    swept, truncated to each rank (timing does not depend on their values)."""
    import torch
    import torch.nn.functional as F

    from bit_w4a4_quantized_b200 import svdq
    from bit_w4a4_quantized_b200 import workloads as WL

    M, K, N = spec.M, spec.K, spec.N
    r = spec.rank + (spec.lora_rank or 0)  # an attached adapter only adds ranks to the branch
    cache = factors_cache
    xkey = (M, K, spec.seed, spec.x_dist, spec.x_outliers, spec.x_outlier_scale)
    if cache.get("x_key") != xkey:  # consecutive points often share X (and W)
        cache["x_key"], cache["x"] = xkey, None
        cache["x"] = WL.make_x(M, K, spec.seed, spec.x_dist, spec.x_outliers, spec.x_outlier_scale)
        cache["amax"] = svdq.calibrate_amax(cache["x"])
    X, amax = cache["x"], cache["amax"]
    wkey = (N, K, spec.seed, spec.w_outliers, spec.w_outlier_scale, spec.w_stream, spec.w_outlier_stream)
    if cache.get("w_key") != wkey:
        cache["w_key"], cache["w"] = wkey, None
        cache["w"] = spec.w()
    W = cache["w"]
    bias = spec.b()
    key = (K, N, spec.seed)  # one SVD per weight; its factors serve every M (timing ignores their values)
    r_max = max(64, r)
    if r > 0 and key not in factors_cache:
        base = svdq.Layer(W, amax, r_max, device=None)
        factors_cache[key] = (base.export(svdq.EXPORT_L1), base.export(svdq.EXPORT_L2))
        base.close()
    epi = svdq.EPI_GELU_TANH if spec.gelu else svdq.EPI_NONE
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.uint16).astype(np.int16)).view(
        torch.bfloat16).to(device)
    Xd = to_dev(X)
    stream = torch.cuda.Stream(device)
    out = {"workload": spec.name, "M": M, "K": K, "N": N, "rank": spec.rank, "rank_total": r,
           "epilogue": "gelu_tanh" if spec.gelu else "none", "bias": bias is not None}

    def layer_at(rank, fmt):
        fac = None
        if rank > 0:
            L1, L2 = factors_cache[key]
            fac = (np.ascontiguousarray(L1[:, :rank]), np.ascontiguousarray(L2[:rank]))
        return svdq.Layer(W, amax, rank, bias=bias, factors=fac, device=device, fmt=fmt)

    per_set = None
    # the NVFP4 layer at its rank and at rank 0, then the INT4 variant at its rank
    runs = ((r, "fused", svdq.FMT_NVFP4), (0, "plain", svdq.FMT_NVFP4)) if r > 0 else ((0, "plain", svdq.FMT_NVFP4),)
    for rank, tag, fmt in runs + ((r, "int4", svdq.FMT_INT4),):
        L0 = layer_at(rank, fmt)
        per_set = L0.device_bytes + L0.act_buffer_bytes(M) + 2 * M * K + 2 * M * N
        nsets = int(min(8, max(2, math.ceil(3 * L2_BYTES / per_set))))
        layers = [L0] + [L0.clone(device=device) for _ in range(nsets - 1)]
        Xs = [Xd] + [Xd.clone() for _ in range(nsets - 1)]
        acts = [L.new_act_buffer(M) for L in layers]
        Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]
        with torch.cuda.stream(stream):
            for i in range(nsets):
                layers[i].quantize_act(Xs[i], acts[i])
                layers[i].linear(acts[i], M, out=Ys[i], epilogue=epi)
            stream.synchronize()
        k1 = _capture([lambda i=i: layers[i].quantize_act(Xs[i], acts[i]) for i in range(nsets)], stream)
        k2 = _capture([lambda i=i: layers[i].linear(acts[i], M, out=Ys[i], epilogue=epi) for i in range(nsets)],
                      stream)
        t1 = _graph_seconds(k1, nsets, steps, stream, device)
        t2 = _graph_seconds(k2, nsets, steps, stream, device)
        if tag == "fused" and spec.name.startswith("qkv") and qkv_shape(N):
            # the fused QKV epilogue (per-head Q/K RMSNorm + rotary turn) on the same layers
            nq, nk = (to_dev(w) for w in WL.make_norm_weights(128, spec.seed))
            rope = torch.from_numpy(WL.make_rope(M, 128)).to(device)
            packed = svdq.rope_pack(rope, stream=stream)
            k3 = _capture([lambda i=i: layers[i].linear_qkv_norm_rope(acts[i], M, nq, nk, packed, out=Ys[i])
                           for i in range(nsets)], stream)
            t3 = _graph_seconds(k3, nsets, steps, stream, device)
            kp = _capture([lambda: svdq.rope_pack(rope, out=packed)], stream)
            tp = _graph_seconds(kp, 1, steps, stream, device)
            out["qkv_norm_rope_gemm_us"] = round(t3 * 1e6, 3)
            out["qkv_norm_rope_overhead_gemm"] = round(t3 / t2 - 1, 4)
            out["rope_pack_us"] = round(tp * 1e6, 3)
            del k3, kp
        for L in layers:
            L.poll_status()
        out[f"{tag}_act_us"] = round(t1 * 1e6, 3)
        out[f"{tag}_gemm_us"] = round(t2 * 1e6, 3)
        out[f"{tag}_layer_us"] = round((t1 + t2) * 1e6, 3)
        out[f"{tag}_gemm_TFLOPs"] = round(2 * M * N * K / t2 / 1e12, 1)
        out[f"{tag}_layer_TFLOPs"] = round(2 * M * N * K / (t1 + t2) / 1e12, 1)
        del k1, k2
        for L in layers:
            L.close()
        del layers, acts, Ys, Xs
    # bf16 cuBLAS dense GEMM of the same shape (X W^T, no bias or activation)
    Wd = to_dev(W)
    nsets = int(min(8, max(2, math.ceil(3 * L2_BYTES / (2 * (M * K + N * K + M * N))))))
    Xs = [Xd] + [Xd.clone() for _ in range(nsets - 1)]
    Ws = [Wd] + [Wd.clone() for _ in range(nsets - 1)]
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]

    mm = [lambda i=i: torch.matmul(Xs[i], Ws[i].t(), out=Ys[i]) for i in range(nsets)]
    with torch.cuda.stream(stream):
        for f in mm:
            f()
        stream.synchronize()
    gl = _capture(mm, stream)
    t_cb = _graph_seconds(gl, nsets, steps, stream, device)
    out["cublas_bf16_us"] = round(t_cb * 1e6, 3)
    out["cublas_bf16_TFLOPs"] = round(2 * M * N * K / t_cb / 1e12, 1)
    out["int4_layer_vs_nvfp4"] = round(out["int4_layer_us"] / out["fused_layer_us" if r > 0 else "plain_layer_us"], 3)
    # the INT4 GEMM runs on the f16 tensor path: its roofline is the measured bf16 rate (f16 runs at the same rate)
    bf16_peak, _, peak_kind = measured_peaks()
    out["int4_gemm_frac_of_bf16_peak"] = round(out["int4_gemm_TFLOPs"] / bf16_peak, 3)
    out["peak_kind"] = peak_kind
    if r > 0:
        out["lowrank_overhead_layer"] = round(out["fused_layer_us"] / out["plain_layer_us"] - 1, 4)
        out["lowrank_overhead_gemm"] = round(out["fused_gemm_us"] / out["plain_gemm_us"] - 1, 4)
        out["speedup_vs_cublas_bf16"] = round(t_cb / (out["fused_layer_us"] * 1e-6), 3)
    else:
        out["speedup_vs_cublas_bf16"] = round(t_cb / (out["plain_layer_us"] * 1e-6), 3)
    del gl
    return out


def w4a16_point(spec, device, steps):
    """The W4A16 layer on one modulation shape: kernel time over rotating weight copies (more than L2),
    the weight stream's GB/s against the measured HBM peak, and bf16 cuBLAS on the same shape."""
    import torch

    from bit_w4a4_quantized_b200 import svdq

    M, K, N = spec.M, spec.K, spec.N
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.uint16).astype(np.int16)).view(
        torch.bfloat16).to(device)
    W, s, b = spec.w(), spec.s(), spec.b()
    wbytes = N * K // 2 + N * K // 16
    nsets = int(min(8, max(2, math.ceil(3 * L2_BYTES / wbytes))))
    layers = []
    for _ in range(nsets):
        L = svdq.W4A16Layer(W, s=s, bias=b)
        L.upload(device)
        layers.append(L)
    Xd = to_dev(spec.x())
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(nsets):
            layers[i].linear(Xd, out=Ys[i], stream=stream)
        stream.synchronize()
    gr = _capture([lambda i=i: layers[i].linear(Xd, out=Ys[i], stream=stream) for i in range(nsets)], stream)
    t = _graph_seconds(gr, nsets, steps, stream, device)
    algo = wbytes + 4 * K + 2 * N + 2 * M * K + 2 * M * N  # weights, 1/s, bias, X, Y
    _, peak, peak_kind = measured_peaks()
    Wd = [to_dev(W) for _ in range(nsets)]
    Yc = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]
    mm = [lambda i=i: torch.matmul(Xd, Wd[i].t(), out=Yc[i]) for i in range(nsets)]
    with torch.cuda.stream(stream):
        for f in mm:
            f()
        stream.synchronize()
    gc = _capture(mm, stream)
    tc = _graph_seconds(gc, nsets, steps, stream, device)
    out = {"workload": spec.name, "layer": "w4a16", "M": M, "K": K, "N": N, "w4a16_us": round(t * 1e6, 3),
           "bytes": algo, "GBps": round(algo / t / 1e9, 1), "hbm_peak_GBps": peak, "peak_kind": peak_kind,
           "frac_of_hbm": round(algo / t / 1e9 / peak, 3),
           "cublas_bf16_us": round(tc * 1e6, 3), "speedup_vs_cublas_bf16": round(tc / t, 3)}
    del gr, gc
    for L in layers:
        L.close()
    return out


def mlp_pair_point(device, steps):
    """The MLP pair of the workload (fc1 3072 -> 12288 with GELU, fc2 12288 -> 3072, M = 4608, rank 32):
    the unfused pair (fc1's output written and read back) against the fused pair (fc1's epilogue
    writes fc2's activation buffer, then the partial-sum reduction), both over rotating buffer sets."""
    import torch

    from bit_w4a4_quantized_b200 import svdq
    from bit_w4a4_quantized_b200 import workloads as WL

    s1, s2 = WL.CFG3_FC1, WL.CFG3_FC2
    M = s1.M
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.uint16).astype(np.int16)).view(
        torch.bfloat16).to(device)
    X = s1.x()
    amax1 = svdq.calibrate_amax(X)
    g = np.random.default_rng([s1.seed, 99])
    # random bf16 factors stand in for the SVD (timing does not depend on their values)
    fac = lambda K, N, r: (WL.to_bf16(g.normal(0, 0.05, (K, r))), WL.to_bf16(g.normal(0, 0.05, (r, N))))
    fc1 = svdq.Layer(s1.w(), amax1, s1.rank, factors=fac(s1.K, s1.N, s1.rank), device=device)
    # fc2's calibration: the GELU output of fc1 on the batch, from the library's own unfused pass
    act = fc1.quantize_act(to_dev(X))
    h = fc1.linear(act, M, epilogue=svdq.EPI_GELU_TANH)
    hb = h.view(torch.int16).cpu().numpy().view(np.uint16)
    amax2 = svdq.calibrate_amax(hb.view(WL.BF16))
    fc2 = svdq.Layer(s2.w(), amax2, s2.rank, factors=fac(s2.K, s2.N, s2.rank), device=device)
    nsets = 2
    L1s = [fc1] + [fc1.clone(device=device) for _ in range(nsets - 1)]
    L2s = [fc2] + [fc2.clone(device=device) for _ in range(nsets - 1)]
    Xs = [to_dev(X) for _ in range(nsets)]
    a1 = [L.new_act_buffer(M) for L in L1s]
    a2 = [L.new_act_buffer(M) for L in L2s]
    H = [torch.empty((M, s1.N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]
    Y = [torch.empty((M, s2.N), dtype=torch.bfloat16, device=device) for _ in range(nsets)]
    ws = [torch.empty(fc1.mlp_workspace_bytes(fc2, M), dtype=torch.uint8, device=device) for _ in range(nsets)]
    stream = torch.cuda.Stream(device)

    def unfused(i):
        L1s[i].quantize_act(Xs[i], a1[i])
        L1s[i].linear(a1[i], M, out=H[i], epilogue=svdq.EPI_GELU_TANH)
        L2s[i].quantize_act(H[i], a2[i])
        L2s[i].linear(a2[i], M, out=Y[i])

    def fused(i):
        L1s[i].quantize_act(Xs[i], a1[i])
        L1s[i].linear_mlp(a1[i], M, L2s[i], act2=a2[i], workspace=ws[i])
        L2s[i].linear(a2[i], M, out=Y[i])

    def fused_gemm(i):
        L1s[i].linear_mlp(a1[i], M, L2s[i], act2=a2[i], workspace=ws[i])

    def plain_gemm(i):
        L1s[i].linear(a1[i], M, out=H[i], epilogue=svdq.EPI_GELU_TANH)

    with torch.cuda.stream(stream):
        for i in range(nsets):
            unfused(i)
            fused(i)
        stream.synchronize()
    out = {"workload": "mlp_pair_M4608_3072_12288_3072_r32", "M": M, "fc1": [s1.K, s1.N], "fc2": [s2.K, s2.N]}
    for tag, fn in (("unfused_pair", unfused), ("fused_pair", fused), ("fc1_gemm_plain", plain_gemm),
                    ("fc1_gemm_mlp_fused", fused_gemm)):
        gr = _capture([lambda i=i: fn(i) for i in range(nsets)], stream)
        out[f"{tag}_us"] = round(_graph_seconds(gr, nsets, steps, stream, device) * 1e6, 3)
        del gr
    flops = 2 * M * (s1.N * s1.K + s2.N * s2.K)
    out["unfused_pair_TFLOPs"] = round(flops / out["unfused_pair_us"] / 1e6, 1)
    out["fused_pair_TFLOPs"] = round(flops / out["fused_pair_us"] / 1e6, 1)
    out["fused_speedup"] = round(out["unfused_pair_us"] / out["fused_pair_us"], 3)
    for L in L1s + L2s:
        L.poll_status()
        L.close()
    return out


def run_sweep(args):
    import torch

    from bit_w4a4_quantized_b200 import workloads as WL

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    names = args.sweep.split(",")
    specs = []
    for n in names:
        if n == "all":
            specs += [WL.CFG2, WL.CFG3_FC1, WL.CFG3_FC2, WL.CFG4] + WL.sweep()
        elif n == "sweep":
            specs += WL.sweep()
        elif n == "w4a16":
            specs += [WL.w4a16_spec(m, N=nn) for nn in (18432, 9216) for m in (1, 2, 4)]
        elif n == "mlp":
            specs.append("mlp")
        else:
            specs.append(workload_spec(n))
    cache = {}
    props = torch.cuda.get_device_properties(device)
    for spec in specs:
        with ClockSampler(getattr(props, "uuid", None)) as clk:
            if spec == "mlp":
                row = mlp_pair_point(device, args.sweep_steps)
            elif isinstance(spec, WL.W4A16Spec):
                row = w4a16_point(spec, device, args.sweep_steps)
            else:
                row = sweep_point(spec, device, args.sweep_steps, cache)
        row["clocks"] = clk.summary()
        print(json.dumps(row), flush=True)
        torch.cuda.empty_cache()
    return 0


# --------------------------------------------------------- reference arm
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0  # the oracle runs on the host of rank 0 only
    spec = workload_spec(args.workload)
    # every step is a sample of the workload's rows; the budget spreads over all steps, so it is
    # larger than the cpu_baseline's, or a 2000-step run would time one-row calls (call overhead)
    budget = args.ref_budget
    v, el, done, rows, threads = oracle_throughput(spec, budget, steps=args.steps, warmup=args.warmup)
    out = {
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / done * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (oracle: float32 quantization decisions, float64 accumulation)",
        "data": "synthetic (seeded; stands in for FLUX.1 projection inputs)",
        "config": {"workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "rank": spec.rank,
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": round(v, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of {spec.M} rows per step, {done} steps, {el:.1f} s"},
        "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


def _free_port():
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_command(nproc, argv, port):
    """The torch.distributed.run command that starts `nproc` ranks of this script with `argv`."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + list(argv)


def relaunch(args, argv):
    """`--gpus N` (N > 1) started as a plain process: start N ranks under torch.distributed.run
    and return its exit status, so a multi-GPU run never silently measures one replica.  Our arm
    refuses at once when fewer than N GPUs are visible; the reference arm runs on rank 0's host
    cores and needs none."""
    if args.impl == "ours":
        import torch

        have = torch.cuda.device_count()
        if have < args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but only {have} CUDA device(s) are visible")
    cmd = relaunch_command(args.gpus, argv, _free_port())
    sys.stdout.flush()
    return subprocess.run(cmd, env={k: v for k, v in os.environ.items() if k not in
                                    ("RANK", "WORLD_SIZE", "LOCAL_RANK", "LOCAL_WORLD_SIZE")}).returncode


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="cfg2")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of CPU oracle work")
    ap.add_argument("--ref-budget", type=float, default=60.0,
                    help="seconds of CPU oracle work for --impl reference (spread over --steps + --warmup)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-flux-layers", action="store_true",
                    help="skip the extra per-layer kernel times of the larger FLUX layers")
    ap.add_argument("--sweep", default=None,
                    help="per-shape report instead of the bench line: 'all', 'sweep', 'w4a16', 'mlp' or workload names, "
                         "comma separated")
    ap.add_argument("--sweep-steps", type=int, default=50)
    args = ap.parse_args(argv)
    if args.sweep:
        return run_sweep(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    _, world, _ = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(args, sys.argv[1:] if argv is None else list(argv))
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
