"""Benchmark of the FFN-service MoE layer on B200: tokens/s per layer and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config dsv3_256] [--impl ours|reference]
                    [--shapes dsv3_4096,w8a8_8192]

One step = one afd_ffn_forward over one micro-batch (router, top-k, dispatch, gate/up GEMM
with SwiGLU, down GEMM, shared expert, combine).  Default workload: the DeepSeek-V3 shaped
decode micro-batch (T=256, H=7168, E=256 + 1 shared, top-8, I=2048, bf16) on seeded
synthetic inputs.  On one GPU the same line also carries, under "shapes", the T=4096
Zipf-skewed bf16 micro-batch, the T=8192 W8A8 chunk and the T=256 W8A8 decode micro-batch,
each timed the same way (K steps after W warm-ups) with its own roofline, stage split and
clock record.  Its 22.6 GB of expert weights are far larger than the 126 MB L2, so no
flush is needed between steps.  N > 1 runs one independent replica per GPU (the layer is
not sharded: no collective on the data path); value = total tokens of all ranks / the
slowest rank's time.  --impl reference times the fp64 CPU oracle on a bounded sample of the
same workload instead (the reference arm).

    python bench.py --period [--config dsv3_256]

measures the FFN-service micro-pipeline instead: a host attention stub of set duration t_a
feeds the library's serving loop with one or two micro-batches in flight, and the period is
compared with the A/F split's model max(t_a, t_f) + t_comm and with t_a + t_f on one device.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from concurrent.futures import ThreadPoolExecutor  # noqa: E402

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the fused bf16 expert kernel
# of the decode shape, from an ncu capture of a small case of the same kernel (T=16, H=7168,
# E=16 + 1 shared, k=8, I=2048: all 17 experts touched, 1.5 GB of weights): 1 499 667 712 +
# 5 541 888 bytes in one launch.  The weight stream dominates, so the traffic grows with the
# experts whose weights are streamed and is scaled by them; it is reported only while the
# kernel sources and the file that instantiates them are the ones that were captured.
MEASURED_TRAFFIC = {
    "sources_sha256": "bf25b6660b8e09b8d7390c6d39413cbf5b1ccdef277ed8ffb4afae47bae4a6b6",
    "bytes_per_touched_expert": (1499667712 + 5541888) / 17,
}
METRIC = "MoE-FFN tokens/s/layer"


# ----------------------------------------------------------------------------- accounting
def touched_experts(counts, n_shared) -> int:
    return int(np.count_nonzero(np.asarray(counts))) + n_shared


def algorithmic(cfg, counts) -> dict:
    """Per-forward algorithmic bytes and FLOPs (compulsory traffic only).

    weights: every touched expert's W13 and W2 (+ e4m3 scales); activations: the hidden read,
    the output write and the router weight read.  FLOPs: 6 H I (T k + S T) + 2 T H E.
    gemm13: the gate/up GEMM alone -- touched W13 (+ scales), its dispatched input rows and its
    SwiGLU output rows.
    """
    T, H, E, k, I, S = cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.S
    b = 1 if cfg.dtype == "fp8" else 2
    n = touched_experts(counts, S)
    w13 = n * (2 * I * H * b + (2 * I * 4 if b == 1 else 0))
    w2 = n * (H * I * b + (H * 4 if b == 1 else 0))
    act = T * H * 2 + T * H * 2 + E * H * 4
    rows = T * k + S * T
    gemm13 = w13 + rows * H * b + rows * I * (4 if b == 1 else 2)
    # the fused bf16 expert kernel (gate/up + SwiGLU + down): weights, dispatched rows in, outputs out
    expert = w13 + w2 + rows * H * b + rows * H * 4
    flops = 6 * H * I * (T * k + S * T) + 2 * T * H * E
    return {"weight_bytes": w13 + w2, "w13_bytes": w13, "act_bytes": act, "flops": flops, "gemm13_bytes": gemm13,
            "expert_bytes": expert,
            "gemm13_flops": 4 * H * I * rows, "touched_experts": n}


def kernel_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ("gemm.cuh", "ptx.cuh", "common.cuh", "afd_ffn.cu"):
        with open(os.path.join(ROOT, "ffn_side_expert_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def fused_traffic(cfg, acct):
    """Measured DRAM bytes per fused expert-kernel launch scaled to this workload's touched
    experts, or None when the kernel sources (the kernel, its PTX helpers and the file that
    instantiates it) changed since the capture."""
    if kernel_sources_sha256() != MEASURED_TRAFFIC["sources_sha256"]:
        return None
    return int(round(MEASURED_TRAFFIC["bytes_per_touched_expert"] * acct["touched_experts"]))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 20 ms; only the samples written while
    the timed region runs (between entering and leaving the context) are summarised."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.f = None
        self.first = self.last = 0

    def _lines(self) -> list:
        self.f.flush()
        with open(self.f.name) as fh:
            return [r for r in fh.read().splitlines() if r.count(",") >= 8]

    def __enter__(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        if self.proc is not None:
            t_end = time.monotonic() + 3.0        # wait until the sampler is producing lines
            while time.monotonic() < t_end and not self._lines():
                time.sleep(0.02)
            self.first = len(self._lines())
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.last = len(self._lines())
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if self.proc is None or self.f is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        lines = self._lines()
        os.unlink(self.f.name)
        # samples written during the timed region; the one just before it when the region is
        # shorter than the sampling period
        window = lines[self.first:self.last] if self.last > self.first else lines[max(0, self.first - 1):self.first]
        rows = [r.split(",") for r in window]
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                power.append(float(r[3]))
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "sm_mhz_min": min(sm) if sm else None, "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons), "samples": len(sm), "period_ms": 20}


# ----------------------------------------------------------------------------- our arm
def build_inputs(cfg, device):
    """Seeded inputs; the experts go straight to the device (no host copy of the stack, so N
    ranks on one node do not each hold 22.6 GB of host memory)."""
    hidden = synth.gen_hidden(cfg)
    Wr, bias = synth.gen_router(cfg)
    dev = synth.gen_experts_on(cfg, device)
    dev["router_w"] = Wr.to(device)
    if bias is not None:
        dev["router_bias"] = bias.to(device)
    return hidden, Wr, bias, dev


def cpu_baseline(cfg, hidden, Wr, bias, budget_s=15.0) -> dict:
    """The fp64 oracle, as it stands, on the first few tokens of the same micro-batch.  The
    experts those tokens visit are drawn on the host before each timed call."""
    from oracle import moe
    try:
        from threadpoolctl import threadpool_info
        blas = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        blas = None
    cores = len(os.sched_getaffinity(0))
    cache = {}
    fn = lambda e: cache[e]  # noqa: E731
    n, spent, done = 1, 0.0, 0
    while True:
        _, idx, _ = moe.route(hidden[:n], Wr, bias, cfg.k)
        need = sorted((set(np.unique(idx).tolist()) | set(range(cfg.E, cfg.E + cfg.S))) - set(cache))
        with ThreadPoolExecutor(max(1, min(16, cores))) as pool:
            cache.update(zip(need, pool.map(lambda e: synth.gen_expert(cfg, e), need)))
        t0 = time.perf_counter()
        moe.forward(hidden[:n], Wr, bias, fn, cfg.E, cfg.k, cfg.S, fp8=cfg.dtype == "fp8")
        dt = time.perf_counter() - t0
        spent, done = dt, n
        if dt > budget_s / 3 or n >= cfg.T:
            break
        n = min(cfg.T, n * 4)
    return {"value": done / spent, "unit": "tokens/s", "cores": blas or cores, "host_cores": cores,
            "kind": "oracle",
            "sample": f"first {done} of {cfg.T} tokens of the {cfg.name} micro-batch, full fp64 layer "
                      f"(routing, {cfg.k} experts + {cfg.S} shared per token), {spent:.1f} s"}


def workload(args):
    cfg = synth.CONFIGS[args.config]
    over = {k: v for k, v in (("T", args.T), ("E", args.E)) if v is not None}
    return cfg.with_(**over) if over else cfg


def workload_label(args) -> str:
    over = [f"{k}={v}" for k, v in (("T", args.T), ("E", args.E)) if v is not None]
    return args.config + (f"[{','.join(over)}]" if over else "")


def time_forward(layer, h, out, cfg, args, world, local_rank) -> dict:
    """W warm-up forwards, then K timed forwards back to back with CUDA events around the
    whole region and around the dominant kernel (stage 5 -> 6: the fused expert kernel of the
    bf16 decode shape, else the gate/up GEMM), nvidia-smi clocks sampled meanwhile; then a
    second pass of K forwards with every stage boundary recorded for the per-stage split."""
    import ffn_side_expert_b200 as afd
    device = h.device
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        layer.forward(h, out)
    torch.cuda.synchronize()
    st = layer.get_error()
    if st != afd.AFD_OK:
        raise afd.AfdError(st, "warm-up")

    # routing counts of this micro-batch (for the touched-expert byte count)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=device)
    wts = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=device)
    layer.route(h, cfg.T, idx, wts)
    counts = np.bincount(idx.cpu().numpy().ravel(), minlength=cfg.E)
    acct = algorithmic(cfg, counts)

    nev = afd.AFD_FFN_NUM_STAGES + 1
    K0, K1 = 5, 6
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sparse = [[kev[i][0] if s == K0 else kev[i][1] if s == K1 else None for s in range(nev)]
              for i in range(args.steps)]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # torch creates an event's CUDA handle at its first record; create every handle now, so that
    # inside the timed region the stream carries only the two records around the dominant kernel
    for e in [x for pair in kev for x in pair] + [t_start, t_end]:
        e.record(stream)

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            layer.set_stage_events(sparse[i])
            layer.forward(h, out)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    layer.set_stage_events(None)
    ms = t_start.elapsed_time(t_end) / args.steps
    kernel_ms = float(np.mean([kev[i][0].elapsed_time(kev[i][1]) for i in range(args.steps)]))
    st = layer.get_error()
    if st != afd.AFD_OK:
        raise afd.AfdError(st, "timed region")
    for i in range(args.steps):
        layer.set_stage_events(ev[i])
        layer.forward(h, out)
    torch.cuda.synchronize()
    layer.set_stage_events(None)
    stage_ms = np.array([[ev[i][s].elapsed_time(ev[i][s + 1]) for s in range(nev - 1)]
                         for i in range(args.steps)]).mean(axis=0)
    return {"ms": allreduce_max(ms, world), "kernel_ms": allreduce_max(kernel_ms, world),
            "stage_ms": stage_ms, "acct": acct, "cfg": cfg, "clocks": clk.summary()}


def run_ours(args, rank, world, local_rank):
    import ffn_side_expert_b200 as afd
    cfg = workload(args)
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    hidden, Wr, bias, dev = build_inputs(cfg, device)
    layer = afd.AfdFfn(T_max=cfg.T, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.S,
                       fp8=cfg.dtype == "fp8", weights=dev)
    h = hidden.to(device)
    out = torch.empty_like(h)
    stream = torch.cuda.current_stream()
    res = time_forward(layer, h, out, cfg, args, world, local_rank)

    # the same K forwards without any events, timed the same way
    barrier(world)
    torch.cuda.synchronize()
    u0 = torch.cuda.Event(enable_timing=True)
    u1 = torch.cuda.Event(enable_timing=True)
    u0.record(stream)
    for i in range(args.steps):
        layer.forward(h, out)
    u1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    plain_ms = u0.elapsed_time(u1) / args.steps

    # the same forward replayed from a CUDA graph (launch gaps removed), timed the same way
    graph_ms = None
    gs = torch.cuda.Stream()
    gs.wait_stream(stream)
    with torch.cuda.stream(gs):
        layer.forward(h, out, stream=gs)
    stream.wait_stream(gs)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=gs):
        layer.forward(h, out, stream=gs)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(args.steps):
        g.replay()
    g1.record(stream)
    torch.cuda.synchronize()
    graph_ms = g0.elapsed_time(g1) / args.steps
    del g
    st = layer.get_error()
    if st != afd.AFD_OK:
        raise afd.AfdError(st, "graph replay")

    # end to end: host buffers through the C ABI, each step's H2D and D2H copies inside the
    # timed region.  (1) the FFN-service loop over K micro-batches (copies overlapped with the
    # layer); (2) one synchronous call per micro-batch.
    hin = [hidden.clone().pin_memory() for _ in range(2)]
    hout = [torch.empty_like(hidden).pin_memory() for _ in range(2)]
    seq_in = [hin[i % 2] for i in range(args.steps)]
    seq_out = [hout[i % 2] for i in range(args.steps)]
    layer.forward_host_batches(seq_in[:2], seq_out[:2])
    barrier(world)
    t0 = time.perf_counter()
    layer.forward_host_batches(seq_in, seq_out)
    e2e_s = (time.perf_counter() - t0) / args.steps
    barrier(world)
    t0 = time.perf_counter()
    for i in range(args.steps):
        layer.forward_host(seq_in[i], seq_out[i])
    e2e_sync_s = (time.perf_counter() - t0) / args.steps

    res.update(graph_ms=allreduce_max(graph_ms, world), plain_ms=allreduce_max(plain_ms, world),
               e2e_s=allreduce_max(e2e_s, world), e2e_sync_s=allreduce_max(e2e_sync_s, world),
               bytes_io=hidden.numel() * 2)
    if rank == 0 and not args.no_cpu_baseline:
        res["cpu"] = cpu_baseline(cfg, hidden, Wr, bias)
    layer.close()
    del layer, dev, h, out, hin, hout, seq_in, seq_out
    torch.cuda.empty_cache()
    return res


def run_shape(name, args, world, local_rank) -> dict:
    """One more workload timed like the headline (warm-up, K timed forwards, stage pass); its
    handle and weights are freed before returning."""
    import ffn_side_expert_b200 as afd
    cfg = synth.CONFIGS[name]
    device = torch.device("cuda", local_rank)
    hidden, _, _, dev = build_inputs(cfg, device)
    layer = afd.AfdFfn(T_max=cfg.T, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.S,
                       fp8=cfg.dtype == "fp8", weights=dev)
    h = hidden.to(device)
    out = torch.empty_like(h)
    try:
        return time_forward(layer, h, out, cfg, args, world, local_rank)
    finally:
        layer.close()
        del layer, dev, h, out
        torch.cuda.empty_cache()


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def allreduce_max(x: float, world: int) -> float:
    """Max over ranks (the slowest replica sets the job's time)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_replica: int, world: int, slowest_ms: float) -> float:
    """Whole-job tokens/s: every replica's tokens over the slowest replica's step time."""
    return world * tokens_per_replica / (slowest_ms / 1e3)


def fused_decode(cfg) -> bool:
    """The bf16 decode shape runs its expert GEMMs as one fused launch."""
    return cfg.dtype == "bf16" and cfg.T * cfg.k <= 32 * cfg.E


def launches_per_step(cfg) -> int:
    """Library kernel launches of one forward: router GEMM, top-k selection and gate weights,
    dispatch count, dispatch scan, gather, schedule, then the fused expert kernel (bf16 decode
    shape) or gate/up GEMM (+ W8A8 activation quantisation) and down GEMM, then combine."""
    return 8 if fused_decode(cfg) else (10 if cfg.dtype == "fp8" else 9)


def rooflines(cfg, acct, ms, kernel_ms, traffic=None):
    """(roofline of the dominant kernel, roofline of the whole path) for one workload.

    Dominant kernel: the fused expert kernel of the bf16 decode shape, else the gate/up GEMM.
    Its algorithmic bytes are the expert weights it must stream (touched experts only, plus
    the e4m3 scales); its algorithmic FLOPs are 2 per multiply-add of its products.  It is
    reported against whichever of the HBM and tensor-core peaks bounds it (the larger of
    bytes / HBM and FLOPs / tensor peak), with the other fraction beside it.
    Path: t_roof = max(FLOPs / tensor peak, (weight + activation bytes) / HBM) over t_step."""
    peaks, kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    mult = 2.0 if cfg.dtype == "fp8" else 1.0          # e4m3 vs bf16 dense tensor rate
    tc = peaks["bf16_tflops"] * mult
    tc_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * mult
    if fused_decode(cfg):
        kname, kbytes, kflops = ("expert FFN kernel (gate/up + SwiGLU + down, fused)", acct["weight_bytes"],
                                 acct["flops"] - 2 * cfg.T * cfg.H * cfg.E)
    else:
        kname, kbytes, kflops = "grouped_gemm gate/up + SwiGLU", acct["w13_bytes"], acct["gemm13_flops"]
    sec = kernel_ms / 1e3
    gbs, tfs = kbytes / sec / 1e9, kflops / sec / 1e12
    tensor_bound = kflops / (tc * 1e12) > kbytes / (hbm * 1e9)
    roof = {"bound": "tensor" if tensor_bound else "hbm",
            "kernel": kname,
            "achieved": round(tfs if tensor_bound else gbs, 1),
            "peak": tc if tensor_bound else hbm,
            "unit": "TFLOP/s" if tensor_bound else "GB/s",
            "frac": round((tfs / tc) if tensor_bound else (gbs / hbm), 4),
            "traffic": traffic,
            "peak_source": f"{kind} " + ("bf16_tflops x 2 (e4m3)" if tensor_bound and mult == 2 else
                                         "bf16_tflops" if tensor_bound else "hbm_gbs"),
            "algorithmic_bytes_per_launch": kbytes, "algorithmic_flops_per_launch": kflops,
            "avg_launch_ms": round(kernel_ms, 4),
            "hbm_frac": round(gbs / hbm, 4), "tensor_frac": round(tfs / tc, 4),
            "tensor_frac_sustained": round(tfs / tc_sus, 4)}
    t_hbm = (acct["weight_bytes"] + acct["act_bytes"]) / (hbm * 1e9)
    t_tc = acct["flops"] / (tc * 1e12)
    t_roof = max(t_hbm, t_tc)
    # the same bound with the tensor peak a GEMM sustains under the power cap (the timed steps
    # run back to back, and the clock record shows sw_power_cap under load)
    t_roof_sus = max(t_hbm, acct["flops"] / (tc_sus * 1e12))
    path = {"t_roof_ms": round(t_roof * 1e3, 4), "t_hbm_ms": round(t_hbm * 1e3, 4),
            "t_tensor_ms": round(t_tc * 1e3, 4), "frac": round(t_roof * 1e3 / ms, 4),
            "weight_bytes": acct["weight_bytes"], "act_bytes": acct["act_bytes"],
            "flops": acct["flops"], "touched_experts": acct["touched_experts"],
            "peaks": f"{kind}: hbm {hbm} GB/s, tensor {tc} TFLOP/s (burst)",
            "frac_sustained": round(t_roof_sus * 1e3 / ms, 4),
            "t_roof_sustained_ms": round(t_roof_sus * 1e3, 4),
            "peaks_sustained": f"{kind}: hbm {hbm} GB/s, tensor {round(tc_sus, 1)} TFLOP/s (sustained)"}
    return roof, path


def report_shape(args, world, r) -> dict:
    """The JSON object of one extra workload (same timing as the headline's value)."""
    import ffn_side_expert_b200 as afd
    cfg = r["cfg"]
    roof, path = rooflines(cfg, r["acct"], r["ms"], r["kernel_ms"])
    return {"value": round(job_throughput(cfg.T, world, r["ms"]), 1), "unit": "tokens/s",
            "ms_per_step": round(r["ms"], 4),
            "dtype": "fp8_e4m3" if cfg.dtype == "fp8" else "bf16",
            "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k, "I": cfg.I,
                       "n_shared": cfg.S, "weights": cfg.dtype, "seed": cfg.seed,
                       "routing": "Zipf-skewed (router bias)" if cfg.has_bias else "uniform"},
            "roofline": roof, "path_roofline": path,
            "stage_ms": {k: round(float(v), 4) for k, v in zip(afd.STAGE_NAMES, r["stage_ms"])},
            "gpu_launches": launches_per_step(cfg) * args.steps, "clocks": r["clocks"]}


def report_ours(args, world, r) -> dict:
    import ffn_side_expert_b200 as afd
    cfg, acct = r["cfg"], r["acct"]
    ms = r["ms"]
    value = job_throughput(cfg.T, world, ms)
    stage = dict(zip(afd.STAGE_NAMES, [float(x) for x in r["stage_ms"]]))
    traffic = fused_traffic(cfg, acct) if fused_decode(cfg) else None
    roof, path = rooflines(cfg, acct, ms, r["kernel_ms"], traffic)
    launches = launches_per_step(cfg)
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3" if cfg.dtype == "fp8" else "bf16", "data": "synthetic",
        "config": {"workload": workload_label(args), "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k,
                   "I": cfg.I, "n_shared": cfg.S, "weights": cfg.dtype, "seed": cfg.seed,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2 (expert weights {acct['weight_bytes'] / 1e9:.1f} GB >> 126 MB)"},
        "roofline": roof,
        "path_roofline": path,
        "stage_ms": {k: round(v, 4) for k, v in stage.items()},
        "uninstrumented": {"value": round(job_throughput(cfg.T, world, r["plain_ms"]), 1), "unit": "tokens/s",
                           "ms_per_step": round(r["plain_ms"], 4),
                           "how": "the same K eager forwards without the per-stage events, CUDA events"},
        "graph": {"value": round(job_throughput(cfg.T, world, r["graph_ms"]), 1), "unit": "tokens/s",
                  "ms_per_step": round(r["graph_ms"], 4),
                  "how": "one afd_ffn_forward captured in a CUDA graph, replayed K times, CUDA events"},
        "e2e": {"value": round(job_throughput(cfg.T, world, r["e2e_s"] * 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": r["bytes_io"], "d2h_bytes_per_step": r["bytes_io"],
                "api": "afd_ffn_forward_host_batches (pinned host buffers, copies overlapped with the layer)",
                "sync_per_call_value": round(job_throughput(cfg.T, world, r["e2e_sync_s"] * 1e3), 1),
                "sync_per_call_api": "afd_ffn_forward_host, one synchronous call per micro-batch"},
        "gpu_launches": launches * args.steps,
        "clocks": r["clocks"],
        "cpu_baseline": r.get("cpu"),
    }


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The fp64 CPU oracle timed on the host, a bounded token sample per step."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import moe
    if rank != 0:
        return None
    cfg = workload(args)
    hidden = synth.gen_hidden(cfg)
    Wr, bias = synth.gen_router(cfg)
    n = max(1, int(args.ref_tokens))
    plan = [[(i * n + j) % cfg.T for j in range(n)] for i in range(args.warmup + args.steps)]
    # the experts the sampled tokens visit are drawn before any timing
    _, idx, _ = moe.route(hidden[sorted({t for p in plan for t in p})], Wr, bias, cfg.k)
    need = sorted(set(np.unique(idx).tolist()) | set(range(cfg.E, cfg.E + cfg.S)))
    with ThreadPoolExecutor(max(1, min(16, len(os.sched_getaffinity(0))))) as ex:
        cache = dict(zip(need, ex.map(lambda e: synth.gen_expert(cfg, e), need)))
    steps = []
    for i, tok in enumerate(plan):
        t0 = time.perf_counter()
        moe.forward(hidden, Wr, bias, cache.__getitem__, cfg.E, cfg.k, cfg.S, fp8=cfg.dtype == "fp8",
                    tokens=tok)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            steps.append(dt)
    per_tok = sum(steps) / (n * len(steps))
    value = 1.0 / per_tok
    cores = len(os.sched_getaffinity(0))
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * per_tok * cfg.T, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(args), "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k,
                   "I": cfg.I, "n_shared": cfg.S, "weights": cfg.dtype, "seed": cfg.seed},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} token(s) of the {cfg.name} micro-batch per step, full fp64 layer "
                                   f"(expert weights drawn before timing); ms_per_step scaled to T={cfg.T}"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- micro-pipeline period
def _busy_until(t_end_ns: int) -> None:
    while time.monotonic_ns() < t_end_ns:
        pass


def pipeline_period(layer, hidden_host, T, t_a_ms, n_slots, rounds, ref_out=None):
    """One attention stub and the FFN serving loop, `n_slots` micro-batches in flight.

    The attention side is a host stub: per micro-batch it writes the seeded hidden rows into a
    mailbox slot (one memmove on its own thread) and holds the thread busy until t_a has passed
    since it started, then posts the slot; it waits for a slot's output before it starts that
    slot's next micro-batch.  The
    FFN side is the library's serving loop (H2D, afd_ffn_forward, D2H on three streams).  The
    period is the mean interval between outputs landing in host memory (the times the
    library stamps when each D2H completes), after the first round.  Returns (period_ms,
    outputs that differ from ref_out, service stats, median post->take and take->landed ms)."""
    from ffn_side_expert_b200.service import FfnService, Mailbox
    mb = Mailbox(n_slots, T, hidden_host.shape[1])
    svc = FfnService(layer, mb)
    t_a_ns = int(t_a_ms * 1e6)
    rows = hidden_host[:T].contiguous()

    def attention(slot):
        t_end = time.monotonic_ns() + t_a_ns
        mb.write_input(slot, rows)
        _busy_until(t_end)

    nbytes = T * hidden_host.shape[1] * 2
    ref_bytes = None if ref_out is None else ref_out[:T].contiguous().view(torch.int16).numpy().tobytes()
    landed, pickup, serve, tl, mismatches = [], [], [], [], 0
    try:
        for s in range(n_slots):
            attention(s)
            mb.post(s, T)
        for r in range(rounds):
            for s in range(n_slots):
                mb.wait(s, timeout_s=60.0)
                t_post, t_take, t_done = mb.times_ns(s)
                landed.append(t_done)
                if r:
                    pickup.append((t_take - t_post) / 1e6)
                    serve.append((t_done - t_take) / 1e6)
                    tl.append(svc.timeline(s))
                if ref_bytes is not None and r in (0, rounds - 1):   # single-threaded byte compare
                    mismatches += int(ctypes.string_at(mb.output(s).data_ptr(), nbytes) != ref_bytes)
                if r < rounds - 1:
                    attention(s)
                    mb.post(s, T)
    finally:
        stats = svc.stop()
        mb.close()
    w = n_slots
    period_mean = (landed[-1] - landed[w]) / (len(landed) - 1 - w) / 1e6
    # per-round periods (n_slots outputs each) after the first round; the median is robust to a
    # host stall in one round, the mean is reported beside it
    rounds_ms = [(landed[i + n_slots] - landed[i]) / n_slots / 1e6 for i in range(w, len(landed) - n_slots)]
    period = statistics.median(rounds_ms)
    # device timeline: layer start / end of each micro-batch on one clock (the service's origin)
    spans = sorted((m[0] + m[2], m[0] + m[3]) for m in tl)
    gaps = [b0 - a1 for (_, a1), (b0, _) in zip(spans, spans[1:])]
    med = lambda xs: round(statistics.median(xs), 4)  # noqa: E731
    parts = {"post_to_take_ms": med(pickup), "take_to_landed_ms": med(serve),
             "period_mean_ms": round(period_mean, 4),
             "h2d_ms": med([m[1] for m in tl]), "h2d_end_to_layer_ms": med([m[2] - m[1] for m in tl]),
             "layer_ms": med([m[3] - m[2] for m in tl]),
             "layer_gap_ms": med(gaps) if gaps else None,
             "d2h_after_layer_ms": med([m[4] - m[3] for m in tl]),
             # host take -> landed minus the device span H2D start -> D2H end: enqueue latency
             # plus the time from the D2H end to the completion reaching the mailbox
             "host_overhead_ms": med([sv - m[4] for sv, m in zip(serve, tl)])}
    return period, mismatches, stats, parts


def period_models(t_a, t_f, t_h2d, t_d2h, slots) -> dict:
    """Steady-state period of the A/F micro-pipeline, ms per micro-batch.

    page: the A/F 分离 page's model (section 深入推导, 微流水), max(t_a, t_f) + t_comm with
    micro-batches overlapped, t_a + t_f + t_comm without (one slot).
    cycle: a bound for the serving loop, whose copies overlap the layer.  The attention side
    and the layer each serve one micro-batch at a time, and one slot's micro-batch goes round
    attention -> H2D -> layer -> D2H before the slot is used again, so with `slots` of them in
    flight the period is at least max(t_a, t_f, (t_a + t_h2d + t_f + t_d2h) / slots)."""
    t_comm = t_h2d + t_d2h
    page = (max(t_a, t_f) if slots > 1 else t_a + t_f) + t_comm
    cycle = max(t_a, t_f, (t_a + t_h2d + t_f + t_d2h) / slots)
    return {"page": page, "cycle": cycle, "colocated": t_a + t_f}


def period_point(t_a, slots, period, parts, t_f, t_h2d, t_d2h) -> dict:
    """One measured point of --period with its models: the page's, the cycle bound from the
    isolated layer and copy times, and the cycle bound again from the times measured in the
    loop (parts: the breakdown pipeline_period returns)."""
    m = period_models(t_a, t_f, t_h2d, t_d2h, slots)
    m_in_loop = period_models(t_a, parts["layer_ms"], parts["h2d_ms"], parts["d2h_after_layer_ms"], slots)
    return {"t_a_ms": round(t_a, 4), "slots": slots, "period_ms": round(period, 4),
            "model_ms": round(m["page"], 4), "cycle_bound_ms": round(m["cycle"], 4),
            "cycle_bound_in_loop_ms": round(m_in_loop["cycle"], 4),
            "colocated_ms": round(m["colocated"], 4),
            "period_over_colocated": round(period / m["colocated"], 3), **parts}


def run_period(args) -> dict:
    """The micro-pipeline period of the A/F split (A/F 分离 page, section 深入推导, 微流水): the
    steady-state period with the attention of one micro-batch overlapping the FFN of another,
    against max(t_a, t_f) + t_comm and against t_a + t_f when both share one device."""
    import ffn_side_expert_b200 as afd
    cfg = workload(args)
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    hidden, Wr, bias, dev = build_inputs(cfg, device)
    layer = afd.AfdFfn(T_max=cfg.T, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.S,
                       fp8=cfg.dtype == "fp8", weights=dev)
    T, H = cfg.T, cfg.H
    h = hidden.to(device)
    out = torch.empty_like(h)
    for _ in range(args.warmup):
        layer.forward(h, out)
    torch.cuda.synchronize()
    ref_out = out.cpu()
    if layer.get_error() != afd.AFD_OK:
        raise RuntimeError("device error word set during warm-up")

    def device_ms(fn, reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    reps = max(args.steps, 5)
    t_f = device_ms(lambda: layer.forward(h, out), reps)
    host_in = hidden.pin_memory()
    host_out = torch.empty_like(host_in).pin_memory()
    t_h2d = device_ms(lambda: h.copy_(host_in, non_blocking=True), reps)
    t_d2h = device_ms(lambda: host_out.copy_(out, non_blocking=True), reps)
    t_comm = t_h2d + t_d2h
    points, bad = [], 0
    rounds = max(args.steps, 8)
    for ratio in (0.5, 1.0, 1.5):
        t_a = ratio * t_f
        for slots in (1, 2):
            period, mism, st, parts = pipeline_period(layer, host_in, T, t_a, slots, rounds, ref_out)
            bad += mism
            if st.status != afd.AFD_OK or st.device_status != afd.AFD_OK:
                raise afd.AfdError(st.status or st.device_status, "FFN service")
            points.append(period_point(t_a, slots, period, parts, t_f, t_h2d, t_d2h))
    return {
        "metric": "FFN-service micro-pipeline period", "unit": "ms", "higher_is_better": False,
        "config": {"workload": workload_label(args), "T": T, "H": H, "E": cfg.E, "k": cfg.k, "I": cfg.I,
                   "n_shared": cfg.S, "weights": cfg.dtype, "attention": "host stub, busy t_a per micro-batch",
                   "link": "PCIe host<->device copies (pinned)", "rounds": rounds},
        "t_f_ms": round(t_f, 4), "t_comm_ms": {"h2d": round(t_h2d, 4), "d2h": round(t_d2h, 4), "sum": round(t_comm, 4)},
        "models": {"model_ms": "slots=1: t_a + t_f + t_comm; slots=2: max(t_a, t_f) + t_comm",
                   "cycle_bound_ms": "max(t_a, t_f, (t_a + t_h2d + t_f + t_d2h) / slots)",
                   "cycle_bound_in_loop_ms": "the same with the H2D, layer and D2H times measured in the loop",
                   "colocated_ms": "t_a + t_f"},
        "points": points, "outputs_bit_equal_to_forward": bad == 0,
    }


# ----------------------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="dsv3_256", choices=list(synth.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=1, help="reference arm: tokens per step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--T", type=int, default=None,
                    help="profiling only: override the micro-batch size (a smaller case of the same kernels)")
    ap.add_argument("--E", type=int, default=None,
                    help="profiling only: override the number of routed experts")
    ap.add_argument("--shapes", default="dsv3_4096,w8a8_8192,w8a8_256",
                    help="comma-separated workloads timed after the headline one (1 GPU only; '' for none)")
    ap.add_argument("--period", action="store_true",
                    help="measure the FFN-service micro-pipeline period with a host attention stub (1 GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.period:
        if world > 1:
            ap.error("--period runs on one GPU")
        print(json.dumps(run_period(args)), flush=True)
        return 0

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local_rank))
    try:
        r = run_ours(args, rank, world, local_rank)
        # the other shapes the metric names, timed the same way on the same GPU after the
        # headline one (replica runs across GPUs time the headline workload only)
        shapes = {}
        names = [n for n in args.shapes.split(",") if n and n != args.config] if world == 1 else []
        if args.T is None and args.E is None:
            for name in names:
                shapes[name] = report_shape(args, world, run_shape(name, args, world, local_rank))
        if rank == 0:
            line = report_ours(args, world, r)
            if shapes:
                line["shapes"] = shapes
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
