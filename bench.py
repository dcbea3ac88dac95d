"""Benchmark of the sparse MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

A step is one forward of the whole layer (router, permutation, GEMM1 +
SwiGLU, GEMM2, combine) over one batch of synthetic tokens, with every input
already resident in HBM. K steps are timed with CUDA events between a barrier
and a device synchronisation on both sides; the maximum over ranks is taken.
Under torchrun every rank runs its own replica on its own token batch (tokens
are independent, no collective on the data path): weak scaling.

Prints one JSON line (rank 0). ``--impl reference`` times the CPU oracle on
the host cores instead (bounded token samples of the same workload).
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

import moe_inputs as mi  # noqa: E402

METRIC = "MoE layer tokens/s + achieved TFLOP/s or HBM GB/s as % of B200 roofline"
DEFAULT_CONFIG = "mixtral_prefill"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def rank_tokens(cfg, rank: int) -> np.ndarray:
    """Token batch of one replica: rank r draws its own x (seed r); the
    weights and router are shared by every rank."""
    return mi.make_x(cfg.with_(seed=cfg.seed + rank))


def max_over_ranks(value: float, dist, device=None) -> float:
    """All ranks take the same collective step; returns the max of `value`."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(T: int, world: int, ms_per_step: float) -> float:
    """Weak scaling: every rank processes T tokens per step; the job's time is the slowest rank's."""
    return world * T / (ms_per_step / 1e3)


def touched_weight_bytes(cfg, offsets, bytes_per_w=2.0):
    counts = np.diff(offsets)
    ne = int(np.sum(counts > 0))
    return ne * 3 * cfg.H * cfg.I * bytes_per_w, ne


def layer_roofline(flops: float, nbytes: float, ms_per_step: float, peaks: dict, ratio: float,
                   n_exp: int) -> dict:
    """The whole layer against both roofs: achieved TFLOP/s and GB/s with their
    fractions of the measured peaks (the tensor peak x `ratio` for FP8 / FP4),
    and the roofline time max(FLOPs / tensor peak, bytes / HBM bandwidth) with
    the fraction of it the step reaches (1.0 = at the roofline)."""
    s = ms_per_step / 1e3
    tpk = peaks["bf16_tflops_sustained"] * ratio
    roof_ms = max(flops / (tpk * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    return {"tflops": flops / s / 1e12, "tflops_frac": flops / s / 1e12 / tpk,
            "gbs": nbytes / s / 1e9, "gbs_frac": nbytes / s / 1e9 / peaks["hbm_gbs"],
            "roofline_ms": roof_ms, "roofline_frac": roof_ms / ms_per_step,
            "bound": "tensor" if flops / (tpk * 1e12) >= nbytes / (peaks["hbm_gbs"] * 1e9) else "hbm",
            "touched_experts": n_exp}


def kernel_traffic(cfg_name: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's sources are unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    ent = d.get(cfg_name, {}).get(kernel)
    if not ent:
        return None
    h = hashlib.sha256()
    for f in ent["sources"]:
        h.update(open(os.path.join(ROOT, "mixture_experts_layer_tcgen05_b200", "csrc", f), "rb").read())
    if h.hexdigest()[:16] != ent["source_sha"]:
        return None
    return ent["dram_bytes_per_launch"]


# ---------------------------------------------------------------------------
# CPU oracle (baseline only)
# ---------------------------------------------------------------------------
def oracle_inputs(cfg, L):
    """Keyword arguments for oracle.moe_forward; FP8 weights are quantised by the oracle itself."""
    import oracle

    if cfg.fp4:
        return {"fp4": oracle.quant_weight_fp4(L["w13"]) + oracle.quant_weight_fp4(L["w2"])}
    if cfg.fp8:
        w13q, w13s = oracle.quant_weight_fp8(L["w13"], ue8m0=cfg.ue8m0)
        w2q, w2s = oracle.quant_weight_fp8(L["w2"], ue8m0=cfg.ue8m0)
        return {"fp8": (w13q, w13s, w2q, w2s), "ue8m0": cfg.ue8m0}
    return {"w13": L["w13"], "w2": L["w2"]}


def cpu_model() -> str | None:
    """The host CPU's model name (first `model name` line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_tokens_per_s(cfg, L, budget_s: float, kw=None):
    import oracle

    T = cfg.T
    kw = oracle_inputs(cfg, L) if kw is None else kw

    def run(n):
        toks = mi.token_subset(cfg, n) if n < T else np.arange(T, dtype=np.int32)
        t0 = time.perf_counter()
        oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, tokens=toks, **kw)
        return time.perf_counter() - t0

    n0 = min(T, max(1, oracle.threads()))
    t0 = run(n0)
    per_tok = t0 / n0
    n = int(min(T, max(n0, budget_s / max(per_tok, 1e-9))))
    t = run(n) if n != n0 else t0
    return n / t, n, t


def reference_arm(args, cfg):
    import oracle

    rank, _, world = dist_env()
    if rank != 0:
        return
    L = mi.make_layer(cfg)
    kw = oracle_inputs(cfg, L)
    total_budget = float(os.environ.get("MOE_REF_BUDGET_S", "120"))
    per_step = max(2.0, total_budget / max(1, args.steps + args.warmup))
    # calibrate the sample size to the per-step budget
    _, n, t = oracle_tokens_per_s(cfg, L, per_step, kw)
    toks = mi.token_subset(cfg, n) if n < cfg.T else np.arange(cfg.T, dtype=np.int32)
    for _ in range(args.warmup):
        oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, tokens=toks, **kw)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, tokens=toks, **kw)
        times.append(time.perf_counter() - t0)
    value = len(toks) * args.steps / sum(times)
    sample = f"{len(toks)} of {cfg.T} tokens per step (seeded subset), whole layer per token"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.desc, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(),
                         "cpu": cpu_model(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def gpu_arm(args, cfg):
    import torch

    import mixture_experts_layer_tcgen05_b200 as moe

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    def barrier():
        if dist is not None:
            dist.barrier()

    # each rank draws its own token batch; weights are shared
    L = mi.make_layer(cfg)
    if rank > 0:
        L["x"] = rank_tokens(cfg, rank)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    x, wr = bf(L["x"]), bf(L["wr"])
    bias = torch.from_numpy(L["bias"]).cuda()
    w13, w2 = bf(L["w13"]), bf(L["w2"])
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    quant = cfg.fp8 or cfg.fp4
    dt = (moe.MOE_DTYPE_FP4_E2M1 if cfg.fp4 else
          (moe.MOE_DTYPE_FP8_E4M3_UE8M0 if cfg.ue8m0 else moe.MOE_DTYPE_FP8_E4M3) if cfg.fp8
          else moe.MOE_DTYPE_BF16)
    sfmt = moe.MOE_SCALE_UE8M0 if cfg.ue8m0 else moe.MOE_SCALE_F32
    if cfg.fp4:
        # one-time weight preparation (untimed): packed e2m1 with one e8m0 scale per (row, 32)
        w13q = torch.empty(cfg.E, 2 * cfg.I, cfg.H // 2, dtype=torch.uint8, device="cuda")
        w13s = torch.empty(cfg.E, 2 * cfg.I, cfg.H // 32, dtype=torch.uint8, device="cuda")
        w2q = torch.empty(cfg.E, cfg.H, cfg.I // 2, dtype=torch.uint8, device="cuda")
        w2s = torch.empty(cfg.E, cfg.H, cfg.I // 32, dtype=torch.uint8, device="cuda")
        moe.moe_quantize_weight_fp4(w13, cfg.E, 2 * cfg.I, cfg.H, w13q, w13s)
        moe.moe_quantize_weight_fp4(w2, cfg.E, cfg.H, cfg.I, w2q, w2s)
        torch.cuda.synchronize()
        del w13, w2
    elif cfg.fp8:
        # one-time weight preparation (untimed): e4m3 with one scale per 128 x 128 block
        w13q = torch.empty(cfg.E, 2 * cfg.I, cfg.H, dtype=torch.uint8, device="cuda")
        w13s = torch.empty(cfg.E, 2 * cfg.I // 128, cfg.H // 128, dtype=torch.float32, device="cuda")
        w2q = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.uint8, device="cuda")
        w2s = torch.empty(cfg.E, cfg.H // 128, cfg.I // 128, dtype=torch.float32, device="cuda")
        moe.moe_quantize_weight_fp8_fmt(w13, cfg.E, 2 * cfg.I, cfg.H, w13q, w13s, sfmt)
        moe.moe_quantize_weight_fp8_fmt(w2, cfg.E, cfg.H, cfg.I, w2q, w2s, sfmt)
        torch.cuda.synchronize()
        del w13, w2
    ws_bytes = moe.moe_workspace_size(d, dt)
    io_bytes = cfg.T * cfg.H * 2
    io_al = (io_bytes + 255) // 256 * 256
    ws = torch.zeros(ws_bytes + 2 * io_al, dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(xin=None):
        xin = x if xin is None else xin
        if cfg.fp4:
            moe.moe_forward_fp4(xin, wr, bias, w13q, w13s, w2q, w2s, d, moe.MOE_EPILOGUE_SWIGLU, out,
                                ws, ws_bytes)
        elif cfg.fp8 and cfg.ue8m0:
            moe.moe_forward_fp8_ue8m0(xin, wr, bias, w13q, w13s, w2q, w2s, d, moe.MOE_EPILOGUE_SWIGLU,
                                      out, ws, ws_bytes)
        elif cfg.fp8:
            moe.moe_forward_fp8(xin, wr, bias, w13q, w13s, w2q, w2s, d, out, ws, ws_bytes)
        else:
            moe.moe_forward(xin, wr, bias, w13, w2, d, out, ws, ws_bytes)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    status = moe.moe_get_device_status(ws)
    if status != 0:
        raise SystemExit(f"device status {status} after warm-up")
    lay = moe.moe_workspace_layout(d)
    offsets = ws[lay.offsets:lay.offsets + 4 * (cfg.E + 1)].cpu().numpy().view(np.int32)

    # ---- timed region: K forwards, stage events per step ----
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(torch.cuda.current_device())
    if rank == 0:
        clocks.start()
    barrier()
    torch.cuda.synchronize()
    n0 = moe.moe_launch_count()
    t_start.record(stream)
    for i in range(args.steps):
        moe.moe_set_stage_events(stage_ev[i])
        step()
    t_end.record(stream)
    moe.moe_set_stage_events(None)
    torch.cuda.synchronize()
    barrier()
    launches = moe.moe_launch_count() - n0
    clk = clocks.stop() if rank == 0 else None
    ms = t_start.elapsed_time(t_end)
    stages = np.array([[ev[j].elapsed_time(ev[j + 1]) for j in range(5)] for ev in stage_ev])
    stage_ms = stages.mean(0)
    ms = max_over_ranks(ms, dist, "cuda")
    ms_per_step = ms / args.steps
    value = whole_job_tokens_per_s(cfg.T, world, ms_per_step)

    # ---- the same forward replayed from a CUDA graph (launch overhead removed) ----
    graph = None
    try:
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            step()  # warm the capture stream
            cs.synchronize()
            with torch.cuda.graph(g, stream=cs):
                step()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        gms = max_over_ranks(g0.elapsed_time(g1), dist, "cuda") / args.steps
        graph = {"ms_per_step": gms, "value": whole_job_tokens_per_s(cfg.T, world, gms),
                 "unit": "tokens/s"}
        del g
    except Exception as exc:  # reported, not fatal: the eager number above stands
        graph = {"error": str(exc)[:200]}

    # ---- end to end: pinned host tokens in, pinned host result out, every step ----
    # Two streams with a workspace each: step i+1's host->device copy runs on
    # the copy engine while step i computes (as a serving loop would overlap).
    x_host = torch.from_numpy(np.ascontiguousarray(L["x"]).view(np.int16)).pin_memory()
    streams = [stream, torch.cuda.Stream()]
    wss = [ws, torch.zeros_like(ws)]
    outs_host = [torch.empty(cfg.T * cfg.H, dtype=torch.int16).pin_memory() for _ in range(2)]
    outs_dev = [out, torch.empty_like(out)]
    xs_dev = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    def e2e_step(i):
        j = i & 1
        with torch.cuda.stream(streams[j]):
            if quant:
                xs_dev[j].view(torch.int16).copy_(x_host.view(cfg.T, cfg.H), non_blocking=True)
                if cfg.fp4:
                    moe.moe_forward_fp4(xs_dev[j], wr, bias, w13q, w13s, w2q, w2s, d,
                                        moe.MOE_EPILOGUE_SWIGLU, outs_dev[j], wss[j], ws_bytes,
                                        stream=streams[j])
                elif cfg.ue8m0:
                    moe.moe_forward_fp8_ue8m0(xs_dev[j], wr, bias, w13q, w13s, w2q, w2s, d,
                                              moe.MOE_EPILOGUE_SWIGLU, outs_dev[j], wss[j], ws_bytes,
                                              stream=streams[j])
                else:
                    moe.moe_forward_fp8(xs_dev[j], wr, bias, w13q, w13s, w2q, w2s, d, outs_dev[j],
                                        wss[j], ws_bytes, stream=streams[j])
                outs_host[j].copy_(outs_dev[j].view(torch.int16).view(-1), non_blocking=True)
            else:  # the C ABI's host-buffer entry point does both copies on its stream
                moe.moe_forward_hostio(x_host, wr, bias, w13, w2, d, outs_host[j], wss[j],
                                       stream=streams[j])

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    streams[1].wait_stream(stream)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_stream(streams[1])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ems = e0.elapsed_time(e1)
    ems = max_over_ranks(ems, dist, "cuda")
    e2e_value = whole_job_tokens_per_s(cfg.T, world, ems / args.steps)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    flops = 6.0 * cfg.T * cfg.k * cfg.H * cfg.I
    # bytes per expert weight: e2m1 + one e8m0 byte per 32; e4m3 (+ block scales, counted below); bf16
    wbytes, n_exp = touched_weight_bytes(cfg, offsets, (0.5 + 1.0 / 32) if cfg.fp4 else
                                         1.0 if cfg.fp8 else 2.0)
    layer_bytes = wbytes + 2 * cfg.T * cfg.H * 2 + cfg.H * cfg.E * 2
    gemm1_ms = float(stage_ms[2])
    decode = cfg.T * cfg.k <= 64 * cfg.E and cfg.T <= 64
    if decode:
        # touched expert weights of GEMM-1 (e4m3 codes + one fp32 scale per 128 x 128 block)
        g1_bytes = n_exp * 2 * cfg.H * cfg.I * ((0.5 + 1.0 / 32) if cfg.fp4 else
                                                (1.0 + 4.0 / (128 * 128)) if cfg.fp8 else 2.0)
        ach = g1_bytes / (gemm1_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"],
                "traffic": kernel_traffic(cfg.name, "gemm1"),
                "kernel": ("gemm_mx_kernel<SwiGLU, e2m1 B> (FP4 GEMM1 + SwiGLU + h quantisation)"
                           if cfg.fp4 else
                           "gemm_mx_kernel<SwiGLU> (block-scaled FP8 GEMM1 + SwiGLU + h quantisation)"
                           if cfg.ue8m0 else
                           "gemm_rows_fp8_kernel<SwiGLU> (FP8 GEMM1 + SwiGLU + h quantisation)"
                           if cfg.fp8 else "gemm_swap_kernel<SwiGLU> (GEMM1, small-M)"),
                "algorithmic_bytes_per_launch": g1_bytes, "peak_source": peak_src}
    else:
        g1_flops = 4.0 * cfg.T * cfg.k * cfg.H * cfg.I
        ach = g1_flops / (gemm1_ms / 1e3) / 1e12
        # FP8 peak = the measured bf16 peak x the nominal fp8/bf16 ratio (2); e4m3 x e2m1 runs on
        # the same f8f6f4 MMA, at the FP8 rate
        ratio = 2.0 if quant else 1.0
        pk, pk_burst = ratio * peaks["bf16_tflops_sustained"], ratio * peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
                "traffic": kernel_traffic(cfg.name, "gemm1"),
                "kernel": ("gemm_mx_kernel<SwiGLU, e2m1 B> (block-scaled FP4 GEMM1 + SwiGLU + h "
                           "quantisation)" if cfg.fp4 else
                           "gemm_mx_kernel<SwiGLU> (block-scaled FP8 GEMM1 + SwiGLU + h quantisation)"
                           if cfg.ue8m0 else
                           "gemm_rows_fp8_kernel<SwiGLU> (FP8 GEMM1 + SwiGLU + h quantisation)" if cfg.fp8
                           else "gemm_rows_kernel<SwiGLU,256> (GEMM1 + SwiGLU on the permuted rows)"),
                "algorithmic_flops_per_launch": g1_flops,
                "peak_source": f"{peak_src} bf16 x {ratio:g} (sustained; burst {pk_burst:.1f} -> frac "
                               f"{ach / pk_burst:.3f})"}
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("e4m3 x e2m1 -> fp32 (experts), bf16 router" if cfg.fp4 else
                  "e4m3 x e4m3 -> fp32 (experts), bf16 router" if cfg.fp8 else "bf16 x bf16 -> fp32"),
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights)",
        "config": {"workload": cfg.desc, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "parallelism": f"token-parallel replicas x{world}",
                   "l2": f"inputs larger than L2: {wbytes / 1e9:.2f} GB of expert weights read "
                         "per step, no flush"},
        "roofline": roof,
        "layer": layer_roofline(flops, layer_bytes, ms_per_step, peaks, 2.0 if quant else 1.0, n_exp),
        "stages_us": {n: round(float(v) * 1e3, 2) for n, v in
                      zip(["route", "permute", "gemm1", "gemm2", "combine"], stage_ms)},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
                "d2h_bytes_per_step": io_bytes},
        "graph": graph,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle

        v, n, t = oracle_tokens_per_s(cfg, L, float(os.environ.get("MOE_CPU_BUDGET_S", "20")))
        res["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": oracle.threads(),
                               "cpu": cpu_model(), "kind": "oracle",
                               "sample": f"{n} of {cfg.T} tokens (seeded subset), whole layer "
                                         f"per token, {t:.1f} s"}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(mi.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shape", default="",
                    help="override dims of the config, e.g. T=2048,E=64 (for a smaller profiling "
                         "case; the workload name then says so)")
    args = ap.parse_args()
    cfg = mi.CONFIGS[args.config]
    if args.shape:
        over = {k: int(v) for k, v in (kv.split("=") for kv in args.shape.split(","))}
        bad = set(over) - {"T", "H", "I", "E", "k"}
        if bad:
            raise SystemExit(f"--shape takes T, H, I, E, k (got {sorted(bad)})")
        cfg = cfg.with_(**over, name=f"{cfg.name}@{args.shape}", desc=f"{cfg.desc}; resized to " +
                        " ".join(f"{k}={v}" for k, v in over.items()))
    if args.impl == "reference":
        reference_arm(args, cfg)
    else:
        gpu_arm(args, cfg)


if __name__ == "__main__":
    main()
