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
DEFAULT_CONFIG = "fine_grained"
# measured on the same line as the headline workload (the other full-size configurations)
EXTRA_CONFIGS = ["mixtral_prefill", "mixtral_decode", "fine_grained_fp8"]
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
BURST_REGION_MS = 1000.0  # timed regions shorter than this are compared with the burst peak


def tensor_peak(peaks: dict, ratio: float, region_ms: float):
    """(peak TFLOP/s, label): the measured bf16 peak x `ratio` (the nominal FP8/bf16 ratio
    for the FP8 and FP4 layers), burst for a region under a second, sustained otherwise."""
    if region_ms < BURST_REGION_MS or "bf16_tflops_sustained" not in peaks:
        return ratio * peaks["bf16_tflops"], "burst"
    return ratio * peaks["bf16_tflops_sustained"], "sustained"


def cublas_peaks(torch, n: int = 8192, reps: int = 10) -> dict:
    """Dense cuBLAS throughput on this GPU, best of `reps` CUDA-event-timed n^3 products:
    bf16 (torch.matmul) and e4m3 (torch._scaled_mm, bf16 out), plus a 2 GiB copy."""
    def best(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return min(ts)

    g = torch.Generator(device="cuda").manual_seed(0)
    a = torch.randn(n, n, device="cuda", dtype=torch.bfloat16, generator=g)
    b = torch.randn(n, n, device="cuda", dtype=torch.bfloat16, generator=g)
    out = {"n": n, "reps": reps}
    out["bf16_tflops"] = 2 * n ** 3 / best(lambda: torch.matmul(a, b)) / 1e9
    a8 = a.to(torch.float8_e4m3fn)
    b8 = b.to(torch.float8_e4m3fn).t()  # column-major second operand, as _scaled_mm wants
    one = torch.ones((), device="cuda", dtype=torch.float32)
    out["e4m3_tflops"] = 2 * n ** 3 / best(
        lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)) / 1e9
    del a, b, a8, b8
    src = torch.empty(1 << 30, dtype=torch.bfloat16, device="cuda")
    dst = torch.empty_like(src)
    out["hbm_copy_gbs"] = 2 * src.numel() * 2 / best(lambda: dst.copy_(src)) / 1e6
    return out


class Workload:
    """One workload's inputs resident in HBM and its forward through the C ABI.

    bf16 expert weights are drawn once per (H, I, E, seed) and shared: the FP8 and
    FP4 layers quantise them on the device (one-time, untimed preparation)."""

    def __init__(self, cfg, rank: int, wcache: dict):
        import torch

        import mixture_experts_layer_tcgen05_b200 as moe

        self.cfg, self.moe = cfg, moe
        L = {"x": mi.make_x(cfg) if rank == 0 else rank_tokens(cfg, rank)}
        L["wr"], L["bias"] = mi.make_router(cfg)
        key = (cfg.H, cfg.I, cfg.E, cfg.seed, cfg.w_sigma)
        if key not in wcache:
            wcache.clear()
            L["w13"], L["w2"] = mi.make_w13(cfg), mi.make_w2(cfg)
            wcache[key] = (L["w13"], L["w2"], self.bf(L["w13"]), self.bf(L["w2"]))
        L["w13"], L["w2"], w13, w2 = wcache[key]
        self.L = L
        self.x, self.wr = self.bf(L["x"]), self.bf(L["wr"])
        self.bias = torch.from_numpy(L["bias"]).cuda()
        self.d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
        self.quant = cfg.fp8 or cfg.fp4
        self.dt = (moe.MOE_DTYPE_FP4_E2M1 if cfg.fp4 else
                   (moe.MOE_DTYPE_FP8_E4M3_UE8M0 if cfg.ue8m0 else moe.MOE_DTYPE_FP8_E4M3)
                   if cfg.fp8 else moe.MOE_DTYPE_BF16)
        sfmt = moe.MOE_SCALE_UE8M0 if cfg.ue8m0 else moe.MOE_SCALE_F32
        E, H, I = cfg.E, cfg.H, cfg.I
        if cfg.fp4:
            # packed e2m1 with one e8m0 scale per (row, 32)
            self.w = [torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device="cuda"),
                      torch.empty(E, 2 * I, H // 32, dtype=torch.uint8, device="cuda"),
                      torch.empty(E, H, I // 2, dtype=torch.uint8, device="cuda"),
                      torch.empty(E, H, I // 32, dtype=torch.uint8, device="cuda")]
            moe.moe_quantize_weight_fp4(w13, E, 2 * I, H, self.w[0], self.w[1])
            moe.moe_quantize_weight_fp4(w2, E, H, I, self.w[2], self.w[3])
        elif cfg.fp8:
            # e4m3 with one scale per 128 x 128 block
            self.w = [torch.empty(E, 2 * I, H, dtype=torch.uint8, device="cuda"),
                      torch.empty(E, 2 * I // 128, H // 128, dtype=torch.float32, device="cuda"),
                      torch.empty(E, H, I, dtype=torch.uint8, device="cuda"),
                      torch.empty(E, H // 128, I // 128, dtype=torch.float32, device="cuda")]
            moe.moe_quantize_weight_fp8_fmt(w13, E, 2 * I, H, self.w[0], self.w[1], sfmt)
            moe.moe_quantize_weight_fp8_fmt(w2, E, H, I, self.w[2], self.w[3], sfmt)
        else:
            self.w = [w13, w2]
        torch.cuda.synchronize()
        self.ws_bytes = moe.moe_workspace_size(self.d, self.dt)
        # the host-buffer entry point keeps its x and out copies after the workspace
        io_al = (cfg.T * H * 2 + 255) // 256 * 256
        self.ws = torch.zeros(self.ws_bytes + 2 * io_al, dtype=torch.uint8, device="cuda")
        self.out = torch.empty(cfg.T, H, dtype=torch.bfloat16, device="cuda")

    @staticmethod
    def bf(a):
        import torch
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    def step(self, xin=None, out=None, ws=None, stream=None):
        moe, cfg, w = self.moe, self.cfg, self.w
        xin = self.x if xin is None else xin
        out = self.out if out is None else out
        ws = self.ws if ws is None else ws
        kw = {} if stream is None else {"stream": stream}
        if cfg.fp4:
            moe.moe_forward_fp4(xin, self.wr, self.bias, *w, self.d, moe.MOE_EPILOGUE_SWIGLU, out,
                                ws, self.ws_bytes, **kw)
        elif cfg.fp8 and cfg.ue8m0:
            moe.moe_forward_fp8_ue8m0(xin, self.wr, self.bias, *w, self.d, moe.MOE_EPILOGUE_SWIGLU,
                                      out, ws, self.ws_bytes, **kw)
        elif cfg.fp8:
            moe.moe_forward_fp8(xin, self.wr, self.bias, *w, self.d, out, ws, self.ws_bytes, **kw)
        else:
            moe.moe_forward(xin, self.wr, self.bias, *w, self.d, out, ws, self.ws_bytes, **kw)

    def offsets(self) -> np.ndarray:
        lay = self.moe.moe_workspace_layout(self.d)
        return self.ws[lay.offsets:lay.offsets + 4 * (self.cfg.E + 1)].cpu().numpy().view(np.int32)


def kernel_name(cfg, decode: bool) -> str:
    if cfg.fp4:
        return "gemm_mx_kernel<SwiGLU, e2m1 B> (block-scaled FP4 GEMM1 + SwiGLU + h quantisation)"
    if cfg.ue8m0:
        return "gemm_mx_kernel<SwiGLU> (block-scaled FP8 GEMM1 + SwiGLU + h quantisation)"
    if cfg.fp8:
        return "gemm_rows_fp8_kernel<SwiGLU> (FP8 GEMM1 + SwiGLU + h quantisation)"
    if decode:
        return "gemm_swap_kernel<SwiGLU> (GEMM1, small-M)"
    return "gemm_rows_kernel<SwiGLU,256> (GEMM1 + SwiGLU on the permuted rows)"


def rooflines(cfg, offsets, ms_per_step: float, stage_ms, region_ms: float, peaks: dict,
              peak_src: str, e4m3_tflops=None):
    """The dominant kernel (GEMM-1) and the whole layer against the measured roofs."""
    flops = 6.0 * cfg.T * cfg.k * cfg.H * cfg.I
    quant = cfg.fp8 or cfg.fp4
    # bytes per expert weight: e2m1 + one e8m0 byte per 32; e4m3 (+ fp32 block scales); bf16
    bpw = (0.5 + 1.0 / 32) if cfg.fp4 else (1.0 + 4.0 / (128 * 128)) if cfg.fp8 else 2.0
    wbytes, n_exp = touched_weight_bytes(cfg, offsets, bpw)
    layer_bytes = wbytes + 2 * cfg.T * cfg.H * 2 + cfg.H * cfg.E * 2
    gemm1_ms = float(stage_ms[2])
    decode = cfg.T * cfg.k <= 64 * cfg.E and cfg.T <= 64
    ratio = 2.0 if quant else 1.0
    tpk, which = tensor_peak(peaks, ratio, region_ms)
    if decode:
        g1_bytes = n_exp * 2 * cfg.H * cfg.I * bpw
        ach = g1_bytes / (gemm1_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": kernel_traffic(cfg.name, "gemm1"),
                "kernel": kernel_name(cfg, True), "algorithmic_bytes_per_launch": g1_bytes,
                "peak_source": f"{peak_src} HBM copy", "frac_of_8tbs": ach / 8000.0}
    else:
        g1_flops = 4.0 * cfg.T * cfg.k * cfg.H * cfg.I
        ach = g1_flops / (gemm1_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tpk, "unit": "TFLOP/s",
                "frac": ach / tpk, "traffic": kernel_traffic(cfg.name, "gemm1"),
                "kernel": kernel_name(cfg, False), "algorithmic_flops_per_launch": g1_flops,
                "peak_source": f"{peak_src} bf16 {which} x {ratio:g} (timed region "
                               f"{region_ms:.0f} ms)"}
        if "bf16_tflops_sustained" in peaks:
            roof["frac_of_sustained"] = ach / (ratio * peaks["bf16_tflops_sustained"])
        if quant and e4m3_tflops:
            roof["frac_of_cublas_e4m3"] = ach / e4m3_tflops
    s = ms_per_step / 1e3
    roof_ms = max(flops / (tpk * 1e12), layer_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    layer = {"tflops": flops / s / 1e12, "tflops_frac": flops / s / 1e12 / tpk,
             "gbs": layer_bytes / s / 1e9, "gbs_frac": layer_bytes / s / 1e9 / peaks["hbm_gbs"],
             "roofline_ms": roof_ms, "roofline_frac": roof_ms / ms_per_step,
             "bound": "tensor" if flops / (tpk * 1e12) >= layer_bytes / (peaks["hbm_gbs"] * 1e9)
             else "hbm", "touched_experts": n_exp,
             "tensor_peak": f"{tpk:.1f} TFLOP/s ({which})"}
    if quant and e4m3_tflops:
        layer["tflops_frac_of_cublas_e4m3"] = flops / s / 1e12 / e4m3_tflops
    return roof, layer, wbytes


def time_steps(torch, moe, w: Workload, steps: int, warmup: int, barrier, clocks=None):
    """After the warm-up, `steps` forwards with per-stage events for the breakdown, then
    the timed region: `steps` forwards and nothing else, between a barrier and a
    synchronise. The breakdown runs first so that both passes see the GPU in the same
    steady state (clock under the power cap). Returns (ms of the timed steps, mean stage
    ms [5], launches, clocks)."""
    stream = torch.cuda.current_stream()
    for _ in range(max(3, warmup)):
        w.step()
    torch.cuda.synchronize()
    status = moe.moe_get_device_status(w.ws)
    if status != 0:
        raise SystemExit(f"device status {status} after warm-up ({w.cfg.name})")
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    for i in range(steps):
        moe.moe_set_stage_events(stage_ev[i])
        w.step()
    moe.moe_set_stage_events(None)
    torch.cuda.synchronize()
    stages = np.array([[ev[j].elapsed_time(ev[j + 1]) for j in range(5)] for ev in stage_ev])
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.start()
    barrier()
    torch.cuda.synchronize()
    n0 = moe.moe_launch_count()
    t0.record(stream)
    for _ in range(steps):
        w.step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = moe.moe_launch_count() - n0
    clk = clocks.stop() if clocks is not None else None
    return t0.elapsed_time(t1), stages.mean(0), launches, clk


def time_graph(torch, w: Workload, steps: int, barrier, dist):
    """The same forward replayed from a CUDA graph (launch overhead removed)."""
    stream = torch.cuda.current_stream()
    try:
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            w.step()  # warm the capture stream
            cs.synchronize()
            with torch.cuda.graph(g, stream=cs):
                w.step()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(steps):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        gms = max_over_ranks(g0.elapsed_time(g1), dist, "cuda") / steps
        del g
        return gms
    except Exception as exc:  # reported, not fatal: the eager number stands
        return str(exc)[:200]


def time_e2e(torch, moe, w: Workload, steps: int, barrier, dist):
    """End to end: pinned host tokens in, pinned host result out, every step. Two streams
    with a workspace each: step i+1's host->device copy runs on the copy engine while step
    i computes, as a serving loop would overlap them. bf16 goes through the C ABI's
    host-buffer entry point; the quantised layers copy with torch around their forward."""
    cfg = w.cfg
    stream = torch.cuda.current_stream()
    x_host = torch.from_numpy(np.ascontiguousarray(w.L["x"]).view(np.int16)).pin_memory()
    streams = [stream, torch.cuda.Stream()]
    wss = [w.ws, torch.zeros_like(w.ws)]
    outs_host = [torch.empty(cfg.T * cfg.H, dtype=torch.int16).pin_memory() for _ in range(2)]
    outs_dev = [w.out, torch.empty_like(w.out)]
    xs_dev = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    def e2e_step(i):
        j = i & 1
        with torch.cuda.stream(streams[j]):
            if w.quant:
                xs_dev[j].view(torch.int16).copy_(x_host.view(cfg.T, cfg.H), non_blocking=True)
                w.step(xs_dev[j], outs_dev[j], wss[j], stream=streams[j])
                outs_host[j].copy_(outs_dev[j].view(torch.int16).view(-1), non_blocking=True)
            else:
                moe.moe_forward_hostio(x_host, w.wr, w.bias, w.w[0], w.w[1], w.d, outs_host[j],
                                       wss[j], stream=streams[j])

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    streams[1].wait_stream(stream)
    for i in range(steps):
        e2e_step(i)
    stream.wait_stream(streams[1])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ems = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
    return ems / steps


def dtype_name(cfg) -> str:
    return ("e4m3 x e2m1 -> fp32 (experts), bf16 router" if cfg.fp4 else
            "e4m3 x e4m3 -> fp32 (experts), bf16 router" if cfg.fp8 else "bf16 x bf16 -> fp32")


def gpu_arm(args, cfg, extra_cfgs):
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

    peaks, peak_src = load_peaks()
    quant_any = any(c.fp8 or c.fp4 for c in [cfg, *extra_cfgs])
    e4m3 = cublas_peaks(torch)["e4m3_tflops"] if quant_any and rank == 0 else None
    wcache: dict = {}

    # ---- the headline workload: timed steps, graph replay, end to end ----
    w = Workload(cfg, rank, wcache)
    clocks = Clocks(torch.cuda.current_device()) if rank == 0 else None
    ms, stage_ms, launches, clk = time_steps(torch, moe, w, args.steps, args.warmup, barrier,
                                             clocks)
    region_ms = max_over_ranks(ms, dist, "cuda")
    ms_per_step = region_ms / args.steps
    value = whole_job_tokens_per_s(cfg.T, world, ms_per_step)
    offsets = w.offsets()
    gms = time_graph(torch, w, args.steps, barrier, dist)
    ems = time_e2e(torch, moe, w, args.steps, barrier, dist)
    io_bytes = cfg.T * cfg.H * 2

    res = None
    if rank == 0:
        roof, layer, wbytes = rooflines(cfg, offsets, ms_per_step, stage_ms, ms, peaks, peak_src,
                                        e4m3)
        counts = np.diff(offsets)
        res = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_name(cfg),
            "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights)",
            "config": {"workload": cfg.desc, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                       "k": cfg.k, "parallelism": f"token-parallel replicas x{world}",
                       "l2": f"inputs larger than L2: {wbytes / 1e9:.2f} GB of expert weights "
                             "read per step, no flush",
                       "expert_rows": {"min": int(counts.min()), "max": int(counts.max()),
                                       "empty": int(np.sum(counts == 0))}},
            "roofline": roof, "layer": layer,
            "stages_us": {n: round(float(v) * 1e3, 2) for n, v in
                          zip(["route", "permute", "gemm1", "gemm2", "combine"], stage_ms)},
            "e2e": {"value": whole_job_tokens_per_s(cfg.T, world, ems), "unit": "tokens/s",
                    "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes},
            "graph": ({"ms_per_step": gms, "value": whole_job_tokens_per_s(cfg.T, world, gms),
                       "unit": "tokens/s"} if isinstance(gms, float) else {"error": gms}),
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        if e4m3:
            res["cublas_e4m3_tflops"] = e4m3

    # ---- the other full-size workloads, on the same line ----
    others = {}
    for c in extra_cfgs:
        del w
        torch.cuda.empty_cache()
        w = Workload(c, rank, wcache)
        ms_c, st_c, _, _ = time_steps(torch, moe, w, args.steps, args.warmup, barrier)
        reg_c = max_over_ranks(ms_c, dist, "cuda")
        mps = reg_c / args.steps
        off_c = w.offsets()
        decode = c.T <= 64
        g_c = time_graph(torch, w, args.steps, barrier, dist) if decode else None
        if rank == 0:
            roof_c, layer_c, _ = rooflines(c, off_c, mps, st_c, ms_c, peaks, peak_src, e4m3)
            others[c.name] = {
                "workload": c.desc, "dtype": dtype_name(c), "ms_per_step": mps,
                "value": whole_job_tokens_per_s(c.T, world, mps), "unit": "tokens/s",
                "roofline": roof_c, "layer": layer_c,
                "stages_us": {n: round(float(v) * 1e3, 2) for n, v in
                              zip(["route", "permute", "gemm1", "gemm2", "combine"], st_c)},
            }
            if isinstance(g_c, float):
                others[c.name]["graph"] = {"ms_per_step": g_c, "value":
                                           whole_job_tokens_per_s(c.T, world, g_c)}
    if rank == 0 and others:
        res["other_workloads"] = others
    del w
    wcache.clear()

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    if world == 1 and not args.no_cpu_baseline:
        import oracle

        L = mi.make_layer(cfg)
        v, n, t = oracle_tokens_per_s(cfg, L, float(os.environ.get("MOE_CPU_BUDGET_S", "20")))
        res["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": oracle.threads(),
                               "cpu": cpu_model(), "kind": "oracle",
                               "sample": f"{n} of {cfg.T} tokens (seeded subset), whole layer "
                                         f"per token, {t:.1f} s"}
    print(json.dumps(res), flush=True)


def peaks_arm():
    """Measured dense cuBLAS peaks of this GPU (bf16 and e4m3 8192^3, best of 10) and a
    2 GiB copy, as one JSON line."""
    import torch

    res = cublas_peaks(torch)
    res["device"] = torch.cuda.get_device_name()
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(mi.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="time only the headline workload (no other full-size workloads)")
    ap.add_argument("--peaks", action="store_true",
                    help="print this GPU's dense cuBLAS bf16 / e4m3 peaks and copy bandwidth")
    ap.add_argument("--shape", default="",
                    help="override dims of the config, e.g. T=2048,E=64 (for a smaller profiling "
                         "case; the workload name then says so)")
    args = ap.parse_args()
    if args.peaks:
        return peaks_arm()
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
        extras = [] if (args.no_extras or args.shape) else \
            [mi.CONFIGS[n] for n in EXTRA_CONFIGS if n != cfg.name]
        gpu_arm(args, cfg, extras)


if __name__ == "__main__":
    main()
