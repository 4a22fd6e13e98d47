#!/usr/bin/env python
"""Benchmark of the routed MoE FFN layer on B200: one JSON line on rank 0.

A step is one moe_forward call (route, permute, quantise, gate|up GEMM, down GEMM, combine)
over one batch of seeded synthetic inputs already resident in HBM.  The default workload is
the Qwen3.5-397B-shaped decode step (T=512, H=4096, 512 experts x 1024, top-10 + shared
1024, FP8 512-sub-channel).  Multi-GPU runs are independent replicas (one process per GPU,
each with its own batch; nothing is exchanged on the data path), so scaling is weak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; % HBM roofline (decode) / % FP8 tensor peak (prefill)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of the gate|up GEMM per algorithmic byte: one ncu capture of
# dram__bytes_read.sum + dram__bytes_write.sum for the gate|up launch of the decode-shaped
# profiling workload (moe_synth "profile-decode": 552,494,080 + 3,675,392 bytes against
# 549,519,360 algorithmic), scaled to a decode launch by its algorithmic bytes.  Stored with
# the hash of the kernel source it was taken on; the figure is null once that source changes.
TRAFFIC = {"decode": {"kernel": "gemm_gateup", "ratio": (552494080 + 3675392) / 549519360,
                      "src_sha": "58749818c856a0d0"}}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="decode")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target oracle time for cpu_baseline")
    ap.add_argument("--no-per-config", action="store_true", help="time the headline workload only")
    ap.add_argument("--per-config-steps", type=int, default=10)
    ap.add_argument("--per-config-cpu-seconds", type=float, default=3.0)
    return ap.parse_args()


def peaks():
    p = dict(FALLBACK_PEAKS)
    src = "fallback"
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        for k in FALLBACK_PEAKS:
            if k in m:
                p[k] = float(m[k])
        src = "measured"
    return p, src


def src_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def dist_setup(args):
    import torch
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:  # host-only ranks (the multi-process tests): the same plumbing over gloo
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, v):
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(ws, tokens_per_rank_step, steps, max_ms):
    """Whole-job tokens/s of ws independent replicas, each doing `steps` steps of
    `tokens_per_rank_step` tokens, timed as the slowest rank's total device time."""
    return ws * tokens_per_rank_step * steps / (max_ms / 1e3)


class ClockSampler:
    """SM clock and clock-event reasons read through NVML (read-only) every ~2 ms by a background
    thread while the timed region runs; falls back to nothing if NVML is unavailable."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, cuda_index):
        import threading
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.stop_ev = threading.Event()
        self.thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(cuda_index)
            try:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        masks = [(n, getattr(nv, a, 0)) for n, a in self.REASONS]
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for n, m in masks:
                    if m and (r & m):
                        self.reasons.add(n)
            except Exception:
                pass
            self.stop_ev.wait(0.002)

    def start(self):
        if self.nv is None:
            return
        import threading
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_ev.set()
        self.thread.join()
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def algorithmic(cfg, counts):
    """Algorithmic bytes and flops of one layer call (experts with >= 1 token only)."""
    H, I, Is, T, k = cfg["H"], cfg["I"], cfg["Is"], cfg["T"], cfg["k"]
    touched = int((counts > 0).sum())
    if cfg["wfmt"] == "fp8":
        nbH, nbI, nbIs = -(-H // 512), -(-I // 512), -(-Is // 512)
        gu = touched * 2 * (I * H + I * nbH * 4) + (2 * (Is * H + Is * nbH * 4) if Is else 0)
        dn = touched * (H * I + H * nbI * 4) + ((H * Is + H * nbIs * 4) if Is else 0)
    else:
        # 4-bit weights: packed nibbles plus the scales (int4: bf16 per 128; MXFP4: one byte per
        # 32; NVFP4: one byte per 16 and an fp32 tensor scale per matrix)
        sb = {"int4": lambda K: (K // 128) * 2, "mxfp4": lambda K: K // 32, "nvfp4": lambda K: K // 16}[cfg["wfmt"]]
        ts = 4 if cfg["wfmt"] == "nvfp4" else 0
        gu = touched * 2 * (I * H // 2 + I * sb(H) + ts) + (2 * (Is * H // 2 + Is * sb(H) + ts) if Is else 0)
        dn = touched * (H * I // 2 + H * sb(I) + ts) + ((H * Is // 2 + H * sb(Is) + ts) if Is else 0)
    act = T * H * 2 + T * H * 2 + T * cfg["E"] * 4  # x in, out, logits
    f_gu = 2 * 2 * H * I * T * k + (2 * 2 * H * Is * T if Is else 0)
    f_dn = 2 * H * I * T * k + (2 * H * Is * T if Is else 0)
    return {"gemm_gateup": gu, "gemm_down": dn, "layer": gu + dn + act, "touched": touched,
            "flops": f_gu + f_dn, "flops_gemm_gateup": f_gu, "flops_gemm_down": f_dn}


def make_host_layer(name, device):
    import moe_synth
    layer = moe_synth.make_layer(name, device=device)
    return moe_synth.to_numpy(layer), layer


def time_oracle(Lnp, n_tokens, seed=7):
    import numpy as np
    import oracle
    T = Lnp["dims"]["T"]
    rng = np.random.default_rng(seed)
    sel = np.sort(rng.choice(T, min(n_tokens, T), replace=False)).astype(np.int32)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.layer(Lnp, sel, nthreads=threads)
    return time.perf_counter() - t0, len(sel), threads


def cpu_baseline(Lnp, target_s):
    """The oracle, as it stands, on a bounded sample of the workload's tokens."""
    dt, n, thr = time_oracle(Lnp, 4)
    per_tok = dt / n
    n2 = max(4, min(Lnp["dims"]["T"], int(target_s / max(per_tok, 1e-6))))
    dt, n, thr = time_oracle(Lnp, n2, seed=8)
    return {"value": n / dt, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{n} of {Lnp['dims']['T']} tokens (random, seeded) through the fp64 oracle, {dt:.1f} s"}


def run_reference(args, ws, rank, cfg_name):
    import moe_synth
    import oracle  # noqa: F401  (the reference arm times the oracle)
    import torch
    if rank != 0:
        return
    cfg = {**moe_synth.CONFIGS, **moe_synth.PROFILE_CONFIGS}[cfg_name]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    Lnp, _ = make_host_layer(cfg_name, dev)
    if dev == "cuda":
        torch.cuda.empty_cache()
    # size a step to ~2 s of oracle work
    dt, n, thr = time_oracle(Lnp, 2)
    per_tok = dt / n
    S = max(2, min(cfg["T"], int(2.0 / max(per_tok, 1e-6))))
    for w in range(args.warmup):
        time_oracle(Lnp, S, seed=100 + w)
    total, toks = 0.0, 0
    for s in range(args.steps):
        dt, n, thr = time_oracle(Lnp, S, seed=1000 + s)
        total += dt
        toks += n
    v = toks / total
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": cfg["workload"], "T": cfg["T"], "H": cfg["H"], "E": cfg["E"], "I": cfg["I"],
                       "k": cfg["k"], "I_shared": cfg["Is"], "wfmt": cfg["wfmt"],
                       "sample_tokens_per_step": S},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": f"{S} random tokens of {cfg['T']} per step through the fp64 oracle"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def fp8_peak_tflops(dev):
    """Dense FP8 (e4m3) tensor throughput of this GPU as cuBLAS reaches it: the best of 10
    8192^3 torch._scaled_mm calls (e4m3 x e4m3 -> bf16).  A measured denominator for the FP8
    tensor fraction; None if the call is unavailable."""
    import torch
    try:
        n = 8192
        a = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = 1e9
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2 * n ** 3 / (best / 1e3) / 1e12
    except Exception:
        return None


def measure_layer(cfg_name, steps, warmup, ws, rank, local, pk, pk_src, fp8_tf, flush, timing_barrier=True):
    """Time `steps` moe_forward calls of one synthetic layer (L2 flushed before each, CUDA
    events on the launching stream), then the same steps with the library's stage events for
    the per-kernel times.  Returns the layer, its MoELayer and the measurement dict."""
    import torch

    import moe_synth
    import mixture_experts_ffn_13_b200 as moe

    cfg = {**moe_synth.CONFIGS, **moe_synth.PROFILE_CONFIGS}[cfg_name]
    dev = torch.device("cuda", torch.cuda.current_device())
    layer = moe_synth.make_layer(cfg_name, device=dev)
    m = moe.MoELayer(layer)
    x, logits = layer["x"], layer["logits"]
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        m(x, logits, out=out)
    torch.cuda.synchronize()
    rc = moe.moe_get_status(m.plan)
    if rc != 0:
        raise RuntimeError(f"{cfg_name}: device status after warm-up: {moe.moe_strerror(rc)}")

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    launches = 0
    if timing_barrier:
        barrier(ws)
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        m(x, logits, out=out)
        ev[i][1].record(stream)
        launches += moe.moe_launch_count(m.plan)
    torch.cuda.synchronize()
    if timing_barrier:
        barrier(ws)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    clk = clocks.stop() if clocks else None
    rc = moe.moe_get_status(m.plan)
    if rc != 0:
        raise RuntimeError(f"{cfg_name}: device status after timing: {moe.moe_strerror(rc)}")
    total_ms = max_over_ranks(ws, sum(step_ms)) if timing_barrier else sum(step_ms)

    # the same steps with the library's stage events on the same stream: per-kernel device
    # times for the roofline of the dominant kernel (events between kernels keep the next
    # kernel from starting early, so this pass is not the one the throughput comes from)
    moe.moe_profile_enable(m.plan, True)
    stage_ms = {s_: 0.0 for s_ in moe.STAGES}
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        m(x, logits, out=out)
        ev[i][1].record(stream)
        for kname, v in moe.moe_profile_read(m.plan).items():
            stage_ms[kname] += v
    torch.cuda.synchronize()
    prof_ms = sum(a.elapsed_time(b) for a, b in ev)
    moe.moe_profile_enable(m.plan, False)

    r = m.route(logits)
    counts = r["counts"].cpu().numpy()
    alg = algorithmic(cfg, counts)
    T = cfg["T"]
    ms_step = total_ms / steps
    mean_stage = {k: v / steps for k, v in stage_ms.items()}
    dom = max(("gemm_gateup", "gemm_down"), key=lambda s_: mean_stage[s_])
    dom_ms = mean_stage[dom]
    if moe.moe_launch_count(m.plan) == 1:
        # the single-kernel small-batch path: one launch does the whole layer, so the dominant
        # kernel is that launch and its bytes are the layer's
        dom, dom_ms = "small_batch", sum(mean_stage.values())
        alg = dict(alg, small_batch=alg["layer"], flops_small_batch=alg["flops"])
    achieved = alg[dom] / (dom_ms / 1e3) / 1e9
    layer_gbs = alg["layer"] / (ms_step / 1e3) / 1e9
    if cfg["wfmt"] == "fp8":
        if fp8_tf:
            tpk, tpk_src = fp8_tf, "cuBLAS e4m3 8192^3 (torch._scaled_mm), measured in this run"
        else:
            tpk, tpk_src = 2 * pk["bf16_tflops"], f"2 x {pk_src} bf16 burst (FP8 = 2x bf16 nominal ratio)"
    else:
        tpk, tpk_src = pk["bf16_tflops"], f"{pk_src} bf16 burst"
    t_hbm = alg["layer"] / (pk["hbm_gbs"] * 1e9) * 1e3
    t_tc = alg["flops"] / (tpk * 1e12) * 1e3
    small = sum(v for k, v in mean_stage.items() if not k.startswith("gemm_"))
    res = {
        "workload": cfg["workload"], "value": replica_throughput(ws, T, steps, total_ms), "unit": UNIT,
        "ms_per_step": ms_step, "steps": steps, "warmup": warmup,
        "experts_touched": alg["touched"], "max_tokens_per_expert": int(counts.max()),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "algorithmic_bytes": alg[dom],
                     "peak_source": pk_src, "layer_achieved_gbs": layer_gbs, "layer_frac": layer_gbs / pk["hbm_gbs"]},
        # tensor-core view of the same run: FP8 MMAs against the FP8 peak named in peak_source,
        # the 4-bit path's bf16 MMAs against the bf16 peak
        "tensor": {"kernel": dom, "achieved": alg["flops_" + dom] / (dom_ms / 1e3) / 1e12,
                   "peak": tpk, "unit": "TFLOP/s",
                   "frac": alg["flops_" + dom] / (dom_ms / 1e3) / 1e12 / tpk,
                   "layer_achieved": alg["flops"] / (ms_step / 1e3) / 1e12,
                   "layer_frac": alg["flops"] / (ms_step / 1e3) / 1e12 / tpk, "peak_source": tpk_src},
        # the layer's binding roofline: the slower of streaming its algorithmic bytes at the
        # measured HBM bandwidth and running its FLOPs at the tensor peak above
        "binding_roofline": {"t_hbm_ms": t_hbm, "t_tensor_ms": t_tc, "bound": "hbm" if t_hbm >= t_tc else "tensor",
                             "frac": max(t_hbm, t_tc) / ms_step},
        "stages_ms": mean_stage,
        "small_kernels_share": small / max(sum(mean_stage.values()), 1e-9),
        "ms_per_step_with_stage_events": prof_ms / steps,
        "gpu_launches": launches,
        "clocks": clk,
    }
    return layer, m, res, cfg


PER_CONFIG = ("tiny", "prefill", "skewed", "int4", "mxfp4", "nvfp4")


def run_ours(args, ws, rank, local, cfg_name):
    import torch

    import moe_synth
    import mixture_experts_ffn_13_b200 as moe
    from mixture_experts_ffn_13_b200 import build as moe_build

    moe_build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    pk, pk_src = peaks()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    fp8_tf = fp8_peak_tflops(dev)
    torch.cuda.empty_cache()
    layer, m, res, cfg = measure_layer(cfg_name, args.steps, args.warmup, ws, rank, local, pk, pk_src, fp8_tf, flush)
    x, logits = layer["x"], layer["logits"]
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()

    # end to end through the public API with host buffers: every step copies its x and logits
    # from pinned host memory and reads its output back.  Copies run on their own streams,
    # double-buffered, so step i+1's upload and step i-1's read-back overlap step i's layer
    # (the copy engines and the SMs work at once); events order each buffer's reuse.  No L2
    # flush here: every step streams the expert weights (far larger than L2) from HBM.
    xh = x.cpu().pin_memory()
    lh = logits.cpu().pin_memory()
    oh = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    ld = [torch.empty_like(logits) for _ in range(2)]
    od = [torch.empty_like(out) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        s_in.wait_event(t0)
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev_done[b])   # the layer two steps back has read xd[b], ld[b]
            with torch.cuda.stream(s_in):
                xd[b].copy_(xh, non_blocking=True)
                ld[b].copy_(lh, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # od[b] has been read back
            m(xd[b], ld[b], out=od[b], stream=stream)
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                oh[b].copy_(od[b], non_blocking=True)
            ev_out[b].record(s_out)
        for b in range(min(n, 2)):
            stream.wait_event(ev_out[b])
        t1.record(stream)
        return t0, t1

    e2e_run(max(2, args.warmup))
    torch.cuda.synchronize()
    barrier(ws)
    t0, t1 = e2e_run(args.steps)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = max_over_ranks(ws, t0.elapsed_time(t1))
    e2e_value = replica_throughput(ws, cfg["T"], args.steps, e2e_ms)

    dom = res["roofline"]["kernel"]
    tr = TRAFFIC.get(cfg_name)
    traffic = None
    if tr and tr["kernel"] == dom and tr["src_sha"] == src_sha(
            os.path.join(ROOT, "mixture_experts_ffn_13_b200", "csrc", "gemm_fp8.cu")):
        traffic = tr["ratio"] * res["roofline"]["algorithmic_bytes"]
    roof = dict(res["roofline"], traffic=traffic)
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8_e4m3" if cfg["wfmt"] == "fp8" else "bf16", "data": "synthetic",
        "config": {"workload": cfg["workload"], "T": cfg["T"], "H": cfg["H"], "E": cfg["E"], "I": cfg["I"],
                   "k": cfg["k"], "I_shared": cfg["Is"], "wfmt": cfg["wfmt"], "seed": cfg["seed"],
                   "parallelism": f"replicas x{ws}", "l2": "flushed (256 MiB write) before every timed step",
                   "experts_touched": res["experts_touched"], "max_tokens_per_expert": res["max_tokens_per_expert"]},
        "roofline": roof,
        "tensor": res["tensor"],
        "binding_roofline": res["binding_roofline"],
        "stages_ms": res["stages_ms"],
        "small_kernels_share": res["small_kernels_share"],
        "ms_per_step_with_stage_events": res["ms_per_step_with_stage_events"],
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": x.numel() * 2 + logits.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 2,
                "copies": "pinned host buffers, H2D and D2H on their own streams, double-buffered "
                          "across steps (overlapping the layer)",
                "l2": "not flushed: every step streams the expert weights (far larger than L2)"},
        "gpu_launches": res["gpu_launches"],
        "clocks": res["clocks"],
        "fp8_peak_tflops_measured": fp8_tf,
    }
    del xd, ld, od, xh, lh, oh
    # small batches of the same layer (the first T tokens): device time per call against each
    # T's own HBM roofline (the touched experts' weights and scales plus x, logits and out);
    # T <= 16 runs the single-kernel small-batch path
    if ws == 1 and not args.no_per_config and cfg["wfmt"] == "fp8":
        sweep = []
        for Tq in (1, 2, 4, 8, 16):
            xs, ls = x[:Tq].contiguous(), logits[:Tq].contiguous()
            os_ = torch.empty_like(xs)
            for _ in range(3):
                m(xs, ls, out=os_)
            torch.cuda.synchronize()
            times = []
            for _ in range(20):
                flush.zero_()
                # hold the stream (~100 us) until the call is enqueued: at these sizes the host's
                # launch latency would otherwise land between the events
                torch.cuda._sleep(200000)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                m(xs, ls, out=os_)
                e1.record(stream)
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            launches = moe.moe_launch_count(m.plan)
            cnt = m.route(ls)["counts"].cpu().numpy()
            alg = algorithmic(dict(cfg, T=Tq), cnt)
            ms = statistics.median(times)
            t_roof = alg["layer"] / (pk["hbm_gbs"] * 1e9) * 1e3
            sweep.append({"T": Tq, "ms": ms, "tokens_per_s": Tq / (ms / 1e3), "hbm_roofline_ms": t_roof,
                          "frac": t_roof / ms, "kernels": launches})
        rc = moe.moe_get_status(m.plan)
        if rc != 0:
            raise RuntimeError(f"device status after the small-batch sweep: {moe.moe_strerror(rc)}")
        line["small_batch_sweep"] = sweep
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        del layer, m
        torch.cuda.empty_cache()
        Lnp, _ = make_host_layer(cfg_name, dev)
        line["cpu_baseline"] = cpu_baseline(Lnp, args.cpu_seconds)
        del Lnp
    else:
        del layer, m
    # every other workload of the build, measured the same way (one GPU only: the scaling runs
    # time the headline workload alone); each with a short oracle sample on the host cores
    if ws == 1 and not args.no_per_config:
        per = {}
        for name in PER_CONFIG:
            if name == cfg_name:
                continue
            torch.cuda.empty_cache()
            lyr, mm, r_, _ = measure_layer(name, args.per_config_steps, max(3, args.warmup), ws, rank, local, pk,
                                           pk_src, fp8_tf, flush, timing_barrier=False)
            del lyr, mm
            torch.cuda.empty_cache()
            if not args.no_cpu_baseline:
                Lnp, _ = make_host_layer(name, dev)
                r_["cpu_baseline"] = cpu_baseline(Lnp, args.per_config_cpu_seconds)
                del Lnp
            per[name] = r_
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    ws, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank, args.config)
        else:
            run_ours(args, ws, rank, local, args.config)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
