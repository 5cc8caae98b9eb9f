#!/usr/bin/env python
"""Benchmark of the expert-parallel MoE-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--mxfp8]

One step = one forward of the whole layer (route -> preprocess -> dispatch ->
grouped expert FFN -> combine) over one batch of T synthetic tokens, inputs
resident in HBM.  L2 is flushed before every timed step (a 256 MiB write, then a read
of the same buffer, so that the write-back of the flush's dirty lines is not charged
to the step), and
each step is timed with CUDA events on the launching stream; the max over ranks
is taken.  With N > 1 (torchrun) every rank runs an independent replica on its
own batch (replicas only: the layer needs no collective on one node here), so
scaling is weak and value = tokens of all ranks / max time.

`--mxfp8` runs the routed experts in MXFP8 (E4M3 with one E8M0 scale per 32; the
opt-in path, MoELayer(mxfp8=True)); routing, shared experts and combine are unchanged.

`--impl reference` times the CPU oracle (float64 numpy, the definition the CUDA
path is checked against) on host cores over a bounded token sample per step.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "deepseek_v3"
METRIC = "MoE-layer fwd tokens/s on 1 B200; grouped-FFN % BF16 peak; permute/combine GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=W.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample", type=int, default=0,
                    help="tokens per CPU-oracle sample (0 = sized for ~12 s of host time)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload's shapes with this many tokens instead of its T "
                         "(serving-sized batches; the line's workload name gets a _t<N> suffix)")
    ap.add_argument("--mxfp8", action="store_true",
                    help="routed experts in MXFP8 (the opt-in path); the workload name gets _mxfp8")
    ap.add_argument("--experts", type=int, default=0,
                    help="run the workload with this many routed experts (a multiple of its "
                         "ep_size; reduced cases for profiling; the name gets an _e<N> suffix)")
    return ap.parse_args()


def pick_workload(args):
    wl = W.get(args.workload)
    if args.tokens > 0:
        wl = wl.with_(T=args.tokens, name=f"{wl.name}_t{args.tokens}")
    if args.experts > 0:
        wl = wl.with_(E=args.experts, name=f"{wl.name}_e{args.experts}")
    return wl


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup(backend="nccl"):
    """Join the process group torchrun describes in the environment (N > 1)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, ws, device="cuda"):
    """Max of a per-rank scalar over all ranks (the slowest rank sets the time)."""
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(tokens_per_rank, ws, steps, total_ms_max):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * ws * steps / (total_ms_max / 1e3)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, index, period=0.002):
        self.samples, self.reasons, self.period = [], 0, period
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"],
                    "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def stage_bytes(wl):
    sx = 4 if wl.x_dtype == "f32" else 2
    T, D, R = wl.T, wl.D, wl.R
    dispatch = T * D * sx + R * D * 2 + R * 4
    combine = R * D * 2 + 2 * T * D * sx + (T * D * 2 if wl.n_shared else 0) + R * 8
    return dispatch, combine


def route_launches(wl):
    """Kernels of moe_route without returned logits: the fused few-expert router, or
    for bf16 x the W_r split + tensor-core filter GEMM + exact refine, else logits + top-k."""
    few = wl.E <= 32 and wl.E * wl.D * 4 <= 200 << 10
    if few:
        return 1
    return 3 if wl.x_dtype == "bf16" and wl.renormalize else 2


def ffn_launches(wl):
    """Kernels of moe_expert_ffn: one persistent launch when every GEMM has 256-wide
    tiles (D and, for GELU, F multiples of 256), else one per GEMM."""
    up256 = wl.act == "swiglu" or wl.F % 256 == 0
    if up256 and wl.D % 256 == 0:
        return 1
    return 4 if wl.n_shared else 2


class HostOracleInputs:
    """The oracle's view of a workload's inputs: x and the router on the host in
    float64, expert weights fetched one expert at a time (bf16 -> float64) from
    wherever the drawn tensors live, so a 256-expert layer never needs its ~90 GB of
    float64 weights at once.  The fetch is part of the oracle's work as timed."""

    def __init__(self, wl, inp):
        f = lambda t: None if t is None else t.detach().cpu().to(torch.float64).numpy()
        self.wl = wl
        self.x = f(inp["x"])
        self.w_router = inp["w_router"].cpu().numpy()
        self.bias = None if inp["bias"] is None else inp["bias"].cpu().numpy()
        self._up = inp["w_gate_up"] if wl.act == "swiglu" else inp["w1"]
        self._down = inp["w_down"]
        self.ws_up, self.ws_down = f(inp["ws_gate_up"]), f(inp["ws_down"])

    def expert(self, e):
        f = lambda t: t.detach().cpu().to(torch.float64).numpy()
        return f(self._up[e]), f(self._down[e])


def cpu_oracle_time(wl, host, n_tok, seed=0):
    """Time the oracle's layer forward on a token sample (weights streamed per expert)."""
    import oracle
    rng = np.random.default_rng(seed)
    # a sample larger than the batch runs the oracle over several random draws of it
    sizes = [wl.T] * (n_tok // wl.T) + ([n_tok % wl.T] if n_tok % wl.T else [])
    t = 0.0
    for n in sizes:
        toks = np.sort(rng.choice(wl.T, size=n, replace=False))
        x = host.x[toks]
        t0 = time.perf_counter()
        oracle.moe_layer(x, host.w_router, host.bias, None, None, host.ws_up, host.ws_down,
                         E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, act=wl.act,
                         renormalize=wl.renormalize, x_is_f32=(wl.x_dtype == "f32"),
                         expert_weights=host.expert)
        t += time.perf_counter() - t0
    return t


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def pick_sample(wl, host, budget_s):
    """Tokens per oracle sample so one sample costs about budget_s on the host: time a
    small probe and scale (tokens are independent; with few tokens per expert the cost
    grows with the experts they touch, about linearly in the tokens), then re-time a
    quarter of that estimate and scale again (the probe carries the per-call costs)."""
    probe = min(2 if wl.E * wl.D * wl.F >= 1 << 30 else 64, wl.T)
    cpu_oracle_time(wl, host, probe, seed=99)            # warm the BLAS threads
    t = cpu_oracle_time(wl, host, probe, seed=98)
    cap = 16 * wl.T
    n = int(max(probe, min(cap, budget_s * probe / max(t, 1e-6))))
    n2 = max(probe, n // 4)
    t2 = cpu_oracle_time(wl, host, n2, seed=97)
    return int(max(probe, min(cap, budget_s * n2 / max(t2, 1e-6))))


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = pick_workload(args)
    # the same seeded draws as the GPU arm (drawn on the GPU where there is one: a
    # 256-expert layer's weights take minutes to draw on the host); the oracle itself
    # runs on the host cores only
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = W.make_inputs(wl, device=dev)
    host = HostOracleInputs(wl, inp)
    n_tok = args.cpu_sample or pick_sample(wl, host, min(10.0, max(0.5, 120.0 / max(1, args.steps))))
    for i in range(args.warmup):
        cpu_oracle_time(wl, host, min(n_tok, 16), seed=i)
    times = [cpu_oracle_time(wl, host, n_tok, seed=100 + i) for i in range(args.steps)]
    total = sum(times)
    value = n_tok * args.steps / total
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "D": wl.D, "E": wl.E, "ep_size": wl.ep_size,
                   "top_k": wl.top_k, "F": wl.F, "n_shared": wl.n_shared, "F_shared": wl.F_shared,
                   "tokens_per_step": n_tok},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_tok} random tokens of the {wl.name} batch per step "
                                   f"(tokens are independent: dropless routing); expert weights "
                                   f"fetched and widened to float64 one expert at a time"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    ws, rank, local = dist_setup()
    torch.cuda.set_device(local)
    import expert_dispatch_fp32_b200 as M

    wl = pick_workload(args)
    peaks, peak_src = load_peaks()
    inp = W.make_inputs(wl, device="cuda")
    if rank > 0:
        inp["x"] = W.make_x(wl, device="cuda", seed=wl.seed + 1000 * rank)
    cpu_host = None
    # (the oracle is the bf16 layer's definition: no CPU baseline for the MXFP8 variant)
    want_cpu = (rank == 0 and ws == 1 and not args.no_cpu_baseline and not args.mxfp8)
    if want_cpu:
        # keeps the drawn weights (bf16, on the device) for the oracle to fetch per expert
        cpu_host = HostOracleInputs(wl, inp)
    up = inp["w_gate_up"] if wl.act == "swiglu" else inp["w1"]
    layer = M.MoELayer(D=wl.D, E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, F=wl.F,
                       w_router=inp["w_router"], w_gate_up=up, w_down=inp["w_down"],
                       expert_bias=inp["bias"], ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"],
                       act=wl.act, renormalize=wl.renormalize, x_dtype=wl.x_dtype, mxfp8=args.mxfp8)
    mx = args.mxfp8
    torch.cuda.synchronize()
    for key in ("w_gate_up", "w1", "w_down", "ws_gate_up", "ws_down"):
        inp.pop(key, None)
    torch.cuda.empty_cache()
    x = inp["x"]
    T = wl.T
    b = layer.allocate(T)
    cfg = layer.config(T)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush_l2():
        # write 256 MiB (more than the 126 MB L2), then read it back: the read evicts the
        # dirty lines (written back here, outside the timed step) and leaves L2 holding
        # clean lines of this buffer only
        flush.zero_()
        flush.view(torch.float32).sum()

    x_bf = x if wl.x_dtype == "bf16" else None

    fused = M.moe_route_dispatch_is_fused(cfg)
    mx_fused_dispatch = mx and not fused and wl.x_dtype == "bf16"

    def expert_ffn():
        if mx:
            M.moe_expert_ffn_mxfp8(cfg, None if mx_fused_dispatch else b["x_perm"], x_bf,
                                   b["expert_offsets"], layer.packed,
                                   layer.packed_mx, b["y_perm"], b["shared_out"], b["workspace"],
                                   b["status"], stream)
        else:
            M.moe_expert_ffn(cfg, b["x_perm"], x_bf, b["expert_offsets"], layer.packed, b["act"],
                             b["y_perm"], b["shared_out"], b["workspace"], b["status"], stream)

    def stages(ev):
        ev[0].record(stream)
        M.moe_route(cfg, x, layer.w_router, layer.expert_bias, None, b["topk_idx"], b["topk_w"],
                    b["workspace"], stream)
        ev[1].record(stream)
        M.moe_preprocess(cfg, b["topk_idx"], b["counts"], b["expert_offsets"], b["rank_splits"],
                         b["rank_offsets"], b["pos"], b["src"], b["workspace"], b["status"], stream)
        ev[2].record(stream)
        if mx_fused_dispatch:
            # MXFP8: the dispatch writes the quantised rows (the layer's forward does the same)
            M.moe_dispatch_mxfp8(cfg, x, b["src"], b["expert_offsets"], b["workspace"], stream)
        else:
            M.moe_dispatch_permute(cfg, x, b["pos"], b["x_perm"], stream)
        ev[3].record(stream)
        expert_ffn()
        ev[4].record(stream)
        M.moe_combine_unpermute(cfg, b["y_perm"], b["pos"], b["topk_w"], x, b["shared_out"],
                                b["out"], stream)
        ev[5].record(stream)

    def stages_fused(ev):
        # the three launches moe_forward runs: router + preprocess + dispatch in one
        ev[0].record(stream)
        M.moe_route_dispatch(cfg, x, layer.w_router, layer.expert_bias, None, b["topk_idx"],
                             b["topk_w"], b["counts"], b["expert_offsets"], b["rank_splits"],
                             b["rank_offsets"], b["pos"], b["src"], b["x_perm"], b["workspace"],
                             b["status"], stream)
        ev[1].record(stream)
        expert_ffn()
        ev[2].record(stream)
        M.moe_combine_unpermute(cfg, b["y_perm"], b["pos"], b["topk_w"], x, b["shared_out"],
                                b["out"], stream)
        ev[3].record(stream)

    def fwd(ev):
        ev[0].record(stream)
        layer.forward(x, stream)
        ev[1].record(stream)

    mk = lambda n=6: [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    # the stage-by-stage step is the layer's forward: check once that both give the same bits
    stages(mk())
    ref_out = b["out"].clone()
    layer.forward(x, stream)
    torch.cuda.synchronize()
    assert torch.equal(ref_out, b["out"]), "stage-by-stage step differs from the layer's forward"
    layer.check_status()

    for _ in range(args.warmup):
        flush_l2()
        fwd(mk(2))
    torch.cuda.synchronize()
    barrier(ws)
    evs = [mk(2) for _ in range(args.steps)]
    torch.cuda.synchronize()
    # timed region: K steps of moe_forward, each after an L2 flush
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush_l2()
            fwd(evs[i])
        torch.cuda.synchronize()
    barrier(ws)
    layer.check_status()
    total_ms = float(sum(e[0].elapsed_time(e[1]) for e in evs))

    # per-stage breakdown, a separate pass with events between the stage calls
    sevs = [mk() for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2()
        stages(sevs[i])
    torch.cuda.synchronize()
    layer.check_status()
    stage_ms = np.zeros(5)
    for ev in sevs:
        stage_ms += [ev[j].elapsed_time(ev[j + 1]) for j in range(5)]
    fused_ms = None
    if fused:
        fevs = [mk(4) for _ in range(args.steps)]
        for i in range(args.steps):
            flush_l2()
            stages_fused(fevs[i])
        torch.cuda.synchronize()
        layer.check_status()
        fused_ms = np.zeros(3)
        for ev in fevs:
            fused_ms += [ev[j].elapsed_time(ev[j + 1]) for j in range(3)]
    total_ms_max = max_over_ranks(total_ms, ws)
    value = replica_value(T, ws, args.steps, total_ms_max)

    # end to end through the C ABI with host buffers: every step uploads its batch from
    # pinned host memory and reads its output back to pinned host memory.  Uploads run on
    # a copy stream and downloads on another, double-buffered, so step i+1's upload and
    # step i-1's download overlap step i's forward; the timed region spans the first
    # upload to the last download (whole-job throughput).
    NBUF = 2
    x_host = [x.cpu().pin_memory() for _ in range(NBUF)]
    out_host = [torch.empty(b["out"].shape, dtype=b["out"].dtype).pin_memory() for _ in range(NBUF)]
    x_dev = [torch.empty_like(x) for _ in range(NBUF)]
    out_dev = [torch.empty_like(b["out"]) for _ in range(NBUF)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(nsteps, t0=None, t1=None):
        up_done = [torch.cuda.Event() for _ in range(nsteps)]
        fw_done = [torch.cuda.Event() for _ in range(nsteps)]
        dn_done = [torch.cuda.Event() for _ in range(nsteps)]
        if t0 is not None:
            t0.record(h2d)
        for i in range(nsteps):
            j = i % NBUF
            with torch.cuda.stream(h2d):
                if i >= NBUF:
                    h2d.wait_event(fw_done[i - NBUF])          # x_dev[j] no longer read
                x_dev[j].copy_(x_host[j], non_blocking=True)
                up_done[i].record(h2d)
            stream.wait_event(up_done[i])
            if i >= NBUF:
                stream.wait_event(dn_done[i - NBUF])           # out_dev[j] already read back
            layer.forward_into(x_dev[j], out_dev[j], stream)      # moe_forward (bf16 path)
            fw_done[i].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(fw_done[i])
                out_host[j].copy_(out_dev[j], non_blocking=True)
                dn_done[i].record(d2h)
        if t1 is not None:
            t1.record(d2h)

    e2e_run(max(args.warmup, NBUF))
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, e0, e1)
    torch.cuda.synchronize()
    barrier(ws)
    layer.check_status()
    assert torch.equal(out_host[(args.steps - 1) % NBUF].to(b["out"].device), ref_out), \
        "end-to-end output differs from the device-resident forward"
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws)
    e2e_value = replica_value(T, ws, args.steps, e2e_ms)
    sx = 4 if wl.x_dtype == "f32" else 2

    # roofline of the dominant kernel: the grouped expert FFN (tcgen05 GEMMs), against the
    # measured bf16 burst peak (a kernel of a few ms, timed alone in the stage pass); the
    # ratio to the seconds-long sustained figure is reported beside it
    ffn_ms = stage_ms[3] / args.steps
    ffn_tflops = wl.ffn_flop() / (ffn_ms / 1e3) / 1e12
    peak_key = "bf16_tflops"
    # MXFP8: dense fp8 runs at twice the bf16 rate (nominal ratio) on the measured figure
    pmul = 2.0 if mx else 1.0
    peak_tf = pmul * peaks.get(peak_key, FALLBACK_PEAKS[peak_key])
    sust_tf = pmul * peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "ffn_traffic.json")
    if os.path.exists(tpath) and not mx:
        try:
            import hashlib
            with open(tpath) as f:
                tj = json.load(f)
            # the FFN kernel's source: grouped_gemm.cu and the tcgen05 helpers it includes
            csrc = os.path.join(ROOT, "expert_dispatch_fp32_b200", "csrc")
            src = b"".join(open(os.path.join(csrc, f), "rb").read() for f in ("grouped_gemm.cu", "tc_common.cuh"))
            ent = tj.get(wl.name)
            if ent and ent.get("kernel_sha256") == hashlib.sha256(src).hexdigest():
                traffic = ent["dram_bytes_per_step"]
        except Exception:
            traffic = None
    disp_b, comb_b = stage_bytes(wl)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    disp_gbs = disp_b / (stage_ms[2] / args.steps / 1e3) / 1e9
    comb_gbs = comb_b / (stage_ms[4] / args.steps / 1e3) / 1e9
    # MXFP8 FFN: x_perm quantiser (inside the dispatch when that is a separate stage),
    # gate_up, down, and the shared experts' launch
    n_ffn = (3 + (1 if wl.n_shared else 0)) if mx else ffn_launches(wl)
    launches_per_step = (1 if fused else route_launches(wl) + 1 + 1) + n_ffn + 1

    # layer roofline: the sum of every stage's ideal time over the measured step.  Ideal
    # times: route = max(bytes / HBM, flop / fp32 peak), the fp32 peak from the unit counts
    # (148 SMs x 128 FP32 lanes x 2 flop x the max SM clock); preprocess and dispatch and
    # combine = bytes / HBM; FFN = max(flop / the bf16 peak used above, bytes of the hit
    # experts' weights / HBM)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    fp32_tf = sms * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    hit = int((b["counts"][:wl.E] > 0).sum().item())
    mats = 3 if wl.act == "swiglu" else 2
    w_bytes = hit * mats * wl.D * wl.F * (1 if mx else 2) + wl.n_shared * 3 * wl.D * wl.F_shared * 2
    hbm_bs = hbm * 1e9
    ideal_us = {
        "route": 1e6 * max((wl.T * wl.D * sx + wl.E * wl.D * 4 + wl.R * 8) / hbm_bs,
                           2.0 * wl.T * wl.D * wl.E / (fp32_tf * 1e12)),
        "preprocess": 1e6 * wl.R * 12 / hbm_bs,
        "dispatch": 1e6 * disp_b / hbm_bs,
        "expert_ffn": 1e6 * max(wl.ffn_flop() / (peak_tf * 1e12), w_bytes / hbm_bs),
        "combine": 1e6 * comb_b / hbm_bs,
    }
    step_us = 1e3 * total_ms_max / args.steps
    layer_roofline = {"ideal_us": ideal_us, "sum_ideal_us": sum(ideal_us.values()),
                      "measured_us": step_us, "frac": sum(ideal_us.values()) / step_us,
                      "fp32_peak_tflops": fp32_tf, "ffn_peak": peak_key}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "mxfp8 routed experts (e4m3, e8m0 per 32), bf16 elsewhere" if mx else "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name + ("_mxfp8" if mx else ""), "T": wl.T, "D": wl.D, "E": wl.E, "ep_size": wl.ep_size,
                   "top_k": wl.top_k, "F": wl.F, "act": wl.act, "n_shared": wl.n_shared,
                   "F_shared": wl.F_shared, "router": "fp32", "parallelism": f"replicas{ws}",
                   "l2": "flushed before every timed step: 256 MiB write, then a read of it (no dirty lines left)"},
        "roofline": {"bound": "tensor", "achieved": ffn_tflops, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": ffn_tflops / peak_tf, "traffic": traffic,
                     "kernel": (("mx_quant_a_kernel + grouped_gemm_mx_kernel x2 (routed gate_up, "
                                 "down; MXFP8)" + (" + shared experts' bf16 launch" if wl.n_shared else ""))
                                if mx else
                                ("grouped_gemm_pair_kernel, one launch" if ffn_launches(wl) == 1
                                 else "grouped_gemm_kernel launches")
                                + " (expert FFN stage: routed gate_up+down"
                                + (", shared gate_up+down" if wl.n_shared else "") + ")"),
                     "timed": "CUDA events around the FFN stage call in a stage-by-stage pass "
                              "of the same kernels, after an L2 flush per step",
                     "peak_source": (f"2 x {peak_src} bf16 burst (fp8 dense = 2 x bf16, nominal ratio)"
                                     if mx else f"{peak_src} bf16 burst (cuBLAS 8192^3, best of 10)"),
                     "frac_of_sustained": ffn_tflops / sust_tf},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * wl.D * sx,
                "d2h_bytes_per_step": T * wl.D * sx},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "stages_us": {n: 1e3 * float(v) / args.steps for n, v in
                      zip(("route", "preprocess", "dispatch", "expert_ffn", "combine"), stage_ms)},
        "forward_stages_us": ({n: 1e3 * float(v) / args.steps for n, v in
                               zip(("route_preprocess_dispatch", "expert_ffn", "combine"), fused_ms)}
                              if fused else None),
        "ffn_tflops": ffn_tflops,
        "layer_roofline": layer_roofline,
        "dispatch_gbs": disp_gbs, "dispatch_frac_hbm": disp_gbs / hbm,
        "combine_gbs": comb_gbs, "combine_frac_hbm": comb_gbs / hbm,
    }
    if want_cpu:
        # sized for 10-20 s of oracle work: the calibration undersizes large samples
        # (their BLAS steps run more efficiently per token), so a sample that ran under
        # 8 s is scaled up and timed again, at most twice (the line reports the last)
        n_tok = args.cpu_sample or pick_sample(wl, cpu_host, 15.0)
        t = cpu_oracle_time(wl, cpu_host, n_tok, seed=1)
        cap = 16 * wl.T
        for rep in range(2):
            if args.cpu_sample or t >= 8.0 or n_tok >= cap:
                break
            n_tok = int(min(cap, n_tok * 15.0 / max(t, 1e-6)))
            t = cpu_oracle_time(wl, cpu_host, n_tok, seed=2 + rep)
        line["cpu_baseline"] = {"value": n_tok / t, "unit": "tokens/s", "cores": cpu_threads(),
                                "kind": "oracle",
                                "sample": f"{n_tok} tokens drawn from the {wl.name} batch "
                                          f"({t:.1f} s of float64 numpy on the host)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
