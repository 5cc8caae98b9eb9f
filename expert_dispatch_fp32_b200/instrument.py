"""Where the expert-FFN kernels spend their cycles, from an instrumented build.

    python -m expert_dispatch_fp32_b200.instrument --workload deepseek_v3 [--mxfp8]

Builds lib/libmoe_instr.so (the same sources with the kernels' clock64 counters compiled
in, -DMOE_INSTRUMENT), loads it in place of libmoe.so, runs the workload's layer once
(warm-up), flushes L2 and runs the expert-FFN stage alone, then reads the counters of
that one launch (moe_instr_read) and prints, for the MMA issuer of every CTA pair summed:
the share of its cycles spent waiting for a drained accumulator, waiting for a filled
stage and issuing; cycles per K step by tile kind (full M = 256, M = 128, folded,
skinny); and the producer's and first epilogue warp's waits.  Counters are SM cycles
(clock64); the counting itself adds a few instructions per K step, so absolute times
are a little above an ordinary build's.
"""
from __future__ import annotations

import argparse
import os
import sys


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="deepseek_v3")
    ap.add_argument("--mxfp8", action="store_true", help="the MXFP8 routed experts")
    ap.add_argument("--tokens", type=int, default=0, help="override T")
    a = ap.parse_args(argv)

    from . import build as _build
    lib_path = _build.build(instrument=True)
    from . import _binding as B
    if B._lib is not None and B.LIB_PATH != lib_path:
        raise RuntimeError("libmoe.so is already loaded in this process")
    B.LIB_PATH = lib_path

    import numpy as np
    import torch
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import moe_workloads as W
    from .layer import MoELayer

    wl = W.get(a.workload)
    if a.tokens:
        wl = wl.with_(T=a.tokens)
    inp = W.make_inputs(wl, device="cuda")
    up = inp["w_gate_up"] if wl.act == "swiglu" else inp["w1"]
    layer = MoELayer(D=wl.D, E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, F=wl.F, w_router=inp["w_router"],
                     w_gate_up=up, w_down=inp["w_down"], expert_bias=inp["bias"],
                     ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"], act=wl.act, x_dtype=wl.x_dtype,
                     mxfp8=a.mxfp8)
    for k in ("w_gate_up", "w1", "w_down", "ws_gate_up", "ws_down"):
        inp.pop(k, None)
    x = inp["x"]
    T = wl.T
    b = layer.allocate(T)
    cfg = layer.config(T)
    layer.forward(x)
    torch.cuda.synchronize()
    layer.check_status()
    kernel = 1 if a.mxfp8 else 0
    B.moe_instr_read(kernel)                       # zero the warm-up's counts
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush.zero_()
    flush.view(torch.float32).sum()
    xb = x if wl.x_dtype == "bf16" else None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    if a.mxfp8:
        fused = wl.x_dtype != "bf16" or B.moe_route_dispatch_is_fused(cfg)
        B.moe_expert_ffn_mxfp8(cfg, b["x_perm"] if fused else None, xb, b["expert_offsets"], layer.packed,
                               layer.packed_mx, b["y_perm"], b["shared_out"], b["workspace"], b["status"])
    else:
        B.moe_expert_ffn(cfg, b["x_perm"], xb, b["expert_offsets"], layer.packed, b["act"], b["y_perm"],
                         b["shared_out"], b["workspace"], b["status"])
    e1.record()
    torch.cuda.synchronize()
    layer.check_status()
    c = B.moe_instr_read(kernel).astype(np.float64)
    lead = c[c[:, 0] > 0]                         # rows of CTAs whose MMA issuer ran
    tot = lead[:, 0].sum()
    ms = e0.elapsed_time(e1)
    print(f"{a.workload}{' mxfp8' if a.mxfp8 else ''}: expert-FFN stage {ms:.3f} ms (instrumented build), "
          f"{len(lead)} MMA issuers")
    if tot == 0:
        print("no counts (the stage ran no instrumented kernel)")
        return 1
    wa, wf = lead[:, 1].sum(), lead[:, 2].sum()
    print(f"MMA issuer cycles: waiting for the accumulator {wa / tot:.3f}, waiting for a filled stage "
          f"{wf / tot:.3f}, issuing {(tot - wa - wf) / tot:.3f}")
    ks = lead[:, 11].sum()
    print(f"K steps {ks:.0f}; issuer cycles per K step, all tiles: {(tot - wa) / max(ks, 1):.0f}")
    print("| tile kind | tiles | K steps | issuer cycles per K step | share of issuer cycles |")
    print("|---|---|---|---|---|")
    for j, name in enumerate(("full M = 256", "M = 128", "folded", "skinny")):
        n, cyc, k = lead[:, 3 + 2 * j].sum(), lead[:, 4 + 2 * j].sum(), lead[:, 16 + j].sum()
        if n:
            print(f"| {name} | {n:.0f} | {k:.0f} | {cyc / max(k, 1):.0f} | {cyc / tot:.3f} |")
    pw, pt = c[:, 12].sum(), c[:, 13].sum()
    ew, et = c[:, 14].sum(), c[:, 15].sum()
    if pt:
        print(f"producers: waiting for a free stage {pw / pt:.3f} of their cycles")
    if et:
        print(f"first epilogue warps: waiting for a full accumulator {ew / et:.3f} of their cycles")
    return 0


if __name__ == "__main__":
    sys.exit(main())
