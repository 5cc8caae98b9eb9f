"""Seeded synthetic workloads for the expert-parallel MoE-layer forward.

This module is shared by both sides of every parity check: the CUDA path's tests
and bench, and the oracle's tests.  It holds workload *shapes* and draws random
numbers in a fixed order; it performs none of the layer's arithmetic (no router,
no selection, no FFN, no combine).  The only values it derives are inputs that
the workload definition itself fixes: the bf16 storage of drawn weights (RNE cast
of fp32 draws) and the per-expert router bias of the load-skew workload.

Draw order (one generator per workload, seeded with ``seed``):
  x, W_r, then per routed expert e: gate_up[e] (or W1[e] for GELU), down[e] (W2[e]),
  then per shared expert i: gate_up_s[i], down_s[i].
Each tensor is drawn in fp32 as N(0, 1) * std, one expert at a time, then cast to
its storage dtype.  Values therefore depend on (workload, seed, device kind): the
CPU and CUDA generators are different streams, and each run hands the *same bits*
to the CUDA path and to the oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    """Shape and distribution of one MoE-layer forward workload."""

    name: str
    T: int                     # tokens
    D: int                     # model dim
    E: int                     # routed experts
    ep_size: int               # virtual expert-parallel ranks
    top_k: int
    F: int                     # routed expert intermediate dim
    act: str = "swiglu"        # "swiglu" | "gelu"
    x_dtype: str = "bf16"      # "bf16" | "f32"
    n_shared: int = 0
    F_shared: int = 0
    renormalize: bool = True
    zipf_bias: bool = False    # router bias b_e = 2*log(1/(e+1))
    x_std: float = 1.0
    w_router_std: float = 0.02
    w1_std: float = 0.02       # gate_up (or W1) std
    w2_std: float = 0.02       # down (or W2) std
    seed: int = 0
    doc: str = field(default="", compare=False)

    @property
    def R(self) -> int:
        """Routed rows = T * top_k (dropless)."""
        return self.T * self.top_k

    @property
    def El(self) -> int:
        return self.E // self.ep_size

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def ffn_flop(self) -> float:
        """Algorithmic FFN flop over real rows only."""
        mats = 3 if self.act == "swiglu" else 2
        routed = 2.0 * self.R * self.D * self.F * mats
        shared = 2.0 * self.T * self.D * self.F_shared * 3 * self.n_shared
        return routed + shared


# The five workloads.  Names say what each is; sizes follow the shapes the pages
# discuss (a 4x4-expert top-2 trace, a Mixtral-8x7B block, a DeepSeek-V3 block,
# and a Zipf-skewed router).
WORKLOADS: dict[str, Workload] = {
    "worked_example_t64": Workload(
        name="worked_example_t64", T=64, D=64, E=16, ep_size=4, top_k=2, F=128,
        act="gelu", x_dtype="f32", w1_std=1.0 / math.sqrt(64), w2_std=1.0 / math.sqrt(128),
        doc="4 virtual ranks x 4 experts, top-2, GELU FFN 64->128->64, fp32 x"),
    "small_e8_d2048": Workload(
        name="small_e8_d2048", T=4096, D=2048, E=8, ep_size=2, top_k=2, F=5632,
        doc="small bf16 block, 2 virtual ranks x 4 experts, SwiGLU F=5632"),
    "mixtral_8x7b": Workload(
        name="mixtral_8x7b", T=8192, D=4096, E=8, ep_size=8, top_k=2, F=14336,
        doc="Mixtral-8x7B-shaped layer, 8 virtual ranks x 1 expert"),
    "deepseek_v3": Workload(
        name="deepseek_v3", T=8192, D=7168, E=256, ep_size=8, top_k=8, F=2048,
        n_shared=1, F_shared=2048,
        doc="DeepSeek-V3-shaped fine-grained layer, 8 x 32 experts, top-8, 1 shared"),
    "zipf_skew_e64": Workload(
        name="zipf_skew_e64", T=16384, D=2048, E=64, ep_size=8, top_k=6, F=1408,
        n_shared=2, F_shared=1408, zipf_bias=True,
        doc="load skew: router bias 2*log(1/(e+1)), many empty experts, 2 shared"),
}

# Listed in the order the workload table gives them.
WORKLOAD_ORDER = ["worked_example_t64", "small_e8_d2048", "mixtral_8x7b",
                  "deepseek_v3", "zipf_skew_e64"]


def get(name: str) -> Workload:
    return WORKLOADS[name]


def _draw(gen: torch.Generator, shape, std: float, device, dtype) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def router_bias(wl: Workload) -> torch.Tensor | None:
    """Per-expert router bias fixed by the load-skew workload: 2*log(1/(e+1)), fp32."""
    if not wl.zipf_bias:
        return None
    return torch.tensor([2.0 * math.log(1.0 / (e + 1)) for e in range(wl.E)], dtype=torch.float32)


def make_inputs(wl: Workload, device="cpu") -> dict:
    """Draw all inputs of ``wl`` on ``device`` in the fixed order.

    Returns a dict of tensors:
      x           [T, D]        fp32 or bf16
      w_router    [E, D]        fp32
      bias        [E] fp32 or None
      w_gate_up   [E, D, 2F]    bf16, first F columns = gate, last F = up  (SwiGLU)
      w1          [E, D, F]     bf16                                       (GELU)
      w_down      [E, F, D]     bf16  (W2 for GELU)
      ws_gate_up  [S, D, 2Fs]   bf16 or None
      ws_down     [S, Fs, D]    bf16 or None
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    xdt = torch.float32 if wl.x_dtype == "f32" else torch.bfloat16
    out: dict = {}
    out["x"] = _draw(gen, (wl.T, wl.D), wl.x_std, device, xdt)
    out["w_router"] = _draw(gen, (wl.E, wl.D), wl.w_router_std, device, torch.float32)
    b = router_bias(wl)
    out["bias"] = None if b is None else b.to(device)
    up_cols = 2 * wl.F if wl.act == "swiglu" else wl.F
    wgu = torch.empty((wl.E, wl.D, up_cols), dtype=torch.bfloat16, device=device)
    wd = torch.empty((wl.E, wl.F, wl.D), dtype=torch.bfloat16, device=device)
    for e in range(wl.E):
        wgu[e] = _draw(gen, (wl.D, up_cols), wl.w1_std, device, torch.bfloat16)
        wd[e] = _draw(gen, (wl.F, wl.D), wl.w2_std, device, torch.bfloat16)
    if wl.act == "swiglu":
        out["w_gate_up"] = wgu
    else:
        out["w1"] = wgu
    out["w_down"] = wd
    if wl.n_shared > 0:
        S, Fs = wl.n_shared, wl.F_shared
        sgu = torch.empty((S, wl.D, 2 * Fs), dtype=torch.bfloat16, device=device)
        sd = torch.empty((S, Fs, wl.D), dtype=torch.bfloat16, device=device)
        for i in range(S):
            sgu[i] = _draw(gen, (wl.D, 2 * Fs), wl.w1_std, device, torch.bfloat16)
            sd[i] = _draw(gen, (Fs, wl.D), wl.w2_std, device, torch.bfloat16)
        out["ws_gate_up"], out["ws_down"] = sgu, sd
    else:
        out["ws_gate_up"], out["ws_down"] = None, None
    return out


def make_router_inputs(wl: Workload, device="cpu") -> dict:
    """x, w_router and bias only: the first two draws of ``make_inputs`` (same
    generator, same order, so the same bits), without drawing the expert weights."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    xdt = torch.float32 if wl.x_dtype == "f32" else torch.bfloat16
    x = _draw(gen, (wl.T, wl.D), wl.x_std, device, xdt)
    w_router = _draw(gen, (wl.E, wl.D), wl.w_router_std, device, torch.float32)
    b = router_bias(wl)
    return {"x": x, "w_router": w_router, "bias": None if b is None else b.to(device)}


def make_x(wl: Workload, device="cpu", seed: int | None = None) -> torch.Tensor:
    """A fresh activation batch only (same distribution as ``make_inputs``' x)."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed if seed is None else seed)
    xdt = torch.float32 if wl.x_dtype == "f32" else torch.bfloat16
    return _draw(gen, (wl.T, wl.D), wl.x_std, device, xdt)


def to_numpy_f64(t: torch.Tensor):
    """Exact float64 copy of a CPU/GPU tensor (bf16 and fp32 embed exactly in fp64)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def bf16_bits(t: torch.Tensor):
    """Raw bf16 bit patterns as a numpy uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
