"""How close the tensor-core router runs to the error bound its filter relies on.

For bf16 x and many experts, moe_route finds each token's top-k in two steps: the
tensor cores form approx[t,e] = x_t . (hi_e + mid_e) (W_r = hi + mid + lo, hi and mid
bf16, fp32 accumulation), then every expert whose approximate logit is within
2 eps_t of the k-th largest gets an exact fp32 logit, eps_t = coef * sum_d |x_d| wmax_d.
No true top-k expert is dropped as long as |approx - exact| <= eps_t for every expert,
where eps_t assumes each 16-deep MMA instruction adds at most two fp32 rounding
errors of that magnitude ("Expert Parallel (EP)", Configuration: the router runs in
fp32, so the top-k must be the fp32 one).  These tests read the approximate logits
the kernel left in the workspace and measure |approx - exact| / eps_t against the
oracle's logits, on the full-size workloads and on inputs built for heavy
cancellation, where the partial sums are five orders of magnitude larger than the
logits they cancel down to.
"""
import numpy as np
import pytest
import torch

import expert_dispatch_fp32_b200 as M
import moe_workloads as W
import oracle
from parity_helpers import compare_routing, f64, oracle_route

pytestmark = pytest.mark.gpu

MARGIN = 0.5     # the observed error must stay within half the assumed bound


def _route_and_view(wl, inp):
    cfg = M.make_config(wl.T, wl.D, wl.E, wl.ep_size, wl.top_k, wl.F)
    view = M.moe_router_filter_view(cfg)
    assert view is not None, "this configuration should take the tensor-core router"
    ao, ld, wo, coef = view
    ws = torch.zeros(M.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    idx = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.top_k), dtype=torch.float32, device="cuda")
    M.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], None, idx, w, ws)
    torch.cuda.synchronize()
    approx = ws[ao:ao + wl.T * ld * 4].view(torch.float32).view(wl.T, ld)[:, :wl.E]
    wmax = ws[wo:wo + wl.D * 4].view(torch.float32)
    return idx.cpu().numpy(), w.cpu().numpy(), f64(approx), f64(wmax), coef


def _margin(wl, inp, approx, wmax, coef):
    x = f64(inp["x"])
    wr = inp["w_router"].cpu().numpy()
    # wmax is max_e |W_r[e, d]| (what the bound is built from)
    assert np.array_equal(wmax, np.abs(wr.astype(np.float64)).max(axis=0))
    exact = oracle.router_logits(x, wr, None).astype(np.float64)   # no bias: approx has none
    eps = coef * (np.abs(x) @ wmax)
    ratio = np.abs(approx - exact) / eps[:, None]
    return float(ratio.max()), float(np.median(ratio.max(axis=1)))


@pytest.mark.parametrize("name", ["deepseek_v3", "zipf_skew_e64"])
def test_filter_error_within_half_its_bound(name):
    wl = W.get(name)
    inp = W.make_router_inputs(wl, device="cuda")
    idx, w, approx, wmax, coef = _route_and_view(wl, inp)
    worst, typical = _margin(wl, inp, approx, wmax, coef)
    print(f"\n{name}: max |approx - exact| / eps_t = {worst:.3e} (median over tokens "
          f"{typical:.3e}), coef {coef:.3e}")
    assert worst <= MARGIN
    compare_routing(idx, w, oracle_route(wl, inp))


def test_filter_under_heavy_cancellation():
    """x mixes magnitudes from 2^-8 to 2^9 with one sign over the first half of D and the
    negated values over the second, and every router row is 0.5 plus a small per-expert
    part: the bf16 hi rows are all exactly 0.5, so the hi chain of the tensor-core
    product sums to zero only in exact arithmetic, and in fp32 its partial sums climb to
    ~1e5 and drop small terms.  The approximate logits' error then exceeds the spacing
    of the exact ones; the filter must keep every expert the bound cannot exclude and
    the result must still be the exact fp32 top-k."""
    T, D, E, k = 1024, 7168, 256, 8      # enough tokens for the tensor-core router
    wl = W.Workload(name="cancel", T=T, D=D, E=E, ep_size=8, top_k=k, F=128)
    g = torch.Generator(device="cpu").manual_seed(3)
    expo = torch.randint(-8, 10, (T, D // 2), generator=g).to(torch.float32)
    mag = torch.exp2(expo) * (1.0 + torch.rand((T, D // 2), generator=g))
    x = torch.cat([mag, -mag.flip(1)], dim=1).to(torch.bfloat16)      # sum_d x_d = 0 exactly
    tiny = torch.randn((E, D), generator=g) * 1e-3
    wr = (0.5 + tiny).to(torch.float32)
    inp = {"x": x.cuda(), "w_router": wr.cuda(), "bias": None}
    idx, w, approx, wmax, coef = _route_and_view(wl, inp)
    worst, typical = _margin(wl, inp, approx, wmax, coef)
    ref = oracle_route(wl, inp)
    lg = ref["logits"].astype(np.float64)
    srt = -np.sort(-lg, axis=1)
    spacing = float(np.median(srt[:, k - 1] - srt[:, k]))
    err = float(np.abs(approx - oracle.router_logits(f64(inp["x"]), wr.numpy(), None)).max())
    print(f"\ncancellation: max |approx - exact| / eps_t = {worst:.3e}, max |approx - exact| "
          f"{err:.3e}, median k-th/(k+1)-th spacing {spacing:.3e}")
    assert worst <= MARGIN
    # near-ties are legitimate here (constructed logits): exempt tokens are counted, the
    # rest must match the oracle exactly
    compare_routing(idx, w, ref, max_exempt=None)
