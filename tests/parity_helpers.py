"""Shared helpers for the GPU parity tests (CUDA path vs the CPU oracle).

Tolerances (fixed by the layer's stated accuracy contract):
  * routing indices, counts, splits, permutation: bit-exact, except tokens whose
    fp32 gap between the k-th and (k+1)-th logit is below GAP (exempt, counted)
    and, for the order inside the top-k only, tokens with an adjacent in-top-k
    gap below GAP (the set must still match);
  * layer outputs: relative L2 error <= REL_L2 and max-abs error <= MAX_ABS *
    max|ref| against the oracle on the same bf16-rounded inputs and weights.
"""
import numpy as np
import torch

import expert_dispatch_fp32_b200 as M
import moe_workloads as W
import oracle

GAP = 1e-5
REL_L2 = 1e-2
MAX_ABS = 2e-2
W_ATOL = 1e-5          # routing weights: fp32 exp/sum on the GPU vs float64 oracle


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def up_weights(wl, inp):
    return inp["w_gate_up"] if wl.act == "swiglu" else inp["w1"]


def make_layer(wl, inp, keep_logits=False):
    return M.MoELayer(D=wl.D, E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, F=wl.F,
                      w_router=inp["w_router"], w_gate_up=up_weights(wl, inp), w_down=inp["w_down"],
                      expert_bias=inp["bias"], ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"],
                      act=wl.act, renormalize=wl.renormalize, x_dtype=wl.x_dtype,
                      keep_router_logits=keep_logits)


def host_bias(inp):
    return None if inp["bias"] is None else inp["bias"].cpu().numpy()


def oracle_route(wl, inp, tokens=None):
    x = inp["x"] if tokens is None else inp["x"][torch.as_tensor(tokens, device=inp["x"].device)]
    logits = oracle.router_logits(f64(x), inp["w_router"].cpu().numpy(), host_bias(inp))
    idx, w = oracle.topk_select(logits, wl.top_k, wl.renormalize)
    gap, inner = oracle.route_gaps(logits, wl.top_k)
    return dict(logits=logits, idx=idx, w=w, gap=gap, inner=inner)


MAX_EXEMPT_FRAC = 0.005   # near-tie tokens allowed before a test calls the exemption suspect


def compare_routing(gpu_idx, gpu_w, ref, max_exempt="default"):
    """Assert routing parity; returns (n_exempt, n_exempt_that_differ).

    The exemption must stay rare: random logits put a k-th/(k+1)-th gap below 1e-5
    on about 1e-4 of tokens, so more than MAX_EXEMPT_FRAC of T (at least 2 tokens)
    means the gaps are wrong, not the routing.  Tests built on exact ties pass
    max_exempt=None."""
    idx, w = ref["idx"], ref["w"]
    exempt = ref["gap"] < GAP
    order_exempt = (ref["inner"] < GAP) & ~exempt
    if max_exempt == "default":
        max_exempt = max(2, int(MAX_EXEMPT_FRAC * len(idx)))
    n_ex = int(exempt.sum() + order_exempt.sum())
    print(f"[routing] tokens {len(idx)}, set-exempt {int(exempt.sum())}, "
          f"order-exempt {int(order_exempt.sum())}")
    if max_exempt is not None:
        assert n_ex <= max_exempt, f"{n_ex} exempt tokens of {len(idx)} (bound {max_exempt})"
    strict = ~exempt & ~order_exempt
    bad = np.nonzero(~np.all(gpu_idx[strict] == idx[strict], axis=1))[0]
    assert bad.size == 0, f"{bad.size} non-exempt tokens route differently, e.g. {np.nonzero(strict)[0][bad[:5]]}"
    if order_exempt.any():
        assert np.array_equal(np.sort(gpu_idx[order_exempt], 1), np.sort(idx[order_exempt], 1))
    assert np.allclose(gpu_w[strict], w[strict], rtol=0, atol=W_ATOL)
    if order_exempt.any():   # same set: compare the weights matched by expert id
        for t in np.nonzero(order_exempt)[0]:
            a = dict(zip(gpu_idx[t].tolist(), gpu_w[t].tolist()))
            b = dict(zip(idx[t].tolist(), w[t].tolist()))
            assert all(abs(a[e] - b[e]) <= W_ATOL for e in b)
    differ = exempt & ~np.all(gpu_idx == idx, axis=1)
    return int(exempt.sum()), int(differ.sum())


def layer_errors(got, ref, resid):
    got, ref, resid = (np.asarray(a, dtype=np.float64) for a in (got, ref, resid))
    d = got - ref
    rel_l2 = np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300)
    max_abs = np.abs(d).max() / max(np.abs(ref).max(), 1e-300)
    moe_ref = ref - resid
    moe_rel = np.linalg.norm(d) / max(np.linalg.norm(moe_ref), 1e-300)
    return rel_l2, max_abs, moe_rel


def assert_layer_close(got, ref, resid, what="out"):
    """Assert the output contract; the error on the MoE part (out - x) is returned
    for reporting only: with a bf16 output it is dominated by the one rounding of
    x + moe whenever the MoE part is small next to the residual."""
    rel_l2, max_abs, moe_rel = layer_errors(got, ref, resid)
    assert rel_l2 <= REL_L2, f"{what}: rel-L2 {rel_l2:.3e}"
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} of max|ref|"
    return rel_l2, max_abs, moe_rel


def oracle_layer(wl, inp, tokens=None):
    """Oracle forward for all tokens or a token subset, streaming expert weights."""
    x = inp["x"] if tokens is None else inp["x"][torch.as_tensor(tokens, device=inp["x"].device)]
    wup = up_weights(wl, inp)
    cache = {}

    def fetch(e):
        if e not in cache:
            cache.clear()
            cache[e] = (f64(wup[e]), f64(inp["w_down"][e]))
        return cache[e]

    swu = None if inp["ws_gate_up"] is None else f64(inp["ws_gate_up"])
    swd = None if inp["ws_down"] is None else f64(inp["ws_down"])
    return oracle.moe_layer(f64(x), inp["w_router"].cpu().numpy(), host_bias(inp), None, None, swu,
                            swd, E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, act=wl.act,
                            renormalize=wl.renormalize, x_is_f32=(wl.x_dtype == "f32"),
                            expert_weights=fetch)


def sample_tokens(T, n, seed=0):
    """First, last and random interior tokens (crossing tile boundaries)."""
    rng = np.random.default_rng(seed)
    picks = {0, T - 1, min(127, T - 1), min(128, T - 1)}
    picks.update(rng.choice(T, size=min(n, T), replace=False).tolist())
    return np.array(sorted(picks))


def cuda_inputs(wl):
    torch.cuda.empty_cache()
    return W.make_inputs(wl, device="cuda")
