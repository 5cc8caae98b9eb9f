"""Seeded input generator: determinism, shapes, dtypes, and the skew recipe."""
import math

import numpy as np
import torch

import moe_workloads as W
import oracle


def test_presets_shapes():
    for name in W.WORKLOAD_ORDER:
        wl = W.get(name)
        assert wl.E % wl.ep_size == 0
        assert 1 <= wl.top_k <= wl.E
        assert wl.D % 64 == 0
        assert (wl.F % 128 == 0) if wl.act == "swiglu" else (wl.F % 64 == 0)


def test_make_inputs_deterministic_and_typed():
    wl = W.get("worked_example_t64")
    a = W.make_inputs(wl)
    b = W.make_inputs(wl)
    for key in ("x", "w_router", "w1", "w_down"):
        assert torch.equal(a[key], b[key])
    assert a["x"].dtype == torch.float32 and a["w1"].dtype == torch.bfloat16
    assert a["w1"].shape == (16, 64, 128) and a["w_down"].shape == (16, 128, 64)
    assert a["bias"] is None and a["ws_gate_up"] is None
    # std of the drawn weights follows the recipe (1/sqrt(fan_in))
    assert abs(a["w1"].float().std().item() - 1 / 8) < 0.01
    assert abs(a["w_down"].float().std().item() - 1 / math.sqrt(128)) < 0.01


def test_small_skew_recipe():
    wl = W.get("zipf_skew_e64").with_(T=512, D=128, F=128, F_shared=128)
    inp = W.make_inputs(wl)
    b = inp["bias"].numpy()
    assert b.dtype == np.float32 and b[0] == 0.0
    assert np.allclose(b, [2 * math.log(1 / (e + 1)) for e in range(64)], rtol=1e-6)
    assert inp["ws_gate_up"].shape == (2, 128, 256) and inp["ws_down"].shape == (2, 128, 128)
    # the bias skews the load: expert 0 takes most tokens, high experts get none
    x = W.to_numpy_f64(inp["x"])
    logits = oracle.router_logits(x, inp["w_router"].numpy(), b)
    idx, _ = oracle.topk_select(logits, wl.top_k)
    counts = np.bincount(idx.ravel(), minlength=64)
    assert counts[0] > 0.9 * wl.T and (counts == 0).sum() >= 10


def test_oracle_full_tiny_workload():
    wl = W.get("worked_example_t64")
    inp = W.make_inputs(wl)
    res = oracle.moe_layer(W.to_numpy_f64(inp["x"]), inp["w_router"].numpy(), None,
                           W.to_numpy_f64(inp["w1"]), W.to_numpy_f64(inp["w_down"]), None, None,
                           E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, act="gelu", x_is_f32=True)
    assert res["out"].shape == (64, 64)
    assert res["counts"].sum() == wl.R
    assert np.all(np.isfinite(res["out"]))


def test_router_inputs_are_the_first_draws():
    wl = W.get("zipf_skew_e64").with_(T=96, D=128, F=128, F_shared=128)
    full = W.make_inputs(wl)
    part = W.make_router_inputs(wl)
    for key in ("x", "w_router", "bias"):
        assert torch.equal(full[key], part[key]), key
