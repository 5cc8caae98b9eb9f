"""GPU edge cases: ragged batches, skewed and empty experts, k = E, ties, the
worked example's closed form, device error reporting and determinism."""
import math
import os

import numpy as np
import pytest
import torch

import expert_dispatch_fp32_b200 as M
import moe_workloads as W
import oracle
from conftest import read_golden
from parity_helpers import (assert_layer_close, compare_routing, f64, make_layer, oracle_layer,
                            oracle_route, up_weights)

pytestmark = pytest.mark.gpu

BASE = W.Workload(name="edge", T=256, D=128, E=8, ep_size=2, top_k=2, F=256, act="swiglu")


def run_and_compare(wl, inp=None, full=True):
    inp = inp or W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    out = layer.forward(inp["x"])
    torch.cuda.synchronize()
    layer.check_status()
    ref = oracle_route(wl, inp)
    b = layer.buf
    compare_routing(b["topk_idx"].cpu().numpy(), b["topk_w"].cpu().numpy(), ref)
    pre = oracle.preprocess(ref["idx"], wl.E, wl.ep_size)
    if np.array_equal(b["topk_idx"].cpu().numpy(), ref["idx"]):
        for key in ("counts", "expert_offsets", "rank_splits", "rank_offsets", "pos", "src"):
            assert np.array_equal(b[key].cpu().numpy(), pre[key]), key
    res = oracle_layer(wl, inp)
    assert_layer_close(f64(out), res["out"], f64(inp["x"]))
    return layer, inp, res


@pytest.mark.parametrize("T", [1, 3, 127, 128, 129, 1000])
def test_ragged_batches(T):
    run_and_compare(BASE.with_(T=T, seed=T))


@pytest.mark.parametrize("D,F,act", [(64, 128, "swiglu"), (128, 128, "gelu"), (192, 64, "gelu"),
                                     (320, 384, "swiglu")])
def test_tile_widths(D, F, act):
    # D % 256 != 0 and F % 256 != 0 take the 128- and 64-wide tiles; K = 64 is one K step
    run_and_compare(BASE.with_(T=300, D=D, F=F, act=act, x_dtype="f32" if act == "gelu" else "bf16"))


@pytest.mark.parametrize("T", [5, 40])
def test_decode_batch_with_shared_experts(T):
    """Decode-sized batches: every expert group and the shared expert's single band
    hold at most 64 rows, so every tile of the FFN launch is skinny."""
    run_and_compare(BASE.with_(T=T, D=256, E=16, ep_size=4, top_k=2, F=256, n_shared=1,
                               F_shared=256, seed=T))


@pytest.mark.parametrize("T,E,k,zipf", [(24, 64, 6, True), (9, 256, 8, False)])
def test_decode_batch_many_experts(T, E, k, zipf):
    """A decode-sized forward with more than 32 experts: the split-K router, skinny FFN
    tiles (every group holds a few rows), shared experts and the hoisted combine, against
    the oracle."""
    run_and_compare(BASE.with_(T=T, D=512, E=E, ep_size=8, top_k=k, F=256, n_shared=1,
                               F_shared=256, zipf_bias=zipf, seed=T))


def test_k_equals_e_and_no_renormalisation():
    run_and_compare(BASE.with_(T=200, E=8, top_k=8, ep_size=4))
    run_and_compare(BASE.with_(T=200, renormalize=False))


def test_shared_experts_small():
    run_and_compare(BASE.with_(T=333, E=16, ep_size=4, top_k=3, n_shared=2, F_shared=128))


def test_all_tokens_to_one_expert_and_empty_experts():
    wl = BASE.with_(T=700, E=16, ep_size=4, top_k=2, zipf_bias=False)
    inp = W.make_inputs(wl, device="cuda")
    bias = torch.full((16,), -50.0, device="cuda")
    bias[5] = 50.0       # expert 5 is every token's first choice
    bias[9] = 40.0       # expert 9 every token's second
    inp["bias"] = bias
    layer, _, res = run_and_compare(wl, inp)
    counts = layer.buf["counts"].cpu().numpy()
    assert counts[5] == 700 and counts[9] == 700 and counts.sum() == 1400
    assert list(layer.buf["rank_splits"].cpu().numpy()) == [0, 700, 700, 0]


def test_zipf_skew_small():
    run_and_compare(W.get("zipf_skew_e64").with_(T=2000, D=256, F=256, F_shared=128))


@pytest.mark.parametrize("T", [7043, 9000])
def test_few_expert_router_four_tokens_per_warp(T):
    """Batches large enough for the four-tokens-per-warp router (with a ragged last
    group of tokens): routing and the whole layer against the oracle."""
    run_and_compare(BASE.with_(T=T, D=512, E=8, top_k=2, F=128, seed=3))


@pytest.mark.parametrize("T,D,E,k,xdt,renorm,logits,shared", [
    (1, 128, 8, 2, "bf16", True, False, False),
    (3, 256, 8, 8, "bf16", True, True, False),          # k = E
    (129, 512, 16, 4, "f32", False, True, False),        # fp32 x, no renormalisation
    (1000, 256, 32, 6, "bf16", True, True, True),
    (4096, 2048, 8, 2, "bf16", True, False, False),      # the default workload's shape
    (300, 64, 16, 2, "f32", True, False, False),
    (148, 256, 1, 1, "bf16", True, False, False),       # one expert; one token per block
    (445, 128, 4, 4, "bf16", False, True, False),        # k = E, four tokens per block
    (20, 128, 32, 32, "bf16", True, True, True),         # k = E = 32: every lane selects
])
def test_fused_route_dispatch_matches_stage_calls(T, D, E, k, xdt, renorm, logits, shared):
    """moe_route_dispatch as one cooperative launch gives the bits of moe_route +
    moe_preprocess + moe_dispatch_permute (routing, weights, logits, counts, offsets,
    splits, rows, x_perm) and the same layer output."""
    wl = BASE.with_(T=T, D=D, E=E, ep_size=2 if E % 2 == 0 else 1, top_k=k, F=128, x_dtype=xdt,
                    renormalize=renorm, n_shared=1 if shared else 0, F_shared=128 if shared else 0,
                    seed=7)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp, keep_logits=logits)
    layer.allocate(T)
    assert M.moe_route_dispatch_is_fused(layer.config(T))
    keys = ["topk_idx", "topk_w", "counts", "expert_offsets", "rank_splits", "rank_offsets", "pos",
            "src", "x_perm", "out"] + (["logits"] if logits else [])
    res = {}
    for fused in ("0", "1"):
        os.environ["MOE_ROUTE_FUSED"] = fused
        try:
            for key in keys:
                layer.buf[key].fill_(-3)
            layer.forward(inp["x"])
            torch.cuda.synchronize()
            layer.check_status()
        finally:
            del os.environ["MOE_ROUTE_FUSED"]
        res[fused] = {key: layer.buf[key].clone() for key in keys}
    for key in keys:
        assert torch.equal(res["0"][key], res["1"][key]), key
    ref = oracle_route(wl, inp)
    compare_routing(res["1"]["topk_idx"].cpu().numpy(), res["1"]["topk_w"].cpu().numpy(), ref)


@pytest.mark.parametrize("k", [2, 6])
def test_long_batch_grid_stride(k):
    """More tokens than the dispatch grid's 65535-block cap (two rows per block for k <= 4,
    one for k = 6): the grid-stride loops of the stage kernels, the fused launch's
    ~950 tokens per block, and the combine's capped grid.  Stage calls and the fused launch
    give the same bits; routing for every token and the layer on sampled tokens against
    the oracle."""
    T = 140001
    wl = BASE.with_(T=T, D=64, E=8, ep_size=2, top_k=k, F=128, seed=13)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    layer.allocate(T)
    keys = ["topk_idx", "topk_w", "pos", "src", "x_perm", "out"]
    res = {}
    for fused in ("0", "1"):
        os.environ["MOE_ROUTE_FUSED"] = fused
        try:
            for key in keys:
                layer.buf[key].fill_(-3)
            layer.forward(inp["x"])
            torch.cuda.synchronize()
            layer.check_status()
        finally:
            del os.environ["MOE_ROUTE_FUSED"]
        res[fused] = {key: layer.buf[key].clone() for key in keys}
    for key in keys:
        assert torch.equal(res["0"][key], res["1"][key]), key
    ref = oracle_route(wl, inp)
    compare_routing(res["1"]["topk_idx"].cpu().numpy(), res["1"]["topk_w"].cpu().numpy(), ref)
    tokens = np.unique(np.concatenate([np.arange(4), [65534, 65535, 65536, 131069, 131070, 131071],
                                       np.random.default_rng(2).choice(T, 300, replace=False),
                                       [T - 2, T - 1]]))
    part = oracle_layer(wl, inp, tokens)
    got = f64(res["1"]["out"][torch.from_numpy(tokens).cuda()])
    assert_layer_close(got, part["out"], f64(inp["x"][torch.from_numpy(tokens).cuda()]))


@pytest.mark.parametrize("k,D,shared", [(1, 704, False), (2, 320, True), (2, 1600, False),
                                        (3, 576, True), (4, 1088, False), (5, 512, True),
                                        (6, 320, True), (7, 512, False), (8, 1088, True)])
def test_combine_forms_agree(k, D, shared):
    """The combine that loads every routed row of a step before its multiply-adds (U
    column chunks per row: 4 for k = 1, 2 for k <= 4, 1 above) gives the bits of the
    slot-by-slot form, and the layer matches the oracle (D not a multiple of 256 * U: a
    ragged last step)."""
    wl = BASE.with_(T=333, D=D, E=16, ep_size=4, top_k=k, F=128,
                    n_shared=1 if shared else 0, F_shared=128 if shared else 0, seed=4)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    outs = []
    for form in ("0", "1"):
        os.environ["MOE_PERMUTE_V"] = form
        try:
            outs.append(layer.forward(inp["x"]).clone())
            torch.cuda.synchronize()
        finally:
            del os.environ["MOE_PERMUTE_V"]
    layer.check_status()
    assert torch.equal(outs[0], outs[1])
    res = oracle_layer(wl, inp)
    assert_layer_close(f64(outs[1]), res["out"], f64(inp["x"]))


def test_ties_go_to_the_lower_index():
    wl = BASE.with_(T=512, E=8, top_k=2)
    inp = W.make_inputs(wl, device="cuda")
    wr = inp["w_router"]
    wr[6] = wr[1]           # experts 1 and 6 always tie exactly on the device
    layer = make_layer(wl, inp, keep_logits=True)
    layer.forward(inp["x"])
    torch.cuda.synchronize()
    idx = layer.buf["topk_idx"].cpu().numpy()
    logits = layer.buf["logits"].cpu().numpy()
    assert np.array_equal(logits[:, 1], logits[:, 6])
    for row in idx:
        r = row.tolist()
        if 6 in r:
            assert 1 in r and r.index(1) < r.index(6)


def test_worked_example_on_gpu():
    g = read_golden("worked_example.txt")
    E, k, ep = g["num_experts"][0], g["top_k"][0], g["num_devices"][0]
    D, F = 64, 128
    e_a, e_b = g["chosen_experts"]
    wa, wb = g["routing_weights"]
    x = torch.zeros((1, D), dtype=torch.float32)
    x[0, 0] = 1.0
    w_r = torch.zeros((E, D), dtype=torch.float32)
    w_r[:, 0] = -10.0
    w_r[e_a, 0] = math.log(wa / wb)
    w_r[e_b, 0] = 0.0
    w1 = torch.zeros((E, D, F))
    w2 = torch.zeros((E, F, D))
    for e in range(E):
        w1[e, 0, e], w1[e, 0, 64 + e] = 1.0, -1.0
        w2[e, e, 1] = w2[e, 64 + e, 2] = (e + 1) / 16.0
    layer = M.MoELayer(D=D, E=E, ep_size=ep, top_k=k, F=F, w_router=w_r.cuda(),
                       w_gate_up=w1.to(torch.bfloat16).cuda(), w_down=w2.to(torch.bfloat16).cuda(),
                       act="gelu", x_dtype="f32")
    out = layer.forward(x.cuda())
    torch.cuda.synchronize()
    b = layer.buf
    assert b["topk_idx"].cpu().tolist() == [g["chosen_experts"]]
    assert np.allclose(b["topk_w"].cpu().numpy()[0], g["routing_weights"], atol=1e-6)
    ro = b["rank_offsets"].cpu().numpy()
    for j, dev in enumerate(g["device_of_chosen"]):
        assert ro[dev] <= int(b["pos"][j]) < ro[dev + 1]
    phi1 = 0.5 * (1 + math.erf(1 / math.sqrt(2)))
    sa, sb = (e_a + 1) / 16, (e_b + 1) / 16
    expect = np.zeros(D)
    expect[0] = 1.0
    expect[1] = wa * sa * phi1 + wb * sb * phi1
    expect[2] = -(wa * sa * (1 - phi1) + wb * sb * (1 - phi1))
    assert np.allclose(out.cpu().numpy()[0], expect, rtol=1e-2, atol=2e-3)


def test_out_of_range_index_sets_status():
    wl = BASE.with_(T=64)
    cfg = M.make_config(wl.T, wl.D, wl.E, wl.ep_size, wl.top_k, wl.F)
    idx = torch.zeros((wl.T, wl.top_k), dtype=torch.int32, device="cuda")
    idx[:, 1] = 1
    idx[10, 1] = 8                       # outside [0, E)
    i32 = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    ws = torch.zeros(M.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    status = i32(1)
    M.moe_preprocess(cfg, idx, i32(wl.E), i32(wl.E + 1), i32(wl.ep_size), i32(wl.ep_size + 1),
                     i32(wl.R), i32(wl.R), ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == M.MOE_ERR_INDEX_OOB


def test_bounded_wait_reports_timeout():
    """A grid-barrier wait that nothing completes runs out (~1 s), the kernel records
    MOE_ERR_TIMEOUT in the status word and returns; the context stays usable (a forward
    afterwards still matches the oracle)."""
    bar = torch.zeros(2, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_check_wait_timeout(bar, status)
    torch.cuda.synchronize()
    assert int(status.item()) == M.MOE_ERR_TIMEOUT
    run_and_compare(BASE.with_(T=64, seed=21))


def test_empty_batch_forward():
    wl = BASE.with_(T=0)
    inp = W.make_inputs(BASE, device="cuda")
    layer = make_layer(BASE, inp)
    layer.forward(inp["x"][:0])
    torch.cuda.synchronize()
    assert int(layer.buf["counts"].sum().item()) == 0


def test_deterministic():
    wl = BASE.with_(T=1000, E=16, ep_size=4, top_k=4)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    a = layer.forward(inp["x"]).clone()
    b = layer.forward(inp["x"]).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("T", [100, 700])
def test_cta_pair_and_single_cta_gemm_agree(T, monkeypatch):
    """The 256x256 CTA-pair tiles and the one-CTA 128x256 tiles both match the
    oracle (ragged expert ends inside a 256-row tile, shared experts included)."""
    wl = BASE.with_(T=T, D=512, E=16, ep_size=4, top_k=3, F=384, n_shared=1, F_shared=256, seed=T)
    inp = W.make_inputs(wl, device="cuda")
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MOE_GEMM_CTA_PAIR", flag)
        layer = make_layer(wl, inp)
        outs.append(layer.forward(inp["x"]).clone())
        torch.cuda.synchronize()
        layer.check_status()
    res = oracle_layer(wl, inp)
    for o in outs:
        assert_layer_close(f64(o), res["out"], f64(inp["x"]))
    d = (outs[0].float() - outs[1].float()).abs().max().item()
    assert d <= 2 ** -6 * outs[1].float().abs().max().item()


@pytest.mark.parametrize("E,k", [(8, 2), (64, 6), (256, 8)])
def test_ties_on_the_tensor_core_router(E, k):
    """Exact ties through the filter-and-refine path: duplicated router rows give
    identical exact logits, and the lower index must come first."""
    wl = BASE.with_(T=300, D=256, E=E, ep_size=8 if E % 8 == 0 else 1, top_k=k, F=128)
    inp = W.make_inputs(wl, device="cuda")
    wr = inp["w_router"]
    wr[E - 1] = wr[0]
    wr[E // 2] = wr[1]
    layer = make_layer(wl, inp)                # no logits returned: tensor-core router
    layer.forward(inp["x"])
    torch.cuda.synchronize()
    idx = layer.buf["topk_idx"].cpu().numpy()
    for a_, b_ in ((0, E - 1), (1, E // 2)):
        for row in idx:
            r = row.tolist()
            if b_ in r:
                assert a_ in r and r.index(a_) < r.index(b_)
    ref = oracle_route(wl, inp)
    compare_routing(idx, layer.buf["topk_w"].cpu().numpy(), ref, max_exempt=None)   # exact ties


@pytest.mark.parametrize("T,D,E,k,xdt,zipf", [(32, 2048, 64, 6, "bf16", True),
                                               (40, 1024, 48, 4, "bf16", False),
                                               (100, 512, 256, 8, "bf16", False),
                                               (7, 7168, 256, 8, "bf16", False),
                                               (32, 1024, 64, 2, "f32", False)])
def test_split_k_router(T, D, E, k, xdt, zipf):
    """Few tokens and more than 32 experts: the logits kernel splits D across blocks
    (fp64 slice totals added in order before the single rounding).  Routing against
    the oracle with and without returned logits, and against the unsplit paths
    (tensor-core filter + refine, or the unsplit SIMT kernel)."""
    wl = BASE.with_(T=T, D=D, E=E, ep_size=8 if E % 8 == 0 else 1, top_k=k, F=128, x_dtype=xdt,
                    zipf_bias=zipf)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    b = layer.allocate(T)
    cfg = layer.config(T)
    ref = oracle_route(wl, inp)
    runs = []
    for split in ("1", "0"):
        os.environ["MOE_ROUTE_SPLIT"] = split
        try:
            for keep in (True, False):
                b["logits"] = torch.full((T, E), float("nan"), device="cuda") if keep else None
                M.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], b["logits"], b["topk_idx"],
                            b["topk_w"], b["workspace"])
                torch.cuda.synchronize()
                if keep:
                    assert np.allclose(b["logits"].cpu().numpy(), ref["logits"], rtol=2e-6, atol=2e-6)
                idx, w = b["topk_idx"].cpu().numpy(), b["topk_w"].cpu().numpy()
                compare_routing(idx, w, ref)
                runs.append(idx)
        finally:
            del os.environ["MOE_ROUTE_SPLIT"]
    for r in runs[1:]:
        assert np.array_equal(r, runs[0])


# per-expert row counts around the 128- and 256-row tile edges: empty, one row, a
# last tile with <= 64 rows (only the first CTA of a pair holds rows), 65..128 rows
# (both CTAs of an M = 128 pair tile), 129..255, exactly 256, 256 + a few (1, 32,
# 33, 64, 128, 129 rows; after two full tiles; in the second band of an expert of
# nine full tiles)
UNEVEN_COUNTS = [0, 1, 64, 65, 100, 128, 129, 200, 256, 257, 320, 384, 385, 115, 0, 3,
                 288, 289, 529, 2344]


@pytest.mark.parametrize("act,extra", [("swiglu", []), ("gelu", []), ("swiglu", [47, 0, 0, 0]),
                                       ("swiglu", [134, 0, 0, 0])])
def test_uneven_expert_tiles(act, extra):
    """Every routed row (and every shared-expert token) of the expert FFN stage
    against the oracle, with hand-set expert sizes that put the last M tile of
    each expert in every tiling case of both GEMM kernels (groups of <= 64 rows run
    as skinny tiles).  The shared expert runs over all T tokens: T = 5857 leaves
    225 rows in its last 256-row band, T + 47 leaves 16 and T + 134 leaves 103
    (M = 128 tiles, the first with rows in one CTA only)."""
    counts = np.array(UNEVEN_COUNTS + extra)
    E, T = counts.size, int(counts.sum())            # top-1: one row per token
    shared = act == "swiglu"
    wl = BASE.with_(T=T, D=256, E=E, ep_size=4, top_k=1, F=256, act=act,
                    n_shared=1 if shared else 0, F_shared=256 if shared else 0)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    b = layer.allocate(T)
    cfg = layer.config(T)
    # token t goes to the expert whose block of the (shuffled) assignment holds t
    rng = np.random.default_rng(11)
    assign = rng.permutation(np.repeat(np.arange(E), counts)).astype(np.int32)
    idx = torch.from_numpy(assign.reshape(T, 1)).cuda()
    b["status"].zero_()
    M.moe_preprocess(cfg, idx, b["counts"], b["expert_offsets"], b["rank_splits"],
                     b["rank_offsets"], b["pos"], b["src"], b["workspace"], b["status"])
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    x_perm = torch.randn((T, wl.D), generator=g, device="cuda").to(torch.bfloat16)
    x_bf = inp["x"].to(torch.bfloat16) if shared else None
    # CTA-pair kernel with skinny tiles and folded remainders (257..288-row last bands as
    # one tile; the remainder as one M = 256 product, then as two M = 128 products),
    # without folding, without skinny tiles, then the one-CTA kernel
    for pair, skinny, fold, f256 in (("1", "1", "1", "1"), ("1", "1", "1", "0"), ("1", "1", "0", "1"),
                                     ("1", "0", "1", "1"), ("0", "1", "1", "1")):
        os.environ["MOE_GEMM_CTA_PAIR"] = pair
        os.environ["MOE_GEMM_SKINNY"] = skinny
        os.environ["MOE_GEMM_FOLD"] = fold
        os.environ["MOE_GEMM_FOLD256"] = f256
        try:
            b["y_perm"].zero_()
            M.moe_expert_ffn(cfg, x_perm, x_bf, b["expert_offsets"], layer.packed, b["act"],
                             b["y_perm"], b["shared_out"], b["workspace"], b["status"])
            torch.cuda.synchronize()
        finally:
            del os.environ["MOE_GEMM_CTA_PAIR"]
            del os.environ["MOE_GEMM_SKINNY"]
            del os.environ["MOE_GEMM_FOLD"]
            del os.environ["MOE_GEMM_FOLD256"]
        assert int(b["status"].item()) == 0
        off = b["expert_offsets"].cpu().numpy()
        assert np.array_equal(np.diff(off), counts)
        wup = up_weights(wl, inp)
        xp, yp = f64(x_perm), f64(b["y_perm"])
        for e in range(E):
            lo, hi = int(off[e]), int(off[e + 1])
            if hi == lo:
                continue
            ref = oracle.expert_ffn(xp[lo:hi], f64(wup[e]), f64(inp["w_down"][e]), act)
            assert_layer_close(yp[lo:hi], ref, np.zeros_like(ref), f"y_perm expert {e} ({hi - lo} rows)")
        if shared:
            s_ref = oracle.shared_experts(f64(x_bf), f64(inp["ws_gate_up"]), f64(inp["ws_down"]))
            assert_layer_close(f64(b["shared_out"]), s_ref, np.zeros_like(s_ref), "shared_out")


@pytest.mark.parametrize("T", [700, 1400])
def test_fused_and_separate_ffn_launches_agree(monkeypatch, T):
    """The single persistent launch (gate_up, shared gate_up, down, shared down with
    band dependencies) gives the same bits as one launch per GEMM, and both match
    the oracle (ragged expert ends and a partial last band of the shared expert; with
    1400 tokens most experts hold 257..320 rows, so their down tiles wait on folded
    gate_up tiles)."""
    wl = BASE.with_(T=T, D=512, E=16, ep_size=4, top_k=3, F=512, n_shared=2, F_shared=256, seed=9)
    inp = W.make_inputs(wl, device="cuda")
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MOE_GEMM_FUSED", flag)
        layer = make_layer(wl, inp)
        outs.append(layer.forward(inp["x"]).clone())
        torch.cuda.synchronize()
        layer.check_status()
    assert torch.equal(outs[0], outs[1])
    res = oracle_layer(wl, inp)
    assert_layer_close(f64(outs[0]), res["out"], f64(inp["x"]))
