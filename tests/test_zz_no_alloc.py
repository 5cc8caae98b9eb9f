"""moe_preprocess_noalloc: the preprocess stage for callers that cannot allocate
device memory (a plugin whose host framework owns all device memory, or a loop
where a cudaMalloc and its implicit device synchronisation are not acceptable).
Its scratch lives in a fixed device array inside libmoe.so instead of a caller
workspace; its outputs must equal moe_preprocess's, bit for bit, call after call.

This file sorts last so a run that stops at the first failure has run every other
test before it; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import expert_dispatch_fp32_b200 as M
import moe_workloads as W
import oracle

KEYS = ("counts", "expert_offsets", "rank_splits", "rank_offsets", "pos", "src")


def _buffers(wl):
    i32 = lambda n: torch.full((n,), -7, dtype=torch.int32, device="cuda")
    return dict(counts=i32(wl.E), expert_offsets=i32(wl.E + 1), rank_splits=i32(wl.ep_size),
                rank_offsets=i32(wl.ep_size + 1), pos=i32(wl.R), src=i32(wl.R),
                status=torch.zeros(1, dtype=torch.int32, device="cuda"))


def _topk_for(wl, seed):
    # routing of a seeded batch, decided by the oracle (an input, not a product output)
    inp = W.make_inputs(wl.with_(seed=seed), device="cpu")
    x = inp["x"].to(torch.float64).numpy()
    logits = oracle.router_logits(x, inp["w_router"].numpy(),
                                  None if inp["bias"] is None else inp["bias"].numpy())
    idx, _ = oracle.topk_select(logits, wl.top_k)
    return torch.from_numpy(idx).cuda()


@pytest.mark.gpu
def test_noalloc_preprocess_matches_workspace_preprocess_twice():
    wl = W.get("zipf_skew_e64").with_(T=3000, D=128, F=128, F_shared=128)
    cfg = M.make_config(wl.T, wl.D, wl.E, wl.ep_size, wl.top_k, wl.F, n_shared=wl.n_shared,
                        F_shared=wl.F_shared)
    ws = torch.empty(M.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    for call, seed in enumerate((11, 12)):          # two calls in a row share the scratch
        idx = _topk_for(wl, seed)
        ref, got = _buffers(wl), _buffers(wl)
        M.moe_preprocess(cfg, idx, ref["counts"], ref["expert_offsets"], ref["rank_splits"],
                         ref["rank_offsets"], ref["pos"], ref["src"], ws, ref["status"])
        M.moe_preprocess_noalloc(cfg, idx, got["counts"], got["expert_offsets"], got["rank_splits"],
                                 got["rank_offsets"], got["pos"], got["src"], got["status"])
        torch.cuda.synchronize()
        assert int(got["status"].item()) == 0 and int(ref["status"].item()) == 0
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), (call, key)
        assert int(got["counts"].sum().item()) == wl.R
        # and against the oracle's definition of the same bookkeeping
        pre = oracle.preprocess(idx.cpu().numpy(), wl.E, wl.ep_size)
        for key in KEYS:
            assert np.array_equal(got[key].cpu().numpy(), pre[key]), (call, key)


@pytest.mark.gpu
def test_noalloc_rejects_configs_beyond_its_scratch():
    # 2048 tokens x top-8 over 1024 experts: 64 histogram blocks x 1024 experts plus two
    # barrier words need 65 538 int32, two more than the 65 536 the scratch holds.  Real
    # buffers of the right sizes, so nothing would fault even if a launch were enqueued.
    wl = W.Workload(name="wide", T=2048, D=64, E=1024, ep_size=8, top_k=8, F=128)
    cfg = M.make_config(wl.T, wl.D, wl.E, wl.ep_size, wl.top_k, wl.F)
    idx = torch.zeros((wl.T, wl.top_k), dtype=torch.int32, device="cuda")
    got = _buffers(wl)
    st = M.lib().moe_preprocess_noalloc(
        ctypes.byref(cfg), idx.data_ptr(), got["counts"].data_ptr(), got["expert_offsets"].data_ptr(),
        got["rank_splits"].data_ptr(), got["rank_offsets"].data_ptr(), got["pos"].data_ptr(),
        got["src"].data_ptr(), got["status"].data_ptr(), None)
    assert st == M.MOE_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert int(got["counts"][0].item()) == -7          # nothing was written
    # just under the limit: 2016 tokens -> 63 histogram blocks -> 64 514 int32
    wl2 = wl.with_(T=2016)
    cfg2 = M.make_config(wl2.T, wl2.D, wl2.E, wl2.ep_size, wl2.top_k, wl2.F)
    g = torch.Generator(device="cpu").manual_seed(5)
    idx2 = torch.rand((wl2.T, wl2.E), generator=g).argsort(dim=1)[:, :wl2.top_k]
    idx2 = idx2.to(torch.int32).contiguous().cuda()       # k distinct experts per token
    got2 = _buffers(wl2)
    M.moe_preprocess_noalloc(cfg2, idx2, got2["counts"], got2["expert_offsets"], got2["rank_splits"],
                             got2["rank_offsets"], got2["pos"], got2["src"], got2["status"])
    torch.cuda.synchronize()
    assert int(got2["status"].item()) == 0
    pre = oracle.preprocess(idx2.cpu().numpy(), wl2.E, wl2.ep_size)
    for key in KEYS:
        assert np.array_equal(got2[key].cpu().numpy(), pre[key]), key
