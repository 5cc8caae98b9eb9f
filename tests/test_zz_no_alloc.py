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


@pytest.mark.gpu
def test_noalloc_rejects_configs_beyond_its_scratch():
    cfg = M.make_config(1 << 20, 64, 1024, 8, 8, 128)      # 8192 blocks x 1024 experts
    st = M.lib().moe_preprocess_noalloc(ctypes.byref(cfg), *([1 << 20] * 8), None)
    assert st == M.MOE_ERR_SCRATCH_LIMIT
