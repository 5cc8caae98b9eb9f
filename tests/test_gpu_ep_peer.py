"""The expert-parallel forward with the exchange done by peer-memory stores.

P ranks' data on one GPU ("Expert Parallel (EP)", Communication Pattern steps 1-5):
each rank routes its own tokens, sends its counts and its rows straight into the
owning ranks' receive buffers (moe_ep_send_counts / moe_ep_send_rows), the owners
run their local experts on the rows as received, and the output rows go back to the
senders' dispatch rows (moe_ep_return_rows) for the ordinary combine.  Every rank's
output must equal moe_forward of its tokens over all E experts, bit for bit (the same
rows meet the same weights in the same K order), and the oracle on sampled tokens.
"""
import numpy as np
import pytest
import torch

import expert_dispatch_fp32_b200 as M
import moe_workloads as W
from expert_dispatch_fp32_b200.ep import PeerEPGroup, PeerEPRank
from parity_helpers import assert_layer_close, f64, make_layer, oracle_layer, up_weights

pytestmark = pytest.mark.gpu


def _group(wl, P, inp):
    return PeerEPGroup(D=wl.D, E=wl.E, P=P, top_k=wl.top_k, F=wl.F, T=wl.T,
                       w_router=inp["w_router"], w_gate_up=up_weights(wl, inp), w_down=inp["w_down"],
                       expert_bias=inp["bias"], ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"],
                       act=wl.act, renormalize=wl.renormalize, x_dtype=wl.x_dtype)


def _rank_batches(wl, P):
    return torch.stack([W.make_x(wl, device="cuda", seed=100 + r) for r in range(P)])


CASES = [
    # P ranks, workload: DeepSeek-like top-8 over 64 experts with a shared expert, a
    # Mixtral-like top-2 over 8, the worked example's 4 x 4 GELU experts with fp32 x,
    # and a skewed router whose high experts (and so whole ranks) receive no rows
    (2, W.Workload(name="ep_ds", T=384, D=256, E=64, ep_size=2, top_k=8, F=256, n_shared=1,
                   F_shared=256, seed=21)),
    (4, W.Workload(name="ep_ds4", T=200, D=512, E=64, ep_size=4, top_k=6, F=384, n_shared=2,
                   F_shared=128, seed=22)),
    (8, W.Workload(name="ep_mix", T=300, D=256, E=8, ep_size=8, top_k=2, F=512, seed=23)),
    (4, W.get("worked_example_t64")),
    (4, W.Workload(name="ep_skew", T=256, D=256, E=32, ep_size=4, top_k=4, F=256, zipf_bias=True,
                   n_shared=1, F_shared=256, seed=24)),
]


@pytest.mark.parametrize("P,wl", CASES, ids=[c[1].name + f"_p{c[0]}" for c in CASES])
def test_peer_exchange_equals_single_gpu_forward(P, wl):
    wl = wl.with_(ep_size=P)
    inp = W.make_inputs(wl, device="cuda")
    grp = _group(wl, P, inp)
    xs = _rank_batches(wl, P)
    if wl.x_dtype == "f32":
        xs = xs.float()
    layer = make_layer(wl, inp)
    for it in range(2):                      # two forwards: the second exchange's epoch differs
        out = grp.forward(xs).clone()
        torch.cuda.synchronize()
        grp.check_status()
        for r in range(P):
            ref = layer.forward(xs[r]).clone()
            torch.cuda.synchronize()
            layer.check_status()
            assert torch.equal(out[r], ref), (it, r)
    # every rank's rows really crossed: the receive layout holds all T*k*P rows
    assert int(grp.local_off[:, -1].sum().item()) == P * wl.T * wl.top_k
    # and the oracle on a sample of rank 1's tokens
    toks = np.arange(0, wl.T, max(1, wl.T // 24))
    inp1 = dict(inp, x=xs[1])
    res = oracle_layer(wl, inp1, toks)
    assert_layer_close(f64(out[1][torch.from_numpy(toks).cuda()]), res["out"],
                       f64(xs[1][torch.from_numpy(toks).cuda()]))


@pytest.mark.parametrize("fused", ["1", "0"])
def test_fused_and_separate_return_agree(fused, monkeypatch):
    """The local experts' down GEMM storing its rows straight into the senders' y_back
    (moe_ep_expert_ffn_return's default) and the FFN into y_recv followed by the return
    copy (MOE_EP_FUSED_RETURN=0) give the same bits, equal to moe_forward."""
    monkeypatch.setenv("MOE_EP_FUSED_RETURN", fused)
    P, wl = CASES[1]
    wl = wl.with_(ep_size=P)
    inp = W.make_inputs(wl, device="cuda")
    grp = _group(wl, P, inp)
    xs = _rank_batches(wl, P)
    layer = make_layer(wl, inp)
    out = grp.forward(xs).clone()
    torch.cuda.synchronize()
    grp.check_status()
    for r in range(P):
        assert torch.equal(out[r], layer.forward(xs[r])), r


def test_peer_exchange_wait_reports_timeout():
    """A wait for an exchange that never happened (a later epoch nobody signals) runs
    out after about a second and reports MOE_ERR_TIMEOUT; the context stays usable and
    the next forward is still exact."""
    P = 2
    wl = W.Workload(name="ep_to", T=64, D=128, E=8, ep_size=P, top_k=2, F=256, seed=25)
    inp = W.make_inputs(wl, device="cuda")
    grp = _group(wl, P, inp)
    xs = _rank_batches(wl, P)
    grp.forward(xs)
    torch.cuda.synchronize()
    grp.check_status()
    M.moe_ep_wait_returned(grp.tok_cfg, grp.peers, 0, P, grp.epoch + 7, grp.status)
    torch.cuda.synchronize()
    assert int(grp.status.item()) == M.MOE_ERR_TIMEOUT
    grp.status.zero_()
    out = grp.forward(xs).clone()
    torch.cuda.synchronize()
    grp.check_status()
    layer = make_layer(wl, inp)
    for r in range(P):
        assert torch.equal(out[r], layer.forward(xs[r]))


def test_per_process_rank_alone_equals_single_gpu_forward():
    """PeerEPRank, the one-process-per-GPU form, with no process group (one rank): its
    exchange calls cover rank 0 alone (rank0 = 0, nlocal = 1) through tables built
    from its own exchange allocation; two forwards (two epochs) equal moe_forward bit
    for bit.  Ranks on other GPUs would fill the other table entries with mappings
    of their allocations (tests/test_ep_ipc_gloo.py covers that setup on CPU ranks)."""
    wl = W.Workload(name="ep_rank1", T=384, D=256, E=16, ep_size=1, top_k=4, F=256, n_shared=1,
                    F_shared=256, seed=25)
    inp = W.make_inputs(wl, device="cuda")
    rank = PeerEPRank(D=wl.D, E=wl.E, top_k=wl.top_k, F=wl.F, T=wl.T, w_router=inp["w_router"],
                      w_gate_up_local=up_weights(wl, inp), w_down_local=inp["w_down"],
                      expert_bias=inp["bias"], ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"],
                      act=wl.act, renormalize=wl.renormalize, x_dtype=wl.x_dtype)
    layer = make_layer(wl, inp)
    x = W.make_x(wl, device="cuda", seed=7)
    for it in range(2):
        out = rank.forward(x).clone()
        torch.cuda.synchronize()
        rank.check_status()
        ref = layer.forward(x).clone()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), it
    assert int(rank.local_off[-1].item()) == wl.T * wl.top_k
    rank.close()


def test_ipc_export_reports_the_offset_in_the_allocation():
    """moe_ipc_export names the allocation that holds a buffer and the buffer's offset
    in it, so a peer maps the allocation once and adds the offset."""
    t = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    h0, o0 = M.moe_ipc_export(t)
    h1, o1 = M.moe_ipc_export(t[4096:])
    assert len(h0) == M.moe_ipc_handle_bytes() == 64
    assert h0 == h1 and o1 - o0 == 4096
