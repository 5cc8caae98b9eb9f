"""The multi-rank expert-parallel forward on CPU ranks (gloo): two ranks, each with
its own tokens and half of the experts, exchange rows with all_to_all_single and
must produce, per rank, the single-process layer output on that rank's tokens.

The stage operations here are a CPU stand-in written from the oracle (this file
is test code); the layer logic under test — count exchange, split sizes, the two
token all-to-alls, the per-row local-expert ids and the return order — is
expert_dispatch_fp32_b200.ep.EPMoELayer, the same code the GPU ranks run with
GpuOps.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

T, D, E, K, F, S, FS = 37, 16, 8, 3, 12, 1, 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _weights(seed=0):
    g = np.random.default_rng(seed)
    return dict(w_router=g.normal(0, 0.3, (E, D)).astype(np.float32),
                w_up=g.normal(0, 0.2, (E, D, 2 * F)), w_down=g.normal(0, 0.2, (E, F, D)),
                ws_up=g.normal(0, 0.2, (S, D, 2 * FS)), ws_down=g.normal(0, 0.2, (S, FS, D)))


def _tokens(rank):
    return np.random.default_rng(100 + rank).normal(0, 1, (T - 5 * rank, D))


class CpuOps:
    """Oracle-backed stage operations of one rank (float64 rows)."""

    def __init__(self, wts, rank, ep):
        import oracle
        self.o, self.w, self.rank, self.ep, self.E, self.El, self.k = oracle, wts, rank, ep, E, E // ep, K
        lo = rank * self.El
        self.w_up_local = wts["w_up"][lo:lo + self.El]
        self.w_down_local = wts["w_down"][lo:lo + self.El]

    def route_and_preprocess(self, x):
        xn = x.numpy()
        logits = self.o.router_logits(xn, self.w["w_router"], None)
        idx, w = self.o.topk_select(logits, self.k, True)
        pre = self.o.preprocess(idx, self.E, self.ep)
        st = {k_: torch.from_numpy(np.ascontiguousarray(v)) for k_, v in pre.items()}
        st["counts"] = st["counts"].to(torch.int64)
        st["splits"] = st["rank_splits"].to(torch.int64)
        st["idx"], st["w"] = idx, w
        return st

    def dispatch(self, x, st):
        src = st["src"].numpy().astype(np.int64)
        x_perm = torch.from_numpy(self.o.permute(x.numpy(), src, self.k))
        ids = torch.from_numpy((st["idx"].reshape(-1)[src] % self.El).astype(np.int64))
        return x_perm, ids

    def local_experts(self, x_recv, ids_recv):
        xr, ids = x_recv.numpy(), ids_recv.numpy()
        y = np.zeros_like(xr)
        for e in range(self.El):
            m = ids == e
            if m.any():
                y[m] = self.o.expert_ffn(xr[m], self.w_up_local[e], self.w_down_local[e], "swiglu")
        return torch.from_numpy(y)

    def shared_and_combine(self, x, st, y_back):
        xn = x.numpy()
        n = xn.shape[0]
        y_tok = self.o.unpermute(y_back.numpy(), st["pos"].numpy().astype(np.int64), n, self.k)
        sh = self.o.shared_experts(xn, self.w["ws_up"], self.w["ws_down"])
        return torch.from_numpy(self.o.combine(y_tok, st["w"], xn, sh))


def _rank_main(rank, ws, port, q):
    os.environ.update(WORLD_SIZE=str(ws), RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    from expert_dispatch_fp32_b200.ep import EPMoELayer
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        wts = _weights()
        layer = EPMoELayer(CpuOps(wts, rank, ws))
        x = torch.from_numpy(_tokens(rank))
        out = layer.forward(x).numpy()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_rank_expert_parallel_matches_single_process():
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wts = _weights()
    for r in range(2):
        x = _tokens(r)
        ref = oracle.moe_layer(x, wts["w_router"], None, wts["w_up"], wts["w_down"], wts["ws_up"],
                               wts["ws_down"], E=E, ep_size=2, top_k=K, act="swiglu")["out"]
        assert res[r].shape == ref.shape
        assert np.allclose(res[r], ref, rtol=1e-12, atol=1e-12)


def test_ep_layer_rejects_a_group_of_the_wrong_size():
    from expert_dispatch_fp32_b200.ep import EPMoELayer

    class Two:
        ep = 2
    with pytest.raises(ValueError):
        EPMoELayer(Two())             # no process group: one rank
