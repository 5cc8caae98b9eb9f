"""The expert-parallel layer's GPU stage operations (libmoe.so) on one rank: with a
one-rank NCCL group the exchanges are real all_to_all_single calls, and the
output must equal the one-GPU forward bit for bit (same rows, same kernels)."""
import datetime
import os
import socket

import pytest
import torch

import expert_dispatch_fp32_b200 as M
import moe_workloads as W
from expert_dispatch_fp32_b200.ep import EPMoELayer, GpuOps
from parity_helpers import make_layer

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def one_rank_group():
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda:0"))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("wl", [
    W.Workload(name="ep_small", T=333, D=256, E=8, ep_size=1, top_k=2, F=256),
    W.Workload(name="ep_shared", T=300, D=512, E=16, ep_size=1, top_k=4, F=256, n_shared=2, F_shared=128),
])
def test_ep_one_rank_equals_forward(wl, one_rank_group):
    inp = W.make_inputs(wl, device="cuda")
    ref_layer = make_layer(wl, inp)
    ref = ref_layer.forward(inp["x"]).clone()
    ops = GpuOps(D=wl.D, E=wl.E, ep_size=1, top_k=wl.top_k, F=wl.F, w_router=inp["w_router"],
                 w_gate_up_local=inp["w_gate_up"], w_down_local=inp["w_down"],
                 expert_bias=inp["bias"], ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"])
    out = EPMoELayer(ops).forward(inp["x"])
    torch.cuda.synchronize()
    ops.check()
    ref_layer.check_status()
    assert torch.equal(out, ref)


def test_gather_rows_and_local_ids():
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    src = torch.randn((50, 64), generator=g, device="cuda").to(torch.bfloat16)
    idx = torch.randperm(50, device="cuda").to(torch.int32)
    idx[7] = 50                                    # out of range: row left unwritten
    dst = torch.zeros((50, 64), dtype=torch.bfloat16, device="cuda")
    M.moe_gather_rows(src, idx, dst, 50, 50, 64)
    torch.cuda.synchronize()
    keep = torch.ones(50, dtype=torch.bool, device="cuda")
    keep[7] = False
    assert torch.equal(dst[keep], src[idx[keep].long()])
    assert torch.count_nonzero(dst[7]) == 0
    cfg = M.make_config(10, 64, 16, 4, 2, 128)
    topk = torch.randint(0, 16, (10, 2), device="cuda", dtype=torch.int32)
    srcp = torch.randperm(20, device="cuda").to(torch.int32)
    ids = torch.empty(20, dtype=torch.int32, device="cuda")
    M.moe_ep_local_ids(cfg, topk, srcp, ids)
    torch.cuda.synchronize()
    assert torch.equal(ids, (topk.view(-1)[srcp.long()] % 4).to(torch.int32))
