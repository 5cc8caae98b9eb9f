"""Host side of the one-process-per-GPU peer exchange (expert_dispatch_fp32_b200.ep:
PeerEPRank's setup), on CPU ranks over gloo.

Each rank exports its exchange allocation, the exports go round the process group, and
each rank builds its pointer tables: entry p of every table is rank p's buffer, i.e.
rank p's allocation (its own, or rank p's export mapped into this process) plus the
buffer's offset in the common layout.  The mapping calls are replaced by a stand-in
that records them (no GPU here); the exchange, the table order and the unmapping are
the code PeerEPRank runs.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from expert_dispatch_fp32_b200.ep import (  # noqa: E402
    EXCHANGE_BUFFERS, check_peer_devices, exchange_layout, gather_infos, peer_tables)


class FakeIpc:
    """Export: handle bytes naming the rank, offset 4096 * (rank + 1).  Import: a
    made-up address derived from the handle and offset.  Records every call."""

    def __init__(self, rank):
        self.rank, self.imported, self.closed = rank, [], []

    def export(self, base):
        return (f"alloc-of-rank-{self.rank}".encode().ljust(64, b"\0"), 4096 * (self.rank + 1))

    @staticmethod
    def address(handle, offset):
        src = int(handle.rstrip(b"\0").decode().rsplit("-", 1)[1])
        return (0x7F00 + src) << 32 | offset

    def import_(self, handle, offset):
        self.imported.append((bytes(handle), offset))
        return self.address(handle, offset)

    def close(self, ptr, offset):
        self.closed.append((ptr, offset))


def _own_base(rank):
    return (0x1000 + rank) << 32


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(WORLD_SIZE=str(ws), RANK=str(rank), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        ipc = FakeIpc(rank)
        offs, _, _ = exchange_layout(ws, 16, 64, 10, 2, ws * 10 * 2)
        info = {"host": "node0", "device": f"gpu-{rank}", "export": ipc.export(_own_base(rank))}
        infos = gather_infos(info)
        check_peer_devices(infos)
        tables, opened = peer_tables(rank, _own_base(rank), offs, infos, ipc)
        for ptr, off in opened:
            ipc.close(ptr, off)
        q.put((rank, tables, opened, ipc.imported, ipc.closed, offs, [i["device"] for i in infos]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 3])
def test_ranks_build_tables_of_each_others_buffers(ws):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        r, *rest = q.get(timeout=180)
        res[r] = rest
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(ws):
        tables, opened, imported, closed, offs, devices = res[r]
        assert devices == [f"gpu-{p}" for p in range(ws)]           # rank order
        peers = [p for p in range(ws) if p != r]
        # one mapping per other rank (never its own), each closed once
        assert [h.rstrip(b"\0").decode() for h, _ in imported] == [f"alloc-of-rank-{p}" for p in peers]
        assert [o for _, o in imported] == [4096 * (p + 1) for p in peers]
        assert sorted(closed) == sorted(opened) and len(opened) == ws - 1
        for name in EXCHANGE_BUFFERS:
            assert len(tables[name]) == ws
            for p in range(ws):
                base = _own_base(r) if p == r else FakeIpc.address(
                    f"alloc-of-rank-{p}".encode(), 4096 * (p + 1))
                assert tables[name][p] == base + offs[name], (r, name, p)


def test_exchange_layout_is_aligned_and_disjoint():
    P, E, D, T, k = 4, 64, 7168, 100, 8
    cap = P * T * min(k, E // P)
    offs, sizes, total = exchange_layout(P, E, D, T, k, cap)
    assert sizes == {"cnt": 4 * P * E, "flags": 12 * P, "recv_x": 2 * cap * D, "recv_src": 4 * cap,
                     "recv_rank": 4 * cap, "y_back": 2 * T * k * D}
    spans = sorted((offs[n], offs[n] + sizes[n]) for n in EXCHANGE_BUFFERS)
    assert all(o % 256 == 0 for o, _ in spans)
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= total and total % 256 == 0


def test_peer_devices_must_be_distinct_gpus_of_one_node():
    check_peer_devices([{"host": "a", "device": "u0"}, {"host": "a", "device": "u1"}])
    with pytest.raises(RuntimeError, match="share device"):
        check_peer_devices([{"host": "a", "device": "u0"}, {"host": "a", "device": "u0"}])
    with pytest.raises(RuntimeError, match="one node"):
        check_peer_devices([{"host": "a", "device": "u0"}, {"host": "b", "device": "u1"}])


def test_one_rank_maps_nothing():
    offs, _, _ = exchange_layout(1, 8, 64, 5, 2, 10)
    ipc = FakeIpc(0)
    tables, opened = peer_tables(0, _own_base(0), offs, [{"export": None}], ipc)
    assert opened == [] and ipc.imported == []
    assert all(tables[n] == [_own_base(0) + offs[n]] for n in EXCHANGE_BUFFERS)
