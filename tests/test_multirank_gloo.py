"""The N > 1 bench path on CPU: two gloo ranks join the group the way torchrun
describes it, take the max of their step times and aggregate whole-job tokens/s;
the reference arm's non-zero ranks exit without work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(WORLD_SIZE=str(ws), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup("gloo")
    my_ms = 10.0 + 2.0 * r                 # rank 1 is the slower one
    bench.barrier(w)
    m = bench.max_over_ranks(my_ms, w, device="cpu")
    v = bench.replica_value(4096, w, 20, m)
    q.put((r, w, m, v))
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, m, v in res:
        assert w == 2 and m == 12.0
        assert v == pytest.approx(4096 * 2 * 20 / 0.012)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "worked_example_t64", "--steps", "2", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_tokens_override():
    """--tokens runs the workload's shapes at another token count and names it so."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "worked_example_t64", "--tokens", "9", "--steps", "1",
                        "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["config"]["workload"] == "worked_example_t64_t9" and line["config"]["T"] == 9
    assert line["value"] > 0


def test_streamed_oracle_inputs_match_the_full_arrays():
    """bench.py's CPU baseline fetches one expert's weights at a time (so a 256-expert
    layer never needs its float64 weights at once); the oracle's output must be the
    same as with the full weight arrays."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import bench
    import moe_workloads as W
    import oracle
    wl = W.get("zipf_skew_e64").with_(T=48, D=128, F=128, F_shared=128)
    inp = W.make_inputs(wl)
    host = bench.HostOracleInputs(wl, inp)
    f = lambda t: t.to(torch.float64).numpy()
    kw = dict(E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, act=wl.act, renormalize=True)
    full = oracle.moe_layer(host.x, host.w_router, host.bias, f(inp["w_gate_up"]), f(inp["w_down"]),
                            host.ws_up, host.ws_down, **kw)
    streamed = oracle.moe_layer(host.x, host.w_router, host.bias, None, None, host.ws_up, host.ws_down,
                                expert_weights=host.expert, **kw)
    assert np.array_equal(full["out"], streamed["out"])
    assert bench.cpu_oracle_time(wl, host, 20, seed=3) > 0


def test_reference_arm_experts_override():
    """--experts runs a reduced expert count (profiling cases) and names it so."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "worked_example_t64", "--experts", "8", "--tokens", "16",
                        "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["config"]["workload"] == "worked_example_t64_t16_e8" and line["config"]["E"] == 8
