"""Host logic of the multi-rank benchmark, with 2 gloo ranks on CPU: ranks
share the weights, draw their own token batches, take the slowest rank's
time, and report all ranks' tokens over it (weak scaling, no collective on
the data path)."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from group_limited_routing_sigmoid_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.WORKLOADS["tiny"]
        weights = W.make_weights(wl, "cpu")
        g = torch.Generator(device="cpu")
        g.manual_seed(bench.token_seed(wl, rank))
        x = W.make_tokens(wl, "cpu", g)["x"]
        local_ms = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.whole_job_tokens_per_s(world, 4, wl.T, ms_max)
        out[rank] = (float(weights["router_w"].sum()), float(x.float().sum()), ms_max, value)
    finally:
        dist.destroy_process_group()


def test_two_rank_host_logic():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0]                      # same weights on every rank
    assert r0[1] != r1[1]                      # each rank its own tokens
    assert r0[2] == r1[2] == 15.0              # slowest rank's time on both
    assert r0[3] == r1[3] == 2 * 4 * 64 / 15e-3


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference` launched the way a multi-GPU run is: rank 0
    alone times the oracle and prints one JSON line; every rank exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--workload", "tiny"]
    res = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["config"]["workload"] == "beam_tiny"
