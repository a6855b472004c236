"""Host-side multi-rank logic of bench.py on 2 gloo ranks (CPU): the maximum
over ranks of the elapsed time, per-rank seeds (independent problems, weak
scaling) and the whole-job throughput."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from rank_latent_attention_mixer_b200 import workloads as W
    r, w, lr = bench.dist_env()
    local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
    mx = bench.reduce_max(local_ms, w)
    seed = bench.rank_seed(W.WORKLOADS["grid85_bf16"].seed, r)
    x = W.make_inputs(W.WORKLOADS["tiny_f32"].with_shape(seed=seed))
    dist.barrier()
    q.put((r, w, lr, mx, seed, float(x["k"].sum())))
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, mx0, s0, k0), (r1, w1, l1, mx1, s1, k1) = out
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    assert mx0 == mx1 == 15.0                         # both ranks see the slowest rank's time
    assert s0 != s1 and k0 != k1                      # independent problems per rank


def test_aggregate_throughput():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 1M tokens x 10 steps in 20 ms -> 1048.576 Mtokens/s
    assert bench.aggregate_mtokens(1048576, 2, 10, 20.0) == pytest.approx(1048.576)
    assert bench.reduce_max(3.5, 1) == 3.5
