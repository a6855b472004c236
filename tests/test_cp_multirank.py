"""Token-sharded forward (rank_latent_attention_mixer_b200/cp.py) on gloo ranks
(CPU).  The ranks run the real orchestration -- shard bounds, the two
all-gathers of latent-sized triples, the merges, the local decode -- with the
library stages replaced by fp64 stand-ins of the same buffer layouts, and the
shards' outputs together must equal the fp64 oracle's (physicsnemo issue
#2024, section 2: the sharded encoder is exact up to rounding)."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LOG2E = 1.0 / math.log(2.0)


class StandInOps:
    """fp64 stand-ins for flarepp_cp_partials / _merge / _decode: triple = O
    rows [B,H,M,D] then (max in log2 units, sum) [B,H,M,2]; a latent state is
    its fp32 rows [B,H,M,D]."""

    @staticmethod
    def cp_triple_bytes(B, H, M, D):
        return B * H * M * (D + 2) * 4

    @staticmethod
    def cp_latent_bytes(B, H, M, D, dtype):
        return B * H * M * D * 4

    @staticmethod
    def _lat(q, shared, B, H, M, D):
        if shared:
            return q.double().expand(B, H, M, D)
        return q.view(torch.float32)[: B * H * M * D].view(B, H, M, D).double()

    @staticmethod
    def _tok(t, layout):
        return t.double() if layout == "bhnd" else t.double().transpose(1, 2)

    def cp_partials(self, q, q_shared, k, v, triple, *, B, H, N, M, D, path, scale, layout, force_chunks,
                    norm_synthesis=False):
        Q = self._lat(q, q_shared, B, H, M, D)
        K, V = self._tok(k, layout), self._tok(v, layout)
        S = Q @ K.transpose(-1, -2) * (scale or 1.0 / math.sqrt(D))
        m = S.max(dim=-1, keepdim=True).values
        P = torch.exp(S - m)
        O = P @ V
        n = B * H * M * D
        triple[:n] = O.reshape(-1).float()
        triple[n:] = torch.stack([m[..., 0] * LOG2E, P.sum(-1)], dim=-1).reshape(-1).float()

    def cp_merge(self, gathered, ranks, q_fixed, gate, state, *, B, H, M, D, dtype):
        n = B * H * M * D
        parts = gathered.view(ranks, -1).double()
        O = parts[:, :n].reshape(ranks, B, H, M, D)
        ml = parts[:, n:].reshape(ranks, B, H, M, 2)
        mstar = ml[..., 0].max(dim=0).values
        w = torch.pow(2.0, ml[..., 0] - mstar)
        out = (w[..., None] * O).sum(0) / (w * ml[..., 1]).sum(0)[..., None]
        if gate is not None:
            out = q_fixed.double() + gate.double().view(H, 1, 1) * out
        state.view(torch.float32)[:n] = out.reshape(-1).float()

    def cp_decode(self, q, q_shared, z_state, k, y, *, B, H, N, M, D, path, scale, layout):
        Q = self._lat(q, q_shared, B, H, M, D)
        Z = self._lat(z_state, False, B, H, M, D)
        K = self._tok(k, layout)
        S = K @ Q.transpose(-1, -2) * (scale or 1.0 / math.sqrt(D))
        out = torch.softmax(S, dim=-1) @ Z
        y.copy_(out if layout == "bhnd" else out.transpose(1, 2))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, gated, layout, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from rank_latent_attention_mixer_b200 import cp
    from rank_latent_attention_mixer_b200 import workloads as W
    x = W.random_inputs(2, 3, 301, 20, 16, dtype="f32", seed=11)
    lo, hi = cp.shard_bounds(301, world, rank)
    sl = lambda t: (t[:, :, lo:hi] if layout == "bhnd" else t[:, :, lo:hi].transpose(1, 2)).contiguous()
    y, qm, zm = cp.mixer_fwd_cp(x["q0"], x["q_fixed"], x["gate"] if gated else None, sl(x["k0"]), sl(x["k"]),
                                sl(x["v"]), layout=layout, return_qz=True, _ops=StandInOps())
    if layout == "bnhd":
        y = y.transpose(1, 2)
    q.put((rank, lo, hi, y.numpy().astype(np.float64), qm.numpy().astype(np.float64),
           zm.numpy().astype(np.float64)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,gated,layout", [(2, True, "bhnd"), (3, True, "bnhd"), (2, False, "bhnd")])
def test_sharded_forward_matches_oracle(world, gated, layout):
    sys.path.insert(0, ROOT)
    import oracle
    from rank_latent_attention_mixer_b200 import workloads as W
    x = W.random_inputs(2, 3, 301, 20, 16, dtype="f32", seed=11)
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"] if gated else None, x["k0"], x["k"],
                                         x["v"], flare=not gated)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, gated, layout, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == sorted(o[1] for o in out) and out[-1][2] == 301
    y = np.concatenate([o[3] for o in out], axis=2)
    for r, lo, hi, _, qm, zm in out:
        assert np.abs(qm - q_ref).max() < 1e-5 * max(1.0, np.abs(q_ref).max())     # same q and z on every rank
        assert np.abs(zm - z_ref).max() < 1e-5 * max(1.0, np.abs(z_ref).max())
    assert np.abs(y - y_ref).max() < 1e-5 * max(1.0, np.abs(y_ref).max())


def test_shard_bounds():
    sys.path.insert(0, ROOT)
    from rank_latent_attention_mixer_b200 import cp
    for N, G in [(301, 2), (301, 3), (8, 8), (1048576, 8), (10, 3)]:
        b = [cp.shard_bounds(N, G, r) for r in range(G)]
        assert b[0][0] == 0 and b[-1][1] == N
        assert all(b[i][1] == b[i + 1][0] for i in range(G - 1))
        sizes = [hi - lo for lo, hi in b]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        cp.shard_bounds(2, 3, 0)
