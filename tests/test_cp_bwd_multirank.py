"""Token-sharded backward (rank_latent_attention_mixer_b200/cp.py,
mixer_bwd_cp) on gloo ranks (CPU).  The ranks run the real orchestration --
the forward's sharded passes with their all-gathers, then the four backward
stages with an all-reduce of the stage's state region after each of the
first three -- with the library stages replaced by fp64 stand-ins of the same
buffer layouts (each stand-in stage sums over this rank's tokens only, as the
library does).  The shards' dk0, dk, dv together and every rank's dq0,
dq_fixed, dgate must equal the fp64 gradient oracle's on the whole sequence
(the sharded backward is exact up to rounding)."""
import math
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from test_cp_multirank import ROOT, LOG2E, StandInOps, _free_port


class _Layout:
    def __init__(self, latd):
        self.bytes = 4 * latd * 4
        self.reduce_offset = [0, 2 * latd * 4, 3 * latd * 4]
        self.reduce_bytes = [2 * latd * 4, latd * 4, latd * 4]


class StandInBwdOps(StandInOps):
    """fp64 stand-ins for flarepp_cp_merge_ex, flarepp_cp_bwd_layout and
    flarepp_cp_bwd_stage.  The state is fp32 [dq_dec, dz | dq_enc | dq0 per
    batch element]; values a stage keeps for a later stage of the same rank
    (dk_dec, dz, dq) live in a dict keyed by the state."""

    def __init__(self):
        self.keep = {}

    def cp_merge(self, gathered, ranks, q_fixed, gate, state, *, B, H, M, D, dtype, lse_out=None,
                 pregate_out=None):
        n = B * H * M * D
        parts = gathered.view(ranks, -1).double()
        O = parts[:, :n].reshape(ranks, B, H, M, D)
        ml = parts[:, n:].reshape(ranks, B, H, M, 2)
        mstar = ml[..., 0].max(dim=0).values
        w = torch.pow(2.0, ml[..., 0] - mstar)
        Lsum = (w * ml[..., 1]).sum(0)
        out = (w[..., None] * O).sum(0) / Lsum[..., None]
        if lse_out is not None:
            lse_out.copy_((mstar + torch.log2(Lsum)).float())
        if gate is not None:
            if pregate_out is not None:
                pregate_out.copy_(out.float())
            out = q_fixed.double() + gate.double().view(H, 1, 1) * out
        state.view(torch.float32)[:n] = out.reshape(-1).float()

    def cp_bwd_layout(self, B, H, N, M, D, dtype, **kw):
        return _Layout(B * H * M * D)

    def cp_bwd_stage(self, stage, q0, q_fixed, gate, q_state, z_state, lse_syn, lse_enc, qdyn, k0, k, v, dy, grads,
                     state, *, B, H, N, M, D, path, scale, force_chunks, layout, norm_synthesis):
        s = scale or 1.0 / math.sqrt(D)
        latd = B * H * M * D
        st = state.view(torch.float32)
        keep = self.keep.setdefault(state.data_ptr(), {})
        gated = gate is not None
        Q = self._lat(q_state if gated else q_fixed, not gated, B, H, M, D)
        Z = self._lat(z_state, False, B, H, M, D)
        K, V, dY = self._tok(k, layout), self._tok(v, layout), self._tok(dy, layout)
        lat = lambda t: t.reshape(B, H, M, D)
        if stage == 1:
            P = torch.softmax(K @ Q.transpose(-1, -2) * s, dim=-1)            # [B,H,N,M], over the latents
            delta = (dY * (P @ Z)).sum(-1, keepdim=True)
            dS = P * (dY @ Z.transpose(-1, -2) - delta)
            keep["dk_dec"] = s * dS @ Q
            st[:latd] = (s * dS.transpose(-1, -2) @ K).reshape(-1).float()   # this rank's dq_dec
            st[latd:2 * latd] = (P.transpose(-1, -2) @ dY).reshape(-1).float()   # this rank's dz
        elif stage == 2:
            dz = lat(st[latd:2 * latd].double())
            keep["dq"] = lat(st[:latd].double())
            delta = (dz * Z).sum(-1, keepdim=True)
            P = torch.pow(2.0, (Q @ K.transpose(-1, -2)) * s * LOG2E - lse_enc.double()[..., None])
            dS = P * (dz @ V.transpose(-1, -2) - delta)                      # [B,H,M,N]
            dk = keep["dk_dec"] + s * dS.transpose(-1, -2) @ Q
            dv = P.transpose(-1, -2) @ dz
            for name, t in (("dk", dk), ("dv", dv)):
                grads[name].copy_(t if layout == "bhnd" else t.transpose(1, 2))
            st[2 * latd:3 * latd] = (s * dS @ K).reshape(-1).float()         # this rank's dq_enc
        elif stage == 3:
            dq = keep["dq"] + lat(st[2 * latd:3 * latd].double())
            keep["dq"] = dq
            if gated:
                K0 = self._tok(k0, layout)
                Q0 = q0.double().expand(B, H, M, D)
                qd = qdyn.double()
                dqd = gate.double().view(1, H, 1, 1) * dq
                delta = (dqd * qd).sum(-1, keepdim=True)
                P = torch.pow(2.0, (Q0 @ K0.transpose(-1, -2)) * s * LOG2E - lse_syn.double()[..., None])
                dS = P * (dqd @ K0.transpose(-1, -2) - delta)
                dk0 = s * dS.transpose(-1, -2) @ Q0 + P.transpose(-1, -2) @ dqd
                grads["dk0"].copy_(dk0 if layout == "bhnd" else dk0.transpose(1, 2))
                st[3 * latd:] = (s * dS @ K0).reshape(-1).float()            # this rank's dq0 per batch element
        else:
            dq = keep["dq"]
            grads["dq_fixed"].copy_(dq.sum(0))
            if gated:
                grads["dq0"].copy_(lat(st[3 * latd:].double()).sum(0))
                grads["dgate"].copy_((dq * qdyn.double()).sum(dim=(0, 2, 3)))


def _worker(rank, world, port, gated, layout, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from rank_latent_attention_mixer_b200 import cp
    from rank_latent_attention_mixer_b200 import workloads as W
    x = W.random_inputs(2, 3, 301, 20, 16, dtype="f32", seed=13)
    dy = W.random_cotangent((2, 3, 301, 16), "f32", seed=113)
    lo, hi = cp.shard_bounds(301, world, rank)
    sl = lambda t: (t[:, :, lo:hi] if layout == "bhnd" else t[:, :, lo:hi].transpose(1, 2)).contiguous()
    g = cp.mixer_bwd_cp(x["q0"], x["q_fixed"], x["gate"] if gated else None, sl(x["k0"]), sl(x["k"]), sl(x["v"]),
                        sl(dy), layout=layout, _ops=StandInBwdOps())
    back = (lambda t: t) if layout == "bhnd" else (lambda t: t.transpose(1, 2))
    q.put((rank, {name: (back(t) if t.dim() == 4 else t).numpy().astype(np.float64) for name, t in g.items()}))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,gated,layout", [(2, True, "bhnd"), (3, True, "bnhd"), (2, False, "bhnd")])
def test_sharded_backward_matches_oracle(world, gated, layout):
    sys.path.insert(0, ROOT)
    from oracle.backward import flarepp_backward
    from rank_latent_attention_mixer_b200 import workloads as W
    x = W.random_inputs(2, 3, 301, 20, 16, dtype="f32", seed=13)
    dy = W.random_cotangent((2, 3, 301, 16), "f32", seed=113)
    gate = x["gate"].numpy().astype(np.float64) if gated else np.zeros(3)
    ref = flarepp_backward(x["q0"].numpy(), x["q_fixed"].numpy(), gate, x["k0"].numpy(), x["k"].numpy(),
                           x["v"].numpy(), dy.numpy())
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
    tol = lambda o: 1e-5 * max(1.0, np.abs(o).max())
    for name in (("dk0", "dk", "dv") if gated else ("dk", "dv")):
        got = np.concatenate([o[1][name] for o in out], axis=2)
        assert np.abs(got - ref[name]).max() < tol(ref[name]), name
    for name in (("dq0", "dq_fixed", "dgate") if gated else ("dq_fixed",)):
        for _, g in out:                                   # the same on every rank
            assert np.abs(g[name] - ref[name]).max() < tol(ref[name]), name
