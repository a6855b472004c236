"""Token-sharded backward (flarepp_cp_merge_ex, flarepp_cp_bwd_stage) on one GPU.

G ranks are emulated in one process: the forward's sharded passes are run
for every shard and their triples laid back to back as the all-gather would
lay them; then each of the four backward stages runs on every shard, and
between stages the regions the stage leaves are summed over the shards and
written back into every shard's state, as the all-reduce would.  The shards'
dk0, dk, dv together and every shard's dq0, dq_fixed, dgate must match the
fp64 gradient oracle on the whole sequence (the sharded backward is exact up
to rounding).  The orchestration module runs here with one rank."""
import numpy as np
import pytest
import torch

from oracle.backward import flarepp_backward
from parity import assert_dgate_parity, assert_grad_parity, to64
from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu


def emulate_bwd(x, dy, G, gated, layout="bhnd", path=0, norm=False):
    from rank_latent_attention_mixer_b200 import binding as b
    from rank_latent_attention_mixer_b200.cp import shard_bounds
    d = {k: t.cuda() for k, t in x.items()}
    dyc = dy.cuda()
    B, H, N, D = d["k"].shape
    M = d["q_fixed"].shape[1]
    dt = b._dtype_code(d["k"])
    tl = (lambda t: t) if layout == "bhnd" else (lambda t: t.transpose(1, 2).contiguous())
    back = (lambda t: t) if layout == "bhnd" else (lambda t: t.transpose(1, 2))
    shards = [shard_bounds(N, G, r) for r in range(G)]
    sl = lambda t, lo, hi: tl(t[:, :, lo:hi].contiguous())
    T = b.cp_triple_bytes(B, H, M, D) // 4
    L = b.cp_latent_bytes(B, H, M, D, dt)
    common = dict(B=B, H=H, M=M, D=D)
    f32 = dict(dtype=torch.float32, device="cuda")

    def gathered(q, q_shared, kk, vv, nrm=False):
        out = torch.empty(G * T, **f32)
        for r, (lo, hi) in enumerate(shards):
            kr = sl(kk, lo, hi)
            vr = kr if vv is kk else sl(vv, lo, hi)
            b.cp_partials(q, q_shared, kr, vr, out[r * T:(r + 1) * T], N=hi - lo, path=path, layout=layout,
                          norm_synthesis=nrm, **common)
        return out

    lse_enc = torch.empty((B, H, M), **f32)
    lse_syn = qdyn = qs = None
    if gated:
        lse_syn = torch.empty((B, H, M), **f32)
        qdyn = torch.empty((B, H, M, D), **f32)
        qs = torch.empty(L, dtype=torch.uint8, device="cuda")
        b.cp_merge(gathered(d["q0"], True, d["k0"], d["k0"], norm), G, d["q_fixed"], d["gate"], qs, dtype=dt,
                   lse_out=lse_syn, pregate_out=qdyn, **common)
        tg = gathered(qs, False, d["k"], d["v"])
    else:
        tg = gathered(d["q_fixed"], True, d["k"], d["v"])
    zs = torch.empty(L, dtype=torch.uint8, device="cuda")
    b.cp_merge(tg, G, None, None, zs, dtype=dt, lse_out=lse_enc, **common)

    ranks = []
    for lo, hi in shards:
        n = hi - lo
        tok = {name: sl(d[name], lo, hi) for name in ("k0", "k", "v")}
        tok["dy"] = sl(dyc, lo, hi)
        g = {"dk": torch.empty_like(tok["k"]), "dv": torch.empty_like(tok["v"]),
             "dq_fixed": torch.empty((H, M, D), **f32)}
        if gated:
            g.update(dk0=torch.empty_like(tok["k0"]), dq0=torch.empty((H, M, D), **f32),
                     dgate=torch.empty((H,), **f32))
        lay = b.cp_bwd_layout(B, H, n, M, D, dt, path=path, layout=layout, norm_synthesis=norm)
        ranks.append(dict(n=n, tok=tok, g=g, lay=lay, state=torch.zeros(lay.bytes, dtype=torch.uint8, device="cuda")))
    for stage in (1, 2, 3, 4):
        for rk in ranks:
            t = rk["tok"]
            b.cp_bwd_stage(stage, d["q0"], d["q_fixed"], d["gate"] if gated else None, qs, zs, lse_syn, lse_enc,
                           qdyn, t["k0"], t["k"], t["v"], t["dy"], rk["g"], rk["state"], N=rk["n"], path=path,
                           layout=layout, norm_synthesis=norm, **common)
        if stage < 4:
            regions = []
            for rk in ranks:
                off, nb = rk["lay"].reduce_offset[stage - 1], rk["lay"].reduce_bytes[stage - 1]
                regions.append(rk["state"][off:off + nb].view(torch.float32))
            total = torch.stack(regions).sum(0)
            for reg in regions:
                reg.copy_(total)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    out = {}
    for name in ("dk0", "dk", "dv"):
        if name in ranks[0]["g"]:
            out[name] = torch.cat([back(rk["g"][name]) for rk in ranks], dim=2)
    for name in ("dq0", "dq_fixed", "dgate"):
        if name in ranks[0]["g"]:
            out[name] = ranks[0]["g"][name]
            for rk in ranks[1:]:
                assert torch.equal(rk["g"][name], out[name]), f"{name} differs between ranks"
    return out


CASES = [(1, True, "bf16", "bhnd", 0, False), (2, True, "bf16", "bhnd", 0, False), (3, True, "bf16", "bnhd", 0, False),
         (3, False, "bf16", "bhnd", 0, False), (2, True, "f32", "bhnd", 0, False), (3, True, "f16", "bhnd", 0, True),
         (2, True, "bf16", "bhnd", 1, False), (2, False, "f32", "bnhd", 0, False), (8, True, "bf16", "bhnd", 0, True)]


@pytest.mark.parametrize("G,gated,dt,layout,path,norm", CASES,
                         ids=[f"G{c[0]}-{'gated' if c[1] else 'flare'}-{c[2]}-{c[3]}-p{c[4]}{'-norm' if c[5] else ''}"
                              for c in CASES])
def test_sharded_backward_matches_oracle(G, gated, dt, layout, path, norm):
    x = W.random_inputs(2, 2, 1777, 96, 64 if dt != "f32" else 32, dtype=dt, seed=41 + G)
    B, H, N, D = x["k"].shape
    dy = W.random_cotangent((B, H, N, D), dt, seed=141 + G)
    g = emulate_bwd(x, dy, G, gated, layout=layout, path=path, norm=norm)
    ref = flarepp_backward(to64(x["q0"]), to64(x["q_fixed"]), np.zeros(H) if not gated else to64(x["gate"]),
                           to64(x["k0"]), to64(x["k"]), to64(x["v"]), to64(dy), norm_synthesis=norm)
    for name in (("dq0", "dq_fixed", "dk0", "dk", "dv") if gated else ("dq_fixed", "dk", "dv")):
        assert_grad_parity(g[name], ref[name], dt, f"{name} (G={G})")
    if gated:
        assert_dgate_parity(g["dgate"], ref, dt)


def test_orchestration_one_rank_matches_single_gpu_backward():
    """cp.mixer_bwd_cp with one rank (no process group) against flarepp_mixer_bwd."""
    from rank_latent_attention_mixer_b200 import binding as b
    from rank_latent_attention_mixer_b200.cp import mixer_bwd_cp
    x = W.random_inputs(1, 2, 1500, 80, 64, dtype="bf16", seed=47)
    dy = W.random_cotangent((1, 2, 1500, 64), "bf16", seed=147)
    d = {k: t.cuda() for k, t in x.items()}
    args = (d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], dy.cuda())
    g_cp = mixer_bwd_cp(*args)
    g = b.mixer_bwd(*args)
    torch.cuda.synchronize()
    ref = flarepp_backward(*(to64(t) for t in (x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], dy)))
    for name in ("dq0", "dq_fixed", "dk0", "dk", "dv"):
        assert_grad_parity(g_cp[name], ref[name], "bf16", name)
        diff = float((g_cp[name].double() - g[name].double()).abs().max())
        assert diff <= 2e-2 * float(g[name].double().abs().max()), (name, diff)
    assert_dgate_parity(g_cp["dgate"], ref, "bf16")
