"""Token-sharded stages (flarepp_cp_partials / _merge / _decode) on one GPU.

G ranks are emulated in one process, one after the other: every shard's
triple is computed, the triples are laid back to back as the all-gather would
lay them, merged, and every shard decoded.  The shards' y together must match
the fp64 oracle at the workload tolerance, and q, z must match the oracle's
(physicsnemo issue #2024, section 2: the sharded encoder is exact up to
rounding).  The orchestration module (cp.py) runs here with one rank."""
import pytest
import torch

import oracle
from parity import assert_parity, metrics
from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu


def emulate(x, G, gated, layout="bhnd", path=0):
    from rank_latent_attention_mixer_b200 import binding as b
    from rank_latent_attention_mixer_b200.cp import shard_bounds
    d = {k: t.cuda() for k, t in x.items()}
    B, H, N, D = d["k"].shape
    M = d["q_fixed"].shape[1]
    dt = b._dtype_code(d["k"])
    tl = (lambda t: t) if layout == "bhnd" else (lambda t: t.transpose(1, 2).contiguous())
    shards = [shard_bounds(N, G, r) for r in range(G)]
    sl = lambda t, lo, hi: tl(t[:, :, lo:hi].contiguous())
    T = b.cp_triple_bytes(B, H, M, D) // 4
    L = b.cp_latent_bytes(B, H, M, D, dt)
    common = dict(B=B, H=H, M=M, D=D)

    def gathered(q, q_shared, kk, vv):
        out = torch.empty(G * T, dtype=torch.float32, device="cuda")
        for r, (lo, hi) in enumerate(shards):
            kr = sl(kk, lo, hi)
            vr = kr if vv is kk else sl(vv, lo, hi)
            b.cp_partials(q, q_shared, kr, vr, out[r * T:(r + 1) * T], N=hi - lo, path=path, layout=layout,
                          **common)
        return out

    if gated:
        qs = torch.empty(L, dtype=torch.uint8, device="cuda")
        b.cp_merge(gathered(d["q0"], True, d["k0"], d["k0"]), G, d["q_fixed"], d["gate"], qs, dtype=dt, **common)
        tg = gathered(qs, False, d["k"], d["v"])
    else:
        tg = gathered(d["q_fixed"], True, d["k"], d["v"])
    zs = torch.empty(L, dtype=torch.uint8, device="cuda")
    b.cp_merge(tg, G, None, None, zs, dtype=dt, **common)
    ys = []
    for lo, hi in shards:
        kr = sl(d["k"], lo, hi)
        yr = torch.empty_like(kr)
        b.cp_decode(qs if gated else d["q_fixed"], not gated, zs, kr, yr, N=hi - lo, path=path, layout=layout,
                    **common)
        ys.append(yr if layout == "bhnd" else yr.transpose(1, 2))
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    n = B * H * M * D
    z = zs.view(torch.float32)[:n].view(B, H, M, D)
    q = qs.view(torch.float32)[:n].view(B, H, M, D) if gated else None
    return torch.cat(ys, dim=2), q, z


CASES = [
    # (B, H, N, M, D), dtype, path
    ((2, 4, 3001, 128, 32), "bf16", 0),
    ((1, 8, 5000, 256, 64), "f16", 0),
    ((2, 2, 1000, 64, 16), "f32", 0),
    ((1, 3, 2000, 100, 64), "bf16", 1),
    ((1, 4, 2000, 256, 128), "f16", 0),
]


@pytest.mark.parametrize("G", [1, 2, 3, 8])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{'x'.join(map(str, c[0]))}-{c[1]}-p{c[2]}")
def test_sharded_stages_match_oracle(case, G):
    (B, H, N, M, D), dtype, path = case
    x = W.random_inputs(B, H, N, M, D, dtype=dtype, seed=N + G)
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    y, q, z = emulate(x, G, gated=True, path=path)
    assert_parity(q, q_ref, dtype, f"q (G={G})")
    assert_parity(z, z_ref, dtype, f"z (G={G})")
    assert_parity(y, y_ref, dtype, f"y (G={G})")


@pytest.mark.parametrize("layout", ["bhnd", "bnhd"])
def test_sharded_closed_gate_and_layout(layout):
    x = W.random_inputs(2, 4, 2500, 128, 32, dtype="bf16", seed=3)
    y_ref, _, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], None, x["k0"], x["k"], x["v"], flare=True)
    y, _, z = emulate(x, 4, gated=False, layout=layout)
    assert_parity(z, z_ref, "bf16", "z (closed gate)")
    assert_parity(y, y_ref, "bf16", "y (closed gate)")
    y2, q2, z2 = emulate(x, 3, gated=True, layout=layout)
    y3, q3, z3 = emulate(x, 3, gated=True, layout="bhnd")
    assert torch.equal(y2, y3) and torch.equal(q2, q3) and torch.equal(z2, z3)


def test_cp_module_single_rank_equals_whole_call():
    from rank_latent_attention_mixer_b200 import binding as b
    from rank_latent_attention_mixer_b200.cp import mixer_fwd_cp
    x = W.random_inputs(1, 8, 4000, 256, 64, dtype="bf16", seed=9)
    d = {k: t.cuda() for k, t in x.items()}
    y, q, z = mixer_fwd_cp(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], return_qz=True)
    yw, qw, zw = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], return_qz=True)
    torch.cuda.synchronize()
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    assert_parity(y, y_ref, "bf16", "y (cp, 1 rank)")
    assert_parity(q, q_ref, "bf16", "q (cp, 1 rank)")
    # one rank reduces its chunks to a triple and merges it once more: the same
    # softmax as the whole call up to bf16 rounding of the weights
    assert metrics(y, yw)["rel_l2"] < 6e-3 and metrics(z, zw)["rel_l2"] < 6e-3
