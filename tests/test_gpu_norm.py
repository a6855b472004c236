"""The synthesis normalisation (flarepp_options_t.norm_synthesis): q0 and k0
rows RMS-normalised inside the synthesis pass (physicsnemo issue #2024,
FLARE++ list, "Normalizing the synthesis call"), against the fp64 oracle with
the same normalisation, for both kernel families, every head dim, both
latent-tile modes and both token layouts."""
import pytest
import torch

import oracle
from parity import assert_parity, metrics
from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu


def raw_inputs(B, H, N, M, D, dtype, seed):
    """Seeds and synthesis keys far from RMS 1 (scaled, not normalised), so
    that the normalisation changes the result."""
    x = W.random_inputs(B, H, N, M, D, dtype=dtype, seed=seed, rms=False)
    for name, c in (("q0", 3.0), ("k0", 0.4)):
        x[name] = (x[name].double() * c).to(x[name].dtype)
    return x


CASES = [
    ((2, 3, 1000, 64, 32), "bf16", 0),       # interleaved latent tile
    ((1, 4, 3001, 256, 64), "bf16", 0),      # two latent tiles per item
    ((1, 2, 2000, 512, 64), "f16", 0),
    ((2, 2, 700, 100, 16), "bf16", 0),
    ((1, 2, 1500, 128, 128), "bf16", 0),
    ((1, 2, 800, 64, 32), "f32", 0),         # SIMT
    ((1, 2, 900, 130, 64), "bf16", 1),       # SIMT on 16-bit I/O
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{'x'.join(map(str, c[0]))}-{c[1]}-p{c[2]}")
def test_normalised_synthesis_matches_oracle(case):
    from rank_latent_attention_mixer_b200 import binding as b
    (B, H, N, M, D), dtype, path = case
    x = raw_inputs(B, H, N, M, D, dtype, seed=B + N + D)
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"],
                                         norm_synthesis=True)
    d = {k: t.cuda() for k, t in x.items()}
    y, q, z = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], return_qz=True, path=path,
                          norm_synthesis=True)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    assert_parity(q, q_ref, dtype, "q")
    assert_parity(z, z_ref, dtype, "z")
    assert_parity(y, y_ref, dtype, "y")
    # the normalisation matters for these inputs
    _, q_plain, _ = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    assert metrics(q_plain, q_ref)["rel_l2"] > 1e-2
    # and the [B,N,H,D] layout gives the same bits
    t = lambda a: a.transpose(1, 2).contiguous()
    yb = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"], t(d["k0"]), t(d["k"]), t(d["v"]), path=path,
                     layout="bnhd", norm_synthesis=True)
    torch.cuda.synchronize()
    assert torch.equal(yb.transpose(1, 2), y)


def test_normalised_synthesis_sharded():
    """The token-sharded stages with the normalisation in the synthesis call."""
    from rank_latent_attention_mixer_b200 import binding as b
    from rank_latent_attention_mixer_b200.cp import shard_bounds
    B, H, N, M, D = 1, 4, 3000, 128, 64
    x = raw_inputs(B, H, N, M, D, "bf16", seed=77)
    y_ref, q_ref, _ = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"],
                                     norm_synthesis=True)
    d = {k: t.cuda() for k, t in x.items()}
    G = 3
    T = b.cp_triple_bytes(B, H, M, D) // 4
    tg = torch.empty(G * T, dtype=torch.float32, device="cuda")
    for r in range(G):
        lo, hi = shard_bounds(N, G, r)
        kr = d["k0"][:, :, lo:hi].contiguous()
        b.cp_partials(d["q0"], True, kr, kr, tg[r * T:(r + 1) * T], B=B, H=H, N=hi - lo, M=M, D=D,
                      norm_synthesis=True)
    qs = torch.empty(b.cp_latent_bytes(B, H, M, D, b.BF16), dtype=torch.uint8, device="cuda")
    b.cp_merge(tg, G, d["q_fixed"], d["gate"], qs, B=B, H=H, M=M, D=D, dtype=b.BF16)
    torch.cuda.synchronize()
    q = qs.view(torch.float32)[:B * H * M * D].view(B, H, M, D)
    assert_parity(q, q_ref, "bf16", "q (sharded, normalised)")
