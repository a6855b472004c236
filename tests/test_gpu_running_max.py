"""Scores that rise from one key/value tile to the next.

The online softmax of the tcgen05 kernels keeps a running row maximum and only
rescales when a tile's maximum exceeds it by more than 8 log2 units (fp16 I/O
takes the weights against the maximum minus 7, so they stay below 2^15).  These
inputs make later tiles exceed it by a few units, by 8 to 120 units and by far
more (where exponentials against the old maximum would overflow fp32), in the
synthesis, encode and decode passes, with bf16 and fp16 I/O; the result is
compared with the fp64 oracle.  The softmax is the one of scaled dot-product
attention (FLARE++ mixer, encode/decode equations).
"""
import math

import pytest
import torch

import oracle
from parity import assert_parity

pytestmark = pytest.mark.gpu

KT = 128          # key/value tile of the split passes
DEC_KT = 64       # latent tile of the decode pass


def structured(kind, B, H, N, M, D, seed, dtype="bf16"):
    """Latents q0 = q_fixed ~ (1 + m/16) * ones, tokens k0 = k ~ b(n) * ones/8,
    small noise, so that a score is about (1 + m/16) * b(n) * sqrt(D)/8 and
    rises along n (split passes) and along m (decode)."""
    g = torch.Generator().manual_seed(seed)
    n = torch.arange(N, dtype=torch.float64)
    if kind == "ramp":
        b = 10.0 * n / KT
    else:  # one jump after three tiles
        b = torch.where(n < 3 * KT, torch.zeros_like(n), torch.full_like(n, 70.0))
    lat = (1.0 + torch.arange(M, dtype=torch.float64) / 16.0)[:, None].expand(M, D)
    noise = lambda *s: 0.05 * torch.randn(*s, generator=g, dtype=torch.float64)
    io = torch.float16 if dtype == "f16" else torch.bfloat16
    q0 = (lat[None] + noise(H, M, D)).to(io)
    q_fixed = (lat[None] + noise(H, M, D)).to(io)
    tok = (b[:, None] / 8.0).expand(N, D)
    k0 = (tok[None, None] + noise(B, H, N, D)).to(io)
    k = (tok[None, None] + noise(B, H, N, D)).to(io)
    v = torch.randn(B, H, N, D, generator=g, dtype=torch.float64).to(io)
    gate = torch.full((H,), 0.5, dtype=torch.float32)
    return dict(q0=q0, q_fixed=q_fixed, gate=gate, k0=k0, k=k, v=v)


def lags(q, keys, tile, stride):
    """Per query row and tile: how far (log2 units) the tile's maximum score
    exceeds the maximum over the earlier tiles the same warpgroup saw."""
    D = q.shape[-1]
    s = (q.double() @ keys.double().T) / math.sqrt(D) * (1.0 / math.log(2.0))
    T = (s.shape[1] + tile - 1) // tile
    tmax = torch.stack([s[:, t * tile:(t + 1) * tile].max(dim=1).values for t in range(T)], dim=1)
    out = []
    for first in range(stride):
        run = tmax[:, first]
        for t in range(first + stride, T, stride):
            out.append(tmax[:, t] - run)
            run = torch.maximum(run, tmax[:, t])
    return torch.cat(out)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("kind", ["ramp", "jump"])
@pytest.mark.parametrize("M", [128, 256])
def test_lagging_running_max(kind, M, dtype):
    B, H, N, D = 1, 2, 1000, 64
    x = structured(kind, B, H, N, M, D, seed=M + len(kind), dtype=dtype)
    # the inputs reach every case of the check in the synthesis pass (one
    # chunk: an item spans all tiles; M <= 128 gives the warpgroups every
    # other tile)
    lag = lags(x["q0"][0], x["k0"][0, 0], KT, 2 if M <= 128 else 1)
    assert bool(((lag > 8) & (lag <= 120)).any()) and bool((lag > 120).any())

    from rank_latent_attention_mixer_b200 import binding as bnd
    d = {k: t.cuda() for k, t in x.items()}
    for flare in (False, True):
        y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], None if flare else x["gate"],
                                             x["k0"], x["k"], x["v"], flare=flare)
        if flare:
            # decode scores rise along the latents of each token
            dl = lags(x["k"][0, 0], x["q_fixed"][0], DEC_KT, 1)
            assert bool((dl > 120).any())
            assert kind == "jump" or bool(((dl > 8) & (dl <= 120)).any())
        for fc in (0, 1):
            y, q, z = bnd.mixer_fwd(d["q0"], d["q_fixed"], None if flare else d["gate"], d["k0"], d["k"],
                                    d["v"], return_qz=True, path=2, force_chunks=fc)
            torch.cuda.synchronize()
            assert bnd.check_device_status() == 0
            tag = f"{kind} M={M} flare={flare} chunks={fc} {dtype}"
            assert_parity(z, z_ref, dtype, "z " + tag)
            assert_parity(q, q_ref, dtype, "q " + tag)
            assert_parity(y, y_ref, dtype, "y " + tag)
