"""Backward of the mixer (flarepp_mixer_bwd) against the fp64 gradient oracle
(oracle/backward.py, itself pinned by central differences of the forward
oracle), through the C ABI on seeded inputs.

Covers every I/O dtype and head dim, ragged token and latent counts (several
shared-memory stages on both sides, tails), both forward kernel families for
the recomputed passes, the closed gate (FLARE), the scale option, both token
layouts, forced token-chunk counts, and determinism."""
import numpy as np
import pytest
import torch

from oracle.backward import flarepp_backward
from parity import assert_dgate_parity, assert_grad_parity, scale_factor, to64
from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
GRADS = ("dq0", "dq_fixed", "dk0", "dk", "dv")       # dgate: assert_dgate_parity
FLARE_GRADS = ("dq_fixed", "dk", "dv")


def binding():
    from rank_latent_attention_mixer_b200 import binding as b
    return b


def inputs(B, H, N, M, D, dt, seed):
    x = W.random_inputs(B, H, N, M, D, dtype=dt, seed=seed)
    dy = W.random_cotangent((B, H, N, D), dt, seed=seed + 100)
    return x, dy


def oracle_grads(x, dy, gate=None, scale=0.0, norm=False):
    g = x["gate"] if gate is None else gate
    return flarepp_backward(to64(x["q0"]), to64(x["q_fixed"]), to64(g), to64(x["k0"]), to64(x["k"]),
                            to64(x["v"]), to64(dy), scale=scale, norm_synthesis=norm)


def gpu_grads(x, dy, flare=False, **kw):
    b = binding()
    d = {k: v.to(DEV) for k, v in x.items()}
    g = b.mixer_bwd(d["q0"], d["q_fixed"], None if flare else d["gate"], d["k0"], d["k"], d["v"], dy.to(DEV), **kw)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    return g


CASES = [
    # (B, H, N, M, D, dtype, path): ragged N and M, several latent stages (M > 4096/D), every D
    ((1, 2, 1000, 48, 16, "f32"), 0),
    ((2, 1, 530, 70, 128, "f32"), 0),
    ((1, 2, 777, 300, 32, "f32"), 0),
    ((2, 2, 1500, 128, 64, "bf16"), 0),
    ((1, 2, 700, 64, 32, "bf16"), 0),
    ((1, 3, 1100, 200, 16, "bf16"), 0),
    ((1, 2, 650, 96, 128, "bf16"), 0),
    ((1, 2, 700, 96, 32, "f16"), 0),
    ((1, 2, 900, 80, 64, "bf16"), 1),     # the recomputed forward on the SIMT kernels (fp32 routing queries)
    ((1, 2, 600, 40, 64, "f16"), 1),
    ((2, 1, 520, 150, 128, "f16"), 0),    # fp16 on the tensor cores at the widest and narrowest head dims
    ((1, 2, 999, 33, 16, "f16"), 0),
    ((1, 1, 4100, 512, 64, "bf16"), 0),   # M = 512: both latent row groups, many token tiles
]


@pytest.mark.parametrize("case,path", CASES, ids=[f"{'x'.join(map(str, c[:5]))}-{c[5]}-p{p}" for c, p in CASES])
def test_backward_parity(case, path):
    B, H, N, M, D, dt = case
    x, dy = inputs(B, H, N, M, D, dt, seed=sum(case[:5]))
    ref = oracle_grads(x, dy)
    g = gpu_grads(x, dy, path=path)
    for name in GRADS:
        m = assert_grad_parity(g[name], ref[name], dt, name)
        print(case, path, name, {k: m[k] for k in ("rel_l2", "max_abs_rel_to_max") if k in m})
    assert_dgate_parity(g["dgate"], ref, dt)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_closed_gate_is_flare_backward(dt):
    """gate == NULL gives FLARE's gradients; they equal the gated mixer's at gate 0."""
    x, dy = inputs(2, 2, 900, 64, 32, dt, seed=5)
    ref = oracle_grads(x, dy, gate=np.zeros(2))
    g = gpu_grads(x, dy, flare=True)
    assert set(g) == set(FLARE_GRADS)
    for name in FLARE_GRADS:
        assert_grad_parity(g[name], ref[name], dt, name)
    gz = gpu_grads({**x, "gate": torch.zeros_like(x["gate"])}, dy)
    for name in FLARE_GRADS:
        assert torch.equal(g[name], gz[name]), f"{name}: closed gate and zero gate differ"
    assert torch.count_nonzero(gz["dq0"]) == 0 and torch.count_nonzero(gz["dk0"]) == 0
    assert_dgate_parity(gz["dgate"], ref, dt)


@pytest.mark.parametrize("dt,D", [("f32", 32), ("bf16", 32), ("bf16", 64), ("f16", 64)])
def test_scale_option(dt, D):
    """The FLARE block's printed scale=1.0 through the options, on the SIMT
    kernels (fp32) and the tensor-core kernels (bf16, fp16)."""
    x, dy = inputs(1, 2, 640, 40, D, dt, seed=11)
    ref = oracle_grads(x, dy, scale=1.0)
    g = gpu_grads(x, dy, scale=1.0)
    f = scale_factor(1.0, D)              # the bounds for a non-default scale (parity.py)
    for name in GRADS:
        assert_grad_parity(g[name], ref[name], dt, name, factor=f)
    assert_dgate_parity(g["dgate"], ref, dt, factor=f)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_token_layout_bnhd_identical(dt):
    x, dy = inputs(2, 3, 500, 50, 32, dt, seed=13)
    g = gpu_grads(x, dy)
    xt = {k: (v.transpose(1, 2).contiguous() if v.dim() == 4 else v) for k, v in x.items()}
    gt = gpu_grads(xt, dy.transpose(1, 2).contiguous(), layout="bnhd")
    for name in GRADS + ("dgate",):
        a = gt[name].transpose(1, 2) if gt[name].dim() == 4 else gt[name]
        assert torch.equal(a, g[name]), f"{name}: [B,N,H,D] layout differs from [B,H,N,D]"


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_chunk_invariance_and_determinism(dt):
    """The token sums split into chunks are exact up to rounding; repeated calls are bitwise equal."""
    x, dy = inputs(1, 2, 3000, 64, 64, dt, seed=17)
    ref = oracle_grads(x, dy)
    g_def = gpu_grads(x, dy)
    g_again = gpu_grads(x, dy)
    for name in GRADS + ("dgate",):
        assert torch.equal(g_def[name], g_again[name]), f"{name}: not deterministic"
    for chunks in (1, 2, 7):
        g = gpu_grads(x, dy, force_chunks=chunks)
        assert_dgate_parity(g["dgate"], ref, dt)
        for name in GRADS:
            assert_grad_parity(g[name], ref[name], dt, f"{name} (chunks={chunks})")
            diff = (g[name].double() - g_def[name].double()).abs().max().item()
            scale = g_def[name].double().abs().max().item()
            assert diff <= (1e-5 if dt == "f32" else 1e-2) * scale, (name, chunks, diff, scale)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_single_token_and_single_latent(dt):
    """N = 1: every softmax over tokens has one term (its gradients through P vanish);
    M = 1: the decode weight is 1, so dk gets no decode term."""
    for (N, M) in ((1, 8), (37, 1), (33, 129)):
        x, dy = inputs(1, 2, N, M, 16, dt, seed=N + M)
        ref = oracle_grads(x, dy)
        g = gpu_grads(x, dy)
        for name in GRADS:
            assert_grad_parity(g[name], ref[name], dt, f"{name} N={N} M={M}",
                               zero_atol=1e-5 if dt == "f32" else 1e-2)
        assert_dgate_parity(g["dgate"], ref, dt, zero_atol=1e-5 if dt == "f32" else 1e-2)


def test_caller_workspace():
    b = binding()
    x, dy = inputs(1, 2, 300, 32, 32, "bf16", seed=3)
    need = b.bwd_workspace_bytes(1, 2, 300, 32, 32, b.BF16)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    g1 = gpu_grads(x, dy, workspace=ws)
    g2 = gpu_grads(x, dy)
    for name in GRADS + ("dgate",):
        assert torch.equal(g1[name], g2[name])


@pytest.mark.parametrize("dt,path", [("f32", 0), ("bf16", 0), ("f16", 0), ("bf16", 1)])
def test_normalised_synthesis_backward(dt, path):
    """norm_synthesis: the synthesis reads RMS-normalised q0, k0 rows and dq0, dk0
    go through that step; rows scaled far from RMS 1 so the step matters."""
    x, dy = inputs(1, 2, 900, 80, 32, dt, seed=23)
    x["q0"] = (x["q0"].double() * 3.0).to(x["q0"].dtype)
    x["k0"] = (x["k0"].double() * 0.4).to(x["k0"].dtype)
    ref = oracle_grads(x, dy, norm=True)
    g = gpu_grads(x, dy, path=path, norm_synthesis=True)
    for name in GRADS:
        assert_grad_parity(g[name], ref[name], dt, name)
    assert_dgate_parity(g["dgate"], ref, dt)
    # and it differs from the gradient without the step
    plain = oracle_grads(x, dy)
    assert np.max(np.abs(plain["dk0"] - ref["dk0"])) > 10 * np.max(np.abs(to64(g["dk0"]) - ref["dk0"]))


@pytest.mark.parametrize("dt,path,flare,norm", [("bf16", 0, False, False), ("f32", 0, False, False),
                                               ("f16", 0, False, True), ("bf16", 0, True, False),
                                               ("bf16", 1, False, False), ("bf16", 0, False, True)])
def test_training_step_with_saved_state(dt, path, flare, norm):
    """mixer_fwd_train returns the forward's y bitwise and a context; the
    backward from that context (no recomputed forward) matches the oracle and
    the recomputing backward."""
    b = binding()
    x, dy = inputs(2, 2, 1100, 96, 64, dt, seed=29)
    d = {k: v.to(DEV) for k, v in x.items()}
    gate = None if flare else d["gate"]
    y_plain = b.mixer_fwd(d["q0"], d["q_fixed"], gate, d["k0"], d["k"], d["v"], path=path, norm_synthesis=norm)
    y, ctx = b.mixer_fwd_train(d["q0"], d["q_fixed"], gate, d["k0"], d["k"], d["v"], path=path,
                               norm_synthesis=norm)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain), "the training forward must return the forward's y"
    g = b.mixer_bwd(d["q0"], d["q_fixed"], gate, d["k0"], d["k"], d["v"], dy.to(DEV), path=path,
                    norm_synthesis=norm, ctx=ctx, y=y)
    g_re = b.mixer_bwd(d["q0"], d["q_fixed"], gate, d["k0"], d["k"], d["v"], dy.to(DEV), path=path,
                       norm_synthesis=norm)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    ref = oracle_grads(x, dy, gate=np.zeros(2) if flare else None, norm=norm)
    names = FLARE_GRADS if flare else GRADS
    for name in names:
        assert_grad_parity(g[name], ref[name], dt, name + " (saved state)")
        if dt == "f32" or path == 1:
            # the SIMT backward takes nothing from y: the two must agree to rounding of the sums
            assert torch.allclose(g[name].double(), g_re[name].double(), rtol=0,
                                  atol=1e-5 * float(g_re[name].double().abs().max()))
    if not flare:
        assert_dgate_parity(g["dgate"], ref, dt)


def test_saved_state_argument_errors():
    b = binding()
    x, dy = inputs(1, 2, 300, 32, 32, "bf16", seed=31)
    d = {k: v.to(DEV) for k, v in x.items()}
    y, ctx = b.mixer_fwd_train(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"])
    with pytest.raises(b.FlareppError):                     # context too small
        b.mixer_bwd(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], dy.to(DEV), ctx=ctx[:64], y=y)
    with pytest.raises(ValueError):                          # no y
        b.mixer_bwd(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], dy.to(DEV), ctx=ctx)


def test_scale1m_backward_against_simt():
    """The 1M-token workload in the launch configuration the benchmark times.
    The oracle's dense per-head matrices do not fit at this size, so the
    tensor-core backward is checked against the independent SIMT backward
    (fp32 arithmetic throughout; itself checked against the oracle above) on
    the same inputs, within the bf16 gradient bounds, plus determinism and the
    saved-state path."""
    b = binding()
    w = W.WORKLOADS["scale1m_bf16"]
    x = W.make_inputs(w, device=DEV)
    dy = W.random_cotangent((w.B, w.H, w.N, w.D), "bf16", seed=w.seed + 100, device=DEV, device_rng=True)
    args = (x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], dy)
    g_tc = b.mixer_bwd(*args)
    g_tc2 = b.mixer_bwd(*args)
    g_simt = b.mixer_bwd(*args, path=b.PATH_SIMT)
    y, ctx = b.mixer_fwd_train(*args[:6])
    g_ctx = b.mixer_bwd(*args, ctx=ctx, y=y)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    for name in GRADS + ("dgate",):
        assert torch.equal(g_tc[name], g_tc2[name]), f"{name}: not deterministic"
        ref = g_simt[name].double()
        for label, g in (("tcgen05", g_tc[name]), ("saved state", g_ctx[name])):
            err = (g.double() - ref)
            rel_l2 = float(err.norm() / ref.norm())
            rel_max = float(err.abs().max() / ref.abs().max())
            assert rel_l2 <= 1e-2 and rel_max <= 3e-2, (name, label, rel_l2, rel_max)
            assert bool(torch.isfinite(g.float()).all())
