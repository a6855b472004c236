"""CUDA path vs the fp64 oracle on the same seeded inputs, through the C ABI.

Covers the four workloads the oracle finishes in seconds (whole outputs y, q
and z), the closed-gate FLARE form, every supported head dim, ragged and
degenerate sizes, forced chunk counts (the token-split/log-sum-exp merge is
exact up to rounding), both kernel families, and the ABI variants (explicit
or library-managed scratch, host buffers)."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_parity, metrics, scale_factor, to64
from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
_ORACLE_CACHE = {}


def binding():
    from rank_latent_attention_mixer_b200 import binding as b
    return b


def oracle_out(name, x, flare=False):
    key = (name, flare)
    if key not in _ORACLE_CACHE:
        _ORACLE_CACHE[key] = oracle.flarepp(x["q0"], x["q_fixed"], None if flare else x["gate"],
                                            x["k0"], x["k"], x["v"], flare=flare)
    return _ORACLE_CACHE[key]


def cuda_inputs(x):
    return {k: v.to(DEV) for k, v in x.items()}


def run(x, path=0, force_chunks=0, flare=False, scale=0.0):
    b = binding()
    d = cuda_inputs(x)
    y, q, z = b.mixer_fwd(d["q0"], d["q_fixed"], None if flare else d["gate"], d["k0"], d["k"], d["v"],
                          return_qz=True, path=path, force_chunks=force_chunks, scale=scale)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    return y, q, z


SMALL = ["tiny_f32", "grid85_bf16", "grid129_peaky_bf16", "cloud40k_bf16", "cloud40k_f16"]


@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("path", [0, 1], ids=["auto", "simt"])
def test_workload_parity(name, path):
    w = W.WORKLOADS[name]
    x = W.make_inputs(w)
    y_ref, q_ref, z_ref = oracle_out(name, x)
    y, q, z = run(x, path=path)
    assert_parity(q, q_ref, w.dtype, "q")
    assert_parity(z, z_ref, w.dtype, "z")
    m = assert_parity(y, y_ref, w.dtype, "y")
    print(name, path, m)


@pytest.mark.parametrize("name", ["grid85_bf16", "tiny_f32", "cloud40k_f16"])
def test_closed_gate_is_flare(name):
    w = W.WORKLOADS[name]
    x = W.make_inputs(w)
    y_ref, _, _ = oracle_out(name, x, flare=True)
    b = binding()
    d = cuda_inputs(x)
    y_flare = b.flare_fwd(d["q_fixed"], d["k"], d["v"])
    y_null = b.mixer_fwd(d["q0"], d["q_fixed"], None, d["k0"], d["k"], d["v"])
    y_zero = b.mixer_fwd(d["q0"], d["q_fixed"], torch.zeros_like(d["gate"]), d["k0"], d["k"], d["v"])
    torch.cuda.synchronize()
    assert_parity(y_flare, y_ref, w.dtype, "y(flare)")
    assert torch.equal(y_flare, y_null)
    assert torch.equal(y_flare, y_zero), "a zero gate must give exactly the FLARE result"


EDGE = [
    # B, H, N, M, D
    (1, 1, 1, 1, 16),
    (1, 2, 7, 5, 16),
    (2, 1, 129, 17, 32),
    (1, 3, 300, 64, 64),
    (1, 1, 1000, 1, 64),
    (1, 2, 257, 130, 128),
    (3, 2, 513, 64, 16),
    (1, 1, 4097, 256, 32),
    (1, 2, 2000, 512, 64),
    (1, 1, 640, 100, 32),
    (2, 4, 3001, 256, 128),
    (1, 2, 1000, 64, 128),
    (1, 1, 5000, 512, 128),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "x".join(map(str, s)))
def test_edge_shapes(shape, dtype):
    B, H, N, M, D = shape
    x = W.random_inputs(B, H, N, M, D, dtype=dtype, seed=sum(shape))
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    y, q, z = run(x)
    assert_parity(q, q_ref, dtype, "q")
    assert_parity(z, z_ref, dtype, "z")
    assert_parity(y, y_ref, dtype, "y")


@pytest.mark.parametrize("dtype,path", [("bf16", 0), ("f16", 0), ("f32", 0), ("bf16", 1)],
                         ids=["bf16-auto", "f16-auto", "f32", "bf16-simt"])
@pytest.mark.parametrize("shape", [(2, 3, 1000, 64, 32), (1, 8, 3001, 256, 64), (2, 2, 300, 17, 16),
                                   (1, 1, 777, 130, 64), (1, 2, 900, 128, 128)], ids=lambda s: "x".join(map(str, s)))
def test_bnhd_layout(shape, dtype, path):
    """k0, k, v, y in [B,N,H,D] (one token's heads adjacent) give exactly the
    [B,H,N,D] result: only the addressing differs."""
    B, H, N, M, D = shape
    x = W.random_inputs(B, H, N, M, D, dtype=dtype, seed=B * H + N)
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    y, q, z = run(x, path=path)
    b = binding()
    d = cuda_inputs(x)
    t = lambda a: a.transpose(1, 2).contiguous()
    for gated in (True, False):
        yb, qb, zb = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"] if gated else None, t(d["k0"]), t(d["k"]),
                                 t(d["v"]), return_qz=True, path=path, layout="bnhd")
        torch.cuda.synchronize()
        assert b.check_device_status() == 0
        assert yb.shape == (B, N, H, D)
        if gated:
            assert torch.equal(yb.transpose(1, 2), y)
            assert torch.equal(qb, q) and torch.equal(zb, z)
            assert_parity(yb.transpose(1, 2), y_ref, dtype, "y (bnhd)")
        else:
            y_flare = b.mixer_fwd(d["q0"], d["q_fixed"], None, d["k0"], d["k"], d["v"], path=path)
            assert torch.equal(yb.transpose(1, 2), y_flare)


@pytest.mark.parametrize("path", [0, 1], ids=["auto", "simt"])
def test_chunk_invariance(path):
    x = W.random_inputs(2, 2, 3001, 128, 32, dtype="bf16", seed=5)
    y_ref, _, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    outs = []
    for fc in (0, 1, 2, 7):
        y, q, z = run(x, path=path, force_chunks=fc)
        assert_parity(y, y_ref, "bf16")
        outs.append((y, q, z))
    for y, q, z in outs[1:]:
        # The split/merge is exact up to rounding.  The SIMT path keeps the
        # softmax weights in fp32, so chunkings agree to fp32 roundoff; the
        # tcgen05 path rounds the weights to bf16 relative to a running max
        # that depends on the chunking, so they agree to bf16 rounding.
        if path == 1:
            assert metrics(z, outs[0][2])["max_abs"] < 1e-4
            assert metrics(q, outs[0][1])["max_abs"] < 1e-4
        else:
            assert metrics(z, outs[0][2])["rel_l2"] < 6e-3
            assert metrics(q, outs[0][1])["rel_l2"] < 6e-3


def test_scale_argument_flare_scale_one():
    """The FLARE block printed with scale=1.0, via the options' scale."""
    x = W.random_inputs(1, 2, 500, 32, 16, dtype="f32", seed=3)
    y_ref, _, _ = oracle.flarepp(None, x["q_fixed"], None, None, x["k"], x["v"], scale=1.0, flare=True)
    y, _, _ = run(x, flare=True, scale=1.0)
    assert_parity(y, y_ref, "f32")


def test_deterministic_and_abi_variants():
    w = W.WORKLOADS["grid85_bf16"]
    x = W.make_inputs(w)
    d = cuda_inputs(x)
    b = binding()
    y1 = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"])
    y2 = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"])
    y3 = b.mixer_fwd_plain(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], torch.empty_like(d["k"]))
    hx = {k: v.pin_memory() for k, v in x.items()}
    y4 = torch.empty_like(hx["k"]).pin_memory()
    b.mixer_fwd_host(hx["q0"], hx["q_fixed"], hx["gate"], hx["k0"], hx["k"], hx["v"], y4)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(y1, y3)
    # the host entry plans its token chunks per (b, h) slice: equal up to rounding
    assert_parity(y4, y1.cpu(), w.dtype, "host entry vs device entry")
    y_ref, _, _ = oracle_out("grid85_bf16", x)
    assert_parity(y4, y_ref, w.dtype, "host entry vs oracle")


def test_invariants_on_gpu():
    # single latent: every token gets the latent's value
    x = W.random_inputs(1, 2, 999, 1, 32, dtype="f32", seed=11)
    y, _, z = run(x)
    assert torch.allclose(y, z.expand_as(y), rtol=1e-5, atol=1e-6)
    # identical keys: encode returns the mean of v
    x = W.random_inputs(1, 2, 777, 16, 32, dtype="f32", seed=12)
    x["k"][:] = x["k"][:, :, :1]
    _, _, z = run(x)
    mean_v = x["v"].double().mean(dim=2, keepdim=True).expand(-1, -1, 16, -1)
    assert metrics(z, mean_v)["max_abs"] < 1e-5
    # convex hull: each y coordinate within the latents' range
    x = W.random_inputs(2, 2, 3000, 64, 16, dtype="bf16", seed=13)
    y, _, z = run(x)
    lo = z.min(dim=2, keepdim=True).values
    hi = z.max(dim=2, keepdim=True).values
    tol = 2 ** -7 * z.abs().max()
    yf = y.float()
    assert bool(((yf >= lo - tol) & (yf <= hi + tol)).all())


def test_permutation_equivariance_gpu():
    x = W.random_inputs(1, 2, 2500, 64, 32, dtype="f32", seed=21)
    perm = torch.randperm(2500, generator=torch.Generator().manual_seed(0))
    xp = dict(x)
    for kname in ("k0", "k", "v"):
        xp[kname] = x[kname][:, :, perm].contiguous()
    y, q, z = run(x)
    yp, qp, zp = run(xp)
    assert metrics(qp, q)["row_max_rel"] < 1e-4 and metrics(zp, z)["row_max_rel"] < 1e-4
    assert metrics(yp, y[:, :, perm.to(y.device)])["row_max_rel"] < 1e-4


def test_scale1m_full():
    """The 1M-token bf16 workload (B=1, H=8, N=1048576, M=512, D=64) in the
    launch configuration the benchmark times, compared with the oracle in full:
    every head's q and z and every token of y.  The oracle runs one (b, h)
    slice at a time; the bf16 bounds are taken over the whole tensors
    (relative L2 from the accumulated squared norms, max abs over all)."""
    w = W.WORKLOADS["scale1m_bf16"]
    x = W.make_inputs(w, device=DEV)
    b = binding()
    y, q, z = b.mixer_fwd(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], return_qz=True)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    acc = {n: [0.0, 0.0, 0.0] for n in ("y", "q", "z")}      # sum d^2, sum o^2, max |d|
    toks = np.arange(w.N, dtype=np.int64)

    def add(name, got, ref):
        d = to64(got) - ref
        a = acc[name]
        a[0] += float((d * d).sum())
        a[1] += float((ref * ref).sum())
        a[2] = max(a[2], float(np.abs(d).max()))

    for bi in range(w.B):
        for h in range(w.H):
            y_ref, q_ref, z_ref = oracle.flarepp_head(x["q0"][h], x["q_fixed"][h], float(x["gate"][h]),
                                                      x["k0"][bi, h], x["k"][bi, h], x["v"][bi, h], toks)
            add("y", y[bi, h], y_ref)
            add("q", q[bi, h], q_ref)
            add("z", z[bi, h], z_ref)
            del y_ref
    for name, (sd, so, mx) in acc.items():
        rel = (sd / so) ** 0.5
        print(f"scale1m_bf16 full {name}: rel_l2={rel:.3e} max_abs={mx:.3e}")
        assert rel <= 1e-2 and mx <= 2e-2, (name, rel, mx)
    assert bool(torch.isfinite(y.float()).all())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("gated", [True, False], ids=["gated", "closed"])
@pytest.mark.parametrize("D,M", [(16, 64), (32, 200), (64, 300), (128, 130)], ids=lambda v: str(v))
def test_scale_one_tensor_cores(D, M, gated, dtype):
    """The FLARE block's printed scale=1.0 (options' scale) on the tensor-core
    kernels: scores 4-11x larger than at 1/sqrt(D), which exercises the fp16
    weight offset and the lazy rescale of the running maximum.  The bounds are
    the dtype's scaled by sqrt(D) (parity.scale_factor: the error of the
    scores from rounding q to the operand type grows with the scale)."""
    x = W.random_inputs(1, 2, 1100, M, D, dtype=dtype, seed=D + M)
    if gated:
        y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], scale=1.0)
    else:
        y_ref, q_ref, z_ref = oracle.flarepp(None, x["q_fixed"], None, None, x["k"], x["v"], scale=1.0, flare=True)
    y, q, z = run(x, flare=not gated, scale=1.0)
    assert binding().selected_path(1, 2, 1100, M, D, binding().BF16 if dtype == "bf16" else binding().F16) == 2
    print(dtype, D, M, gated, "y", metrics(y, y_ref), "z", metrics(z, z_ref))
    f = scale_factor(1.0, D)              # the bounds for a non-default scale (parity.py)
    assert_parity(q, q_ref, dtype, "q", f)
    assert_parity(z, z_ref, dtype, "z", f)
    assert_parity(y, y_ref, dtype, "y", f)


@pytest.mark.parametrize("shape,dtype", [((1, 1, 3001, 1024, 64), "bf16"), ((1, 1, 3001, 1024, 64), "f16"),
                                         ((1, 2, 2500, 2048, 64), "bf16"), ((1, 1, 2500, 2048, 64), "f16"),
                                         ((1, 1, 1500, 4096, 64), "bf16")],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else v)
def test_large_latent_counts(shape, dtype):
    """Latent ranks above 512, up to the header's limit M = 4096 (the pages use
    M = 2048 at 1M points): more latent row groups in the split passes and more
    latent tiles per decode item than the benchmark workloads."""
    B, H, N, M, D = shape
    x = W.random_inputs(B, H, N, M, D, dtype=dtype, seed=M + N)
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    y, q, z = run(x)
    assert_parity(q, q_ref, dtype, "q")
    assert_parity(z, z_ref, dtype, "z")
    assert_parity(y, y_ref, dtype, "y")


@pytest.mark.parametrize("name", ["scale1m_f16"])
def test_scale1m_sampled(name):
    """The 1M-token fp16 workload in the launch configuration the benchmark
    times: one head checked in full for q and z, and 256 sampled tokens of y
    (the bf16 workload is compared in full above)."""
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, device=DEV)
    b = binding()
    y, q, z = b.mixer_fwd(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], return_qz=True)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    h = 5
    toks = torch.randint(0, w.N, (256,), generator=torch.Generator().manual_seed(1)).numpy()
    toks[:2] = [0, w.N - 1]
    y_ref, q_ref, z_ref = oracle.flarepp_head(x["q0"][h], x["q_fixed"][h], float(x["gate"][h]),
                                              x["k0"][0, h], x["k"][0, h], x["v"][0, h], toks)
    assert_parity(q[0, h], q_ref, w.dtype, "q")
    assert_parity(z[0, h], z_ref, w.dtype, "z")
    assert_parity(y[0, h, torch.from_numpy(toks).to(DEV)], y_ref, w.dtype, "y")
    assert bool(torch.isfinite(y.float()).all())


def test_golden_fixture_gpu():
    from test_golden import load_golden
    c, x, ref = load_golden()
    t = {k: torch.from_numpy(v) for k, v in x.items()}
    for k in ("q0", "q_fixed", "k0", "k", "v"):
        t[k] = t[k].to(torch.bfloat16)
    t["gate"] = t["gate"].float()
    y, q, z = run(t)
    assert_parity(y, ref["y"], "bf16")
    assert_parity(q, ref["q"], "bf16")


def test_invalid_args_on_gpu():
    b = binding()
    x = cuda_inputs(W.random_inputs(1, 2, 64, 16, 16, dtype="bf16"))
    with pytest.raises(b.FlareppError) as e:
        b.mixer_fwd(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], y=x["k"])  # y aliases k
    assert e.value.status == 1
    xf = cuda_inputs(W.random_inputs(1, 2, 64, 16, 16, dtype="f32"))
    with pytest.raises(b.FlareppError) as e:       # fp32 I/O has no tensor-core path
        b.mixer_fwd(xf["q0"], xf["q_fixed"], xf["gate"], xf["k0"], xf["k"], xf["v"], path=b.PATH_TCGEN05)
    assert e.value.status == 2


def test_bounded_wait_reports_timeout():
    """A wait that nothing satisfies gives up within its limit, records
    FLAREPP_ERR_TIMEOUT in the device status word, and leaves the context
    usable: the next forward runs and matches the oracle."""
    b = binding()
    assert b.check_device_status() == 0
    assert b.selftest_wait_timeout(20000) == 0          # 20 ms limit
    assert b.check_device_status() == 5                 # FLAREPP_ERR_TIMEOUT, then cleared
    assert b.check_device_status() == 0
    x = W.random_inputs(1, 2, 700, 64, 32, dtype="bf16", seed=31)
    y_ref, _, _ = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    y, _, _ = run(x)
    assert_parity(y, y_ref, "bf16")
