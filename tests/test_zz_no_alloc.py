"""flarepp_mixer_fwd_noalloc: the mixer forward that allocates no device memory.

Some callers cannot allocate device memory while the mixer runs: their memory
belongs to another allocator (a framework's caching allocator, or an arena
reserved up front that must not be bypassed), or they cannot afford the
implicit synchronisation a cudaMalloc/cudaFree may bring.  For them the
library takes the call's scratch from a fixed device array of
FLAREPP_NOALLOC_SCRATCH_BYTES (32 MiB) instead of allocating it.

Each case calls the entry point through the C ABI twice in a row and checks
both results against the allocating entry point flarepp_mixer_fwd, within the
parity tolerances the other tests use (the no-allocation entry may split the
token axis into fewer chunks to fit its array, which changes rounding only).
Small cases are also compared with the fp64 oracle directly.  A problem too
large for the array must be refused without a launch.  And the promise in
the name is checked: across two calls (after a first call that looks up the
array's address) free device memory does not change and the device's default
memory pool -- where the allocating entry's stream-ordered scratch comes
from -- takes no memory, while the same reading does see the allocating
entry's scratch.
"""
import ctypes
import types

import pytest
import torch

import devmem
import oracle
from parity import assert_parity
from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _lib():
    from rank_latent_attention_mixer_b200 import binding
    fn = binding.lib.flarepp_mixer_fwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    fn.restype = ctypes.c_int
    return binding, fn


@pytest.mark.parametrize("name", ["tiny_f32", "grid85_bf16", "cloud40k_bf16", "scale1m_bf16"])
def test_noalloc_matches_allocating_entry(name):
    b, fn = _lib()
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, device="cuda")
    B, H, N, M, D = w.B, w.H, w.N, w.M, w.D
    dtype = b.F32 if w.dtype == "f32" else b.BF16
    ref = b.mixer_fwd_plain(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], torch.empty_like(x["k"]))
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for _ in range(2):
        y = torch.full_like(x["k"], float("nan"))
        rc = fn(x["q0"].data_ptr(), x["q_fixed"].data_ptr(), x["gate"].data_ptr(), x["k0"].data_ptr(),
                x["k"].data_ptr(), x["v"].data_ptr(), y.data_ptr(), B, H, N, M, D, dtype, stream)
        assert rc == 0, b.status_string(rc)
        outs.append(y)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    for y in outs:
        assert_parity(y, ref, w.dtype, f"{name} noalloc vs flarepp_mixer_fwd")
    assert torch.equal(outs[0], outs[1])


def test_noalloc_refuses_too_large():
    b, fn = _lib()
    # aligned, far enough apart not to overlap at these sizes, never dereferenced: nothing launches
    fake = [(i + 1) << 36 for i in range(7)]
    rc = fn(*fake, 16, 16, 1024, 4096, 128, b.BF16, None)
    assert rc == 4                                    # FLAREPP_ERR_WORKSPACE
    rc = fn(*fake, 1, 2, 64, 16, 48, b.BF16, None)
    assert rc == 2                                    # unsupported head dim, checked first


def _call(fn, b, x, y, w, dtype):
    stream = torch.cuda.current_stream().cuda_stream
    rc = fn(x["q0"].data_ptr(), x["q_fixed"].data_ptr(), x["gate"].data_ptr(), x["k0"].data_ptr(),
            x["k"].data_ptr(), x["v"].data_ptr(), y.data_ptr(), w.B, w.H, w.N, w.M, w.D, dtype, stream)
    assert rc == 0, b.status_string(rc)


@pytest.mark.parametrize("shape,dt", [((1, 2, 1000, 64, 32), "bf16"), ((2, 2, 777, 100, 64), "bf16"),
                                      ((1, 2, 1024, 16, 16), "f32")])
def test_noalloc_matches_oracle(shape, dt):
    """Two calls in a row, each against the fp64 oracle on the same inputs."""
    b, fn = _lib()
    B, H, N, M, D = shape
    x = W.random_inputs(B, H, N, M, D, dtype=dt, seed=11)
    d = {k: v.cuda() for k, v in x.items()}
    w = types.SimpleNamespace(B=B, H=H, N=N, M=M, D=D)
    ref, _, _ = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    for _ in range(2):
        y = torch.full_like(d["k"], float("nan"))
        _call(fn, b, d, y, w, b.F32 if dt == "f32" else b.BF16)
        torch.cuda.synchronize()
        assert b.check_device_status() == 0
        assert_parity(y, ref, dt, f"noalloc {shape} {dt} vs oracle")


def test_noalloc_takes_no_device_memory():
    b, fn = _lib()
    w = W.WORKLOADS["cloud40k_bf16"]
    x = W.make_inputs(w, device="cuda")
    y = torch.empty_like(x["k"])
    _call(fn, b, x, y, w, b.BF16)                 # the first call looks up the array's address
    torch.cuda.synchronize()
    devmem.reset_pool_high_water()
    free0 = devmem.free_bytes()
    for _ in range(2):
        _call(fn, b, x, y, w, b.BF16)
    torch.cuda.synchronize()
    assert devmem.pool_high_water() == 0, "flarepp_mixer_fwd_noalloc took memory from the default pool"
    assert devmem.free_bytes() == free0, "free device memory changed across flarepp_mixer_fwd_noalloc"
    # control: the allocating entry's stream-ordered scratch shows in the same reading
    b.mixer_fwd_plain(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], y)
    torch.cuda.synchronize()
    assert devmem.pool_high_water() >= b.workspace_bytes(w.B, w.H, w.N, w.M, w.D, b.BF16, True, 0)
