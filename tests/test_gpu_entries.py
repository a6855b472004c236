"""The C-ABI entries that mirror the boundary's debug and workspace calls:
flarepp_mixer_fwd_debug returns y and the fp32 intermediates q and z (checked
against the oracle, with a forced chunk count as well), and a workspace
registered with flarepp_set_workspace serves the plain forward without any
allocation from the device's default memory pool, bit-identically to the
library-allocated scratch."""
import pytest
import torch

import devmem
import oracle
from parity import assert_parity
from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu


def binding():
    from rank_latent_attention_mixer_b200 import binding as b
    return b


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("force_chunks", [0, 3])
def test_debug_entry_returns_q_and_z(dtype, force_chunks):
    b = binding()
    x = W.random_inputs(2, 2, 1500, 200, 32, dtype=dtype, seed=41)
    y_ref, q_ref, z_ref = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    d = {k: v.cuda() for k, v in x.items()}
    y, q, z = b.mixer_fwd_debug(d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], force_chunks=force_chunks)
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    assert_parity(y, y_ref, dtype, "y")
    assert_parity(q, q_ref, dtype, "q")
    assert_parity(z, z_ref, dtype, "z")


def test_registered_workspace_is_used():
    b = binding()
    w = W.WORKLOADS["grid129_peaky_bf16"]
    x = W.make_inputs(w, device="cuda")
    ref = b.mixer_fwd_plain(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], torch.empty_like(x["k"]))
    need = b.workspace_bytes(w.B, w.H, w.N, w.M, w.D, b.BF16, True)
    buf = torch.empty(need, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(x["k"])
    b.set_workspace(buf)
    try:
        torch.cuda.synchronize()
        devmem.reset_pool_high_water()
        b.mixer_fwd_plain(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], y)
        torch.cuda.synchronize()
        assert devmem.pool_high_water() == 0, "the registered workspace was not used"
        assert torch.equal(y, ref)
    finally:
        b.set_workspace(None)
    # unregistered again: the library allocates stream-ordered scratch
    b.mixer_fwd_plain(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], y)
    torch.cuda.synchronize()
    assert devmem.pool_high_water() >= need
    assert b.check_device_status() == 0
