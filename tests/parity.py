"""Parity metrics between the CUDA path and the fp64 oracle.

Tolerances of the FLARE++ mixer forward on B200:
  fp32 I/O : elementwise |g - o| / max(|o|, 1e-3 * rms(o)) <= 1e-4
  bf16 I/O : ||g - o||_2 / ||o||_2 <= 1e-2  and  max |g - o| <= 2e-2
The 1e-3*rms floor keeps entries near zero from turning rounding of the
accumulation order into huge relative numbers.
"""
import numpy as np
import torch

FP32_MAX_REL = 1e-4
BF16_REL_L2 = 1e-2
BF16_MAX_ABS = 2e-2


def to64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def metrics(g, o):
    g, o = to64(g), to64(o)
    diff = np.abs(g - o)
    rms = float(np.sqrt(np.mean(o * o)))
    floor = max(1e-3 * rms, 1e-30)
    return {
        "rel_l2": float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30)),
        "max_abs": float(diff.max()),
        "max_rel": float((diff / np.maximum(np.abs(o), floor)).max()),
        "max_rel_unfloored": float((diff / np.maximum(np.abs(o), 1e-30)).max()),
        "finite": bool(np.all(np.isfinite(g))),
    }


def assert_parity(g, o, dtype: str, what: str = "y"):
    m = metrics(g, o)
    assert m["finite"], f"{what}: non-finite values"
    if dtype == "f32":
        assert m["max_rel"] <= FP32_MAX_REL, f"{what}: fp32 max rel {m['max_rel']:.3e} > {FP32_MAX_REL}"
    else:
        assert m["rel_l2"] <= BF16_REL_L2, f"{what}: bf16 rel L2 {m['rel_l2']:.3e} > {BF16_REL_L2}"
        assert m["max_abs"] <= BF16_MAX_ABS, f"{what}: bf16 max abs {m['max_abs']:.3e} > {BF16_MAX_ABS}"
    return m
