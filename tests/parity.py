"""Parity metrics between the CUDA path and the fp64 oracle.

Tolerances of the FLARE++ mixer forward on B200:
  fp32 I/O : max relative error <= 1e-4, taken row by row in the max norm:
             for every output row r (the D-vector of one token or latent),
             max_d |g - o| / max_d |o| <= 1e-4
  bf16 I/O : ||g - o||_2 / ||o||_2 <= 1e-2  and  max |g - o| <= 2e-2
  fp16 I/O : ||g - o||_2 / ||o||_2 <= 2.5e-3 and  max |g - o| <= 5e-3
             (the bf16 bounds scaled by 1/4: the errors come from rounding
             q, z, the weights P and y to the 16-bit type, whose unit
             roundoff is 8 times smaller in fp16; a factor 2 is kept as margin)
An elementwise relative error is ill-conditioned here: z is a weighted mean of
zero-mean values, so single entries cancel to near zero and fp32 rounding of
the accumulation order alone gives them relative errors far above 1e-4.  The
elementwise figure (floored at 1e-3 * rms) is still reported.

Gradients (the backward) are held to bounds taken relative to the gradient
tensor's own size, since their scale follows the upstream gradient and the
sizes of the sums they come from, not the unit scale of y:
  fp32 : max |g - o| <= 1e-4 * max |o|
  bf16 : rel L2 <= 1e-2   and  max |g - o| <= 3e-2 * max |o|
  fp16 : rel L2 <= 2.5e-3 and  max |g - o| <= 7.5e-3 * max |o|
The elementwise bound is wider than y's because 16-bit I/O rounds the routing
queries q to the I/O type where they feed the tensor cores (the forward's
convention), and the latent gradients are sums over all tokens of terms
P (dP - Delta) k that cancel: on a D = 16, M = 200 case an emulation of that
one rounding alone moves max |dq_fixed - o| / max |o| to 1.7e-2 (all the
backward's bf16 roundings together: 2.1e-2), against 1.3e-3 for each of the
others (P, dS, dz, z).  fp16 keeps the factor 1/4 of the forward bounds.

A softmax scale s other than the default 1/sqrt(D) (the FLARE block prints
s = 1): the 16-bit bounds above are multiplied by max(1, s sqrt(D)).  The
routing queries q are rounded to the I/O type as tensor-core operands, so a
score s <q, k> carries an absolute error of about s sqrt(D) |q_d| |k_d| u (u
the unit roundoff); at the default scale that is the error the bounds were set
for, and it grows in proportion to s sqrt(D), and with it the error of every
softmax weight (measured at s = 1: bf16 rel L2 stays under 0.7e-2 for y, q, z,
max abs reaches 0.07 at D = 64-128, where the scaled bound is 0.16-0.23).
"""
import numpy as np
import torch

FP32_MAX_REL = 1e-4
BF16_REL_L2 = 1e-2
BF16_MAX_ABS = 2e-2
F16_REL_L2 = 2.5e-3
F16_MAX_ABS = 5e-3
GRAD_BF16_MAX = 3e-2
GRAD_F16_MAX = 7.5e-3


def to64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def metrics(g, o):
    g, o = to64(g), to64(o)
    diff = np.abs(g - o)
    rms = float(np.sqrt(np.mean(o * o)))
    floor = max(1e-3 * rms, 1e-30)
    D = o.shape[-1]
    gr, orow = g.reshape(-1, D), o.reshape(-1, D)
    row_rel = np.abs(gr - orow).max(axis=1) / np.maximum(np.abs(orow).max(axis=1), 1e-30)
    return {
        "row_max_rel": float(row_rel.max()),
        "rel_l2": float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30)),
        "max_abs": float(diff.max()),
        "max_rel": float((diff / np.maximum(np.abs(o), floor)).max()),
        "max_rel_unfloored": float((diff / np.maximum(np.abs(o), 1e-30)).max()),
        "finite": bool(np.all(np.isfinite(g))),
    }


def scale_factor(scale: float, D: int) -> float:
    """Factor on the 16-bit bounds for a softmax scale other than 1/sqrt(D)
    (scale <= 0 selects the default)."""
    return 1.0 if scale <= 0 else max(1.0, scale * D ** 0.5)


def assert_parity(g, o, dtype: str, what: str = "y", factor: float = 1.0):
    m = metrics(g, o)
    assert m["finite"], f"{what}: non-finite values"
    if dtype == "f32":
        assert m["row_max_rel"] <= FP32_MAX_REL, f"{what}: fp32 row max rel {m['row_max_rel']:.3e} > {FP32_MAX_REL} ({m})"
    elif dtype == "f16":
        assert m["rel_l2"] <= F16_REL_L2 * factor, f"{what}: fp16 rel L2 {m['rel_l2']:.3e} > {F16_REL_L2 * factor} ({m})"
        assert m["max_abs"] <= F16_MAX_ABS * factor, f"{what}: fp16 max abs {m['max_abs']:.3e} > {F16_MAX_ABS * factor} ({m})"
    else:
        assert m["rel_l2"] <= BF16_REL_L2 * factor, f"{what}: bf16 rel L2 {m['rel_l2']:.3e} > {BF16_REL_L2 * factor} ({m})"
        assert m["max_abs"] <= BF16_MAX_ABS * factor, f"{what}: bf16 max abs {m['max_abs']:.3e} > {BF16_MAX_ABS * factor} ({m})"
    return m


def assert_grad_parity(g, o, dtype: str, what: str, zero_atol: float = 1e-5, factor: float = 1.0):
    """A gradient the mathematics makes exactly zero (e.g. the seeds' gradient
    when one token carries all the softmax weight) is held to an absolute
    bound instead: the CUDA path leaves rounding noise there."""
    m = metrics(g, o)
    gmax = float(np.abs(to64(o)).max())
    assert m["finite"], f"{what}: non-finite values"
    if gmax == 0.0:
        assert m["max_abs"] <= zero_atol, f"{what}: exact zero expected, max |g| {m['max_abs']:.3e}"
        return m
    m["max_abs_rel_to_max"] = m["max_abs"] / gmax
    if dtype == "f32":
        assert m["max_abs_rel_to_max"] <= FP32_MAX_REL, f"{what}: fp32 max err / max {m['max_abs_rel_to_max']:.3e} ({m})"
    elif dtype == "f16":
        assert m["rel_l2"] <= F16_REL_L2 * factor, f"{what}: fp16 rel L2 {m['rel_l2']:.3e} ({m})"
        assert m["max_abs_rel_to_max"] <= GRAD_F16_MAX * factor, \
            f"{what}: fp16 max err / max {m['max_abs_rel_to_max']:.3e} ({m})"
    else:
        assert m["rel_l2"] <= BF16_REL_L2 * factor, f"{what}: bf16 rel L2 {m['rel_l2']:.3e} ({m})"
        assert m["max_abs_rel_to_max"] <= GRAD_BF16_MAX * factor, \
            f"{what}: bf16 max err / max {m['max_abs_rel_to_max']:.3e} ({m})"
    return m


def assert_dgate_parity(g, ref: dict, dtype: str, zero_atol: float = 0.0, factor: float = 1.0):
    """dgate[h] = sum over (b, m, d) of dq * q_dyn is a dot product whose terms
    cancel, so its error is bounded through dq's by Cauchy-Schwarz:
    |err_h| <= ||err(dq)_h|| ||q_dyn_h|| <= tol ||dq_h|| ||q_dyn_h||, with tol
    the rel-L2 bound of the dtype (fp32: 1e-4).  Where the mathematics makes
    dq exactly zero (one token) the bound is the absolute zero_atol."""
    g = to64(g)
    o = to64(ref["dgate"])
    dq, qd = to64(ref["dq"]), to64(ref["q_dyn"])
    tol = {"f32": FP32_MAX_REL, "f16": F16_REL_L2 * factor}.get(dtype, BF16_REL_L2 * factor)
    assert np.all(np.isfinite(g)), "dgate: non-finite values"
    for h in range(o.shape[0]):
        bound = max(tol * np.linalg.norm(dq[:, h]) * np.linalg.norm(qd[:, h]), zero_atol)
        assert abs(g[h] - o[h]) <= bound, f"dgate[{h}]: |{g[h]:.6e} - {o[h]:.6e}| > {bound:.3e}"
