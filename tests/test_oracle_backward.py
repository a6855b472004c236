"""The fp64 gradient oracle (oracle/backward.py) against the forward oracle:
directional central differences of L = sum(y * dy) for every input, and the
closed form of a zero gate (the synthesis then has no effect on y).  CPU only."""
import numpy as np
import pytest

import oracle
from oracle.backward import flarepp_backward


def _inputs(seed, B, H, N, M, D):
    r = np.random.default_rng(seed)
    return dict(q0=r.standard_normal((H, M, D)), q_fixed=r.standard_normal((H, M, D)),
                gate=1.0 / (1.0 + np.exp(-r.standard_normal(H))),
                k0=r.standard_normal((B, H, N, D)), k=r.standard_normal((B, H, N, D)),
                v=r.standard_normal((B, H, N, D))), r.standard_normal((B, H, N, D))


def _loss(x, dy, norm=False):
    q0, k0 = (oracle.rms_normalise(x["q0"]), oracle.rms_normalise(x["k0"])) if norm else (x["q0"], x["k0"])
    y, _, _ = oracle.flarepp(q0, x["q_fixed"], x["gate"], k0, x["k"], x["v"])
    return float(np.sum(y * dy))


@pytest.mark.parametrize("shape", [(1, 2, 23, 5, 16), (2, 1, 17, 8, 32)])
def test_gradients_match_central_differences(shape):
    B, H, N, M, D = shape
    x, dy = _inputs(sum(shape), B, H, N, M, D)
    g = flarepp_backward(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], dy)
    y_c, _, _ = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    assert np.max(np.abs(g["y"] - y_c)) < 1e-12
    r = np.random.default_rng(7)
    h = 1e-5
    for name, grad in (("q0", "dq0"), ("q_fixed", "dq_fixed"), ("gate", "dgate"), ("k0", "dk0"), ("k", "dk"),
                       ("v", "dv")):
        for _ in range(3):
            e = r.standard_normal(x[name].shape)
            xp = dict(x); xp[name] = x[name] + h * e
            xm = dict(x); xm[name] = x[name] - h * e
            fd = (_loss(xp, dy) - _loss(xm, dy)) / (2 * h)
            an = float(np.sum(g[grad] * e))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


def test_zero_gate_cuts_the_synthesis():
    x, dy = _inputs(3, 2, 2, 19, 6, 16)
    x["gate"] = np.zeros(2)
    g = flarepp_backward(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], dy)
    assert np.all(g["dq0"] == 0) and np.all(g["dk0"] == 0)
    assert np.any(g["dgate"] != 0)        # the gate's own gradient is not zero


@pytest.mark.parametrize("scale_rows", [1.0, 3.7])
def test_normalised_synthesis_gradients_match_central_differences(scale_rows):
    """With the synthesis reading RMS-normalised q0 and k0 rows, dq0 and dk0 go
    through the normalisation: central differences of the forward oracle with
    the same step.  Rows far from RMS 1 make the step matter."""
    B, H, N, M, D = 1, 2, 19, 6, 16
    x, dy = _inputs(11, B, H, N, M, D)
    x["q0"] = x["q0"] * scale_rows
    x["k0"] = x["k0"] * scale_rows
    g = flarepp_backward(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"], dy, norm_synthesis=True)
    r = np.random.default_rng(5)
    h = 1e-5
    for name, grad in (("q0", "dq0"), ("k0", "dk0"), ("q_fixed", "dq_fixed"), ("gate", "dgate"), ("k", "dk")):
        for _ in range(3):
            e = r.standard_normal(x[name].shape)
            xp = dict(x); xp[name] = x[name] + h * e
            xm = dict(x); xm[name] = x[name] - h * e
            fd = (_loss(xp, dy, True) - _loss(xm, dy, True)) / (2 * h)
            an = float(np.sum(g[grad] * e))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)
    # the normalisation is invariant to each row's scale up to eps, so dq0 and dk0
    # are orthogonal to their rows up to eps / (mean x^2 + eps) ~ 1e-6 (a radial
    # change does almost nothing)
    for gx, xx in ((g["dq0"], x["q0"]), (g["dk0"], x["k0"])):
        radial = np.abs(np.sum(gx * xx, axis=-1))
        assert np.all(radial <= 1e-5 * np.linalg.norm(gx, axis=-1) * np.linalg.norm(xx, axis=-1))
