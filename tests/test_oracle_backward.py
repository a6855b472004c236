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


def _loss(x, dy):
    y, _, _ = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
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
