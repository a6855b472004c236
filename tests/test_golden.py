"""The oracle still reproduces the stored golden fixture (guards against an
unintended change of the oracle's arithmetic)."""
import json
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def load_golden():
    with open(os.path.join(HERE, "golden", "tiny_mixer.json")) as f:
        doc = json.load(f)
    c = doc["case"]
    B, H, N, M, D = c["B"], c["H"], c["N"], c["M"], c["D"]
    shapes = {"q0": (H, M, D), "q_fixed": (H, M, D), "gate": (H,), "k0": (B, H, N, D),
              "k": (B, H, N, D), "v": (B, H, N, D), "y": (B, H, N, D), "q": (B, H, M, D),
              "z": (B, H, M, D), "y_flare": (B, H, N, D)}
    arr = lambda name, src: np.asarray(src[name], dtype=np.float64).reshape(shapes[name])
    inputs = {n: arr(n, doc["inputs"]) for n in doc["inputs"]}
    outputs = {n: arr(n, doc["outputs"]) for n in doc["outputs"]}
    return c, inputs, outputs


def test_oracle_reproduces_golden():
    _, x, ref = load_golden()
    y, q, z = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    np.testing.assert_allclose(y, ref["y"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(q, ref["q"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(z, ref["z"], rtol=0, atol=1e-13)
    yf, _, _ = oracle.flarepp(None, x["q_fixed"], None, None, x["k"], x["v"], flare=True)
    np.testing.assert_allclose(yf, ref["y_flare"], rtol=0, atol=1e-13)
