"""Writes tests/golden/tiny_mixer.json: a small seeded case and the oracle's
fp64 outputs for it.  It calls only the oracle package and the seeded input
generator; no value in the fixture comes from the CUDA library.

The case: B=1, H=2, N=13, M=3, D=16, iid recipe with RMS-normalised q0 and k0,
bf16-representable inputs (FLARE.py README, "FLARE++" code block; shapes from
its docstring), plus the closed-gate FLARE output for the same inputs.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from rank_latent_attention_mixer_b200.workloads import random_inputs  # noqa: E402


def main():
    B, H, N, M, D = 1, 2, 13, 3, 16
    x = random_inputs(B, H, N, M, D, dtype="bf16", seed=1234)
    y, q, z = oracle.flarepp(x["q0"], x["q_fixed"], x["gate"], x["k0"], x["k"], x["v"])
    yf, _, _ = oracle.flarepp(None, x["q_fixed"], None, None, x["k"], x["v"], flare=True)
    as_list = lambda t: t.double().flatten().tolist() if hasattr(t, "double") else t.flatten().tolist()
    doc = {
        "source": "oracle/ (fp64) via tests/golden/make_golden.py",
        "case": {"B": B, "H": H, "N": N, "M": M, "D": D, "dtype": "bf16", "seed": 1234, "recipe": "iid"},
        "inputs": {name: as_list(x[name]) for name in ("q0", "q_fixed", "gate", "k0", "k", "v")},
        "outputs": {"y": as_list(y), "q": as_list(q), "z": as_list(z), "y_flare": as_list(yf)},
    }
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_mixer.json")
    with open(out, "w") as f:
        json.dump(doc, f, separators=(",", ":"))
        f.write("\n")
    print("wrote", out)


if __name__ == "__main__":
    main()
