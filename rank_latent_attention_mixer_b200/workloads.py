"""Seeded synthetic inputs for the FLARE++ mixer forward.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds no arithmetic of the mixer itself: it only draws inputs and rounds them
to the I/O dtype.  The head-wise normalisation of the latent seeds and of the
synthesis keys (physicsnemo issue #2024, "Normalizing the synthesis call") is
applied here, to the inputs, because the FLARE.py README's mixer block is
written "without projections and normalizations": it is a property of the
inputs the mixer sees, not a step of the mixer.

Recipe (one entry per workload, drawn in fp64 with ``torch.Generator('cpu')``
seeded with the workload's seed, in the order q0, q_fixed, g, then the token
tensors; rounded to the I/O dtype with round-to-nearest-even):

* ``gate = sigmoid(g)``, ``g ~ N(0, 1)`` per head, kept in fp32 (the library
  takes the gate value, never the logit).
* RMS normalisation of a row x over D: ``x / sqrt(mean(x**2) + 1e-6)``, no
  learned weight.
* ``iid``: q0, q_fixed, k0, k, v i.i.d. N(0, 1).
* ``peaky``: q0, q_fixed, v ~ N(0, 1); k and k0 are independent N(0, 1) * 2.0.
* ``clusters``: per head 32 centres for k and 32 for k0, all N(0, 1); one
  cluster label per token, uniform over the 32 and shared by every head and
  by k and k0; k = centre + 0.3 * noise, k0 = centre0 + 0.3 * noise0, v ~ N(0, 1).
  Tokens are drawn cluster-contiguous (labels sorted) and then one seeded
  permutation of the N tokens is applied to k0, k and v together.

The 1M-token workload holds 2.7 G random numbers; the CPU generator needs
minutes for that, so its tensors are drawn on the device with
``torch.Generator('cuda')`` from the same recipe (fp32 normals, normalised in
fp32, then rounded to bf16).  Every other workload is drawn on the CPU.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

N_CLUSTERS = 32
RMS_EPS = 1e-6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    M: int
    D: int
    dtype: str          # "f32", "bf16" or "f16"
    seed: int
    recipe: str         # "iid", "peaky" or "clusters"
    rms_q0: bool
    rms_k0: bool
    device_rng: bool = False
    note: str = ""

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[self.dtype]

    @property
    def tokens(self) -> int:
        return self.B * self.N

    def with_shape(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_f32", 1, 2, 1024, 16, 16, "f32", 0, "iid", True, True,
                 note="tiny fp32 case the oracle finishes in well under a second"),
        Workload("grid85_bf16", 4, 8, 7225, 64, 16, "bf16", 1, "iid", True, True,
                 note="85x85 structured-grid tokens, flattened"),
        Workload("grid129_peaky_bf16", 2, 8, 16641, 128, 32, "bf16", 2, "peaky", True, False,
                 note="129x129 grid tokens, keys scaled by 2 for peaky softmaxes"),
        Workload("cloud40k_bf16", 1, 8, 40000, 256, 32, "bf16", 3, "clusters", False, False,
                 note="irregular point cloud, 32 key clusters, tokens randomly permuted"),
        Workload("scale1m_bf16", 1, 8, 1048576, 512, 64, "bf16", 4, "iid", True, True,
                 device_rng=True, note="1M-token scaling case, ~1 GiB per [B,H,N,D] tensor"),
        # variants: the same draws rounded to fp16 (the fp16 forward of the
        # 1M-point runs), and a small fp16 case for parity tests
        Workload("scale1m_f16", 1, 8, 1048576, 512, 64, "f16", 4, "iid", True, True,
                 device_rng=True, note="scale1m_bf16 with fp16 I/O"),
        Workload("cloud40k_f16", 1, 8, 40000, 256, 32, "f16", 3, "clusters", False, False,
                 note="cloud40k_bf16 with fp16 I/O"),
        # head dim 128 (outside the configs above): the widest supported D
        Workload("scale256k_d128_bf16", 1, 8, 262144, 256, 128, "bf16", 5, "iid", True, True,
                 device_rng=True, note="head dim 128, 256K tokens"),
    ]
}
ORDER = ["tiny_f32", "grid85_bf16", "grid129_peaky_bf16", "cloud40k_bf16", "scale1m_bf16"]


def _rms_rows(x: torch.Tensor) -> torch.Tensor:
    return x / torch.sqrt(x.pow(2).mean(dim=-1, keepdim=True) + RMS_EPS)


def _randn(gen: torch.Generator, shape, dtype, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=dtype, device=device)


def make_inputs(w: Workload, device: str = "cpu", gate_zero: bool = False) -> Dict[str, torch.Tensor]:
    """Draw the workload's inputs.  Returns tensors in the I/O dtype on ``device``
    (q0, q_fixed [H,M,D]; k0, k, v [B,H,N,D]) and ``gate`` fp32 [H].

    ``gate_zero`` replaces the drawn gate by zeros (the draw still happens so the
    other tensors are unchanged)."""
    gen_dev = "cuda" if w.device_rng else "cpu"
    work_dtype = torch.float32 if w.device_rng else torch.float64
    if w.device_rng and not torch.cuda.is_available():
        raise RuntimeError(f"workload {w.name} draws its inputs on the GPU; no GPU is available")
    gen = torch.Generator(gen_dev)
    gen.manual_seed(w.seed)
    B, H, N, M, D = w.B, w.H, w.N, w.M, w.D
    out_dtype = w.torch_dtype

    def finish(x: torch.Tensor) -> torch.Tensor:
        return x.to(out_dtype).to(device).contiguous()

    q0 = _randn(gen, (H, M, D), work_dtype, gen_dev)
    if w.rms_q0:
        q0 = _rms_rows(q0)
    q_fixed = _randn(gen, (H, M, D), work_dtype, gen_dev)
    g = _randn(gen, (H,), work_dtype, gen_dev)
    gate = torch.sigmoid(g).to(torch.float32)
    if gate_zero:
        gate = torch.zeros_like(gate)

    res = {"q0": finish(q0), "q_fixed": finish(q_fixed), "gate": gate.to(device).contiguous()}
    if w.recipe == "clusters":
        cen_k = _randn(gen, (H, N_CLUSTERS, D), work_dtype, gen_dev)
        cen_k0 = _randn(gen, (H, N_CLUSTERS, D), work_dtype, gen_dev)
        labels = torch.randint(0, N_CLUSTERS, (N,), generator=gen, device=gen_dev)
        labels, _ = torch.sort(labels)
        noise = _randn(gen, (B, H, N, D), work_dtype, gen_dev)
        noise0 = _randn(gen, (B, H, N, D), work_dtype, gen_dev)
        v = _randn(gen, (B, H, N, D), work_dtype, gen_dev)
        perm = torch.randperm(N, generator=gen, device=gen_dev)
        k = cen_k[:, labels, :].unsqueeze(0) + 0.3 * noise
        k0 = cen_k0[:, labels, :].unsqueeze(0) + 0.3 * noise0
        k, k0, v = k[:, :, perm], k0[:, :, perm], v[:, :, perm]
        res.update(k0=finish(k0), k=finish(k), v=finish(v))
        return res

    key_scale = 2.0 if w.recipe == "peaky" else 1.0
    # Token tensors are drawn one (b, h) slice at a time so the 1M-token case
    # never holds more than one slice in the working precision.
    out = {name: torch.empty((B, H, N, D), dtype=out_dtype, device=device) for name in ("k0", "k", "v")}
    for name in ("k0", "k", "v"):
        for b in range(B):
            for h in range(H):
                x = _randn(gen, (N, D), work_dtype, gen_dev)
                if name in ("k0", "k"):
                    x = x * key_scale
                if name == "k0" and w.rms_k0:
                    x = _rms_rows(x)
                out[name][b, h].copy_(x.to(out_dtype))
    res.update(out)
    return res


def random_inputs(B: int, H: int, N: int, M: int, D: int, dtype: str = "bf16", seed: int = 0,
                  recipe: str = "iid", rms: bool = True, device: str = "cpu",
                  gate_zero: bool = False) -> Dict[str, torch.Tensor]:
    """Inputs of any shape from the same recipe (CPU generator); for edge cases."""
    w = Workload(f"custom_{B}x{H}x{N}x{M}x{D}", B, H, N, M, D, dtype, seed, recipe, rms, rms)
    return make_inputs(w, device=device, gate_zero=gate_zero)


def random_cotangent(shape, dtype: str = "bf16", seed: int = 0, device: str = "cpu",
                     device_rng: bool = False) -> torch.Tensor:
    """An upstream gradient dy for the backward: i.i.d. N(0, 1) of the given
    shape, drawn in fp64 with ``torch.Generator('cpu')`` seeded with ``seed``
    (or in fp32 on the device with ``device_rng``, for the 1M-token sizes) and
    rounded to the I/O dtype."""
    out_dtype = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    gen_dev = "cuda" if device_rng else "cpu"
    gen = torch.Generator(gen_dev)
    gen.manual_seed(seed)
    x = torch.randn(*shape, generator=gen, dtype=torch.float32 if device_rng else torch.float64, device=gen_dev)
    return x.to(out_dtype).to(device).contiguous()


def algorithmic_counts(w: Workload, flare: bool = False) -> Dict[str, float]:
    """Per-call algorithmic work: HBM bytes of the inputs read and the output
    written once, tensor-core FLOPs of the score and value contractions, and
    exponentials (one per score of each softmax)."""
    s = 4 if w.dtype == "f32" else 2
    bhnd = w.B * w.H * w.N * w.D
    bhnmd = w.B * w.H * w.N * w.M * w.D
    passes = 2 if flare else 3
    return {
        "bytes": (4 if flare else 5) * bhnd * s,
        "flops": 4.0 * passes * bhnmd,
        "exps": float(passes * w.B * w.H * w.N * w.M),
        "tokens": float(w.B * w.N),
    }


def describe(w: Workload) -> str:
    return (f"{w.name}: B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} {w.dtype} seed={w.seed} "
            f"recipe={w.recipe} rms(q0)={w.rms_q0} rms(k0)={w.rms_k0}")


__all__ = ["Workload", "WORKLOADS", "ORDER", "make_inputs", "random_inputs", "random_cotangent",
           "algorithmic_counts", "describe"]
