"""fp64 CPU oracle for the gradients of the FLARE++ mixer.

TEST INFRASTRUCTURE ONLY (same rules as the rest of ``oracle/``).

The forward is the FLARE++ block of the FLARE.py README ("FLARE++" code
block, three scaled-dot-product-attention calls):

    q_dyn = SDPA(q0, k0, k0);  q = q_fixed + gate * q_dyn;  z = SDPA(q, k, v);  y = SDPA(k, q, z)

and this module returns the gradients of a scalar loss L with dL/dy = dy with
respect to q0, q_fixed, gate, k0, k and v, by the chain rule through each
softmax attention O = softmax(s Q K^T) V (row-wise softmax over the keys):

    dV = P^T dO,   dP = dO V^T,   dS = P * (dP - rowsum(P * dP)),
    dQ = s dS K,   dK = s dS^T Q

applied to the decode, the encode, the gate and the synthesis in that order
(q0 and q_fixed are shared by the batch, so their gradients sum over b; k0 is
both the keys and the values of the synthesis, so it collects both terms).
Plain numpy in fp64 with explicit [M, N] matrices per (b, h): for small cases.
"""
from __future__ import annotations

import numpy as np

from . import NORM_EPS, _f64


def _softmax_rows(S):
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    return E / E.sum(axis=1, keepdims=True)


def _sdpa_fwd(Q, K, V, s):
    P = _softmax_rows(s * (Q @ K.T))
    return P, P @ V


def _sdpa_bwd(Q, K, V, P, dO, s):
    """Gradients of O = softmax(s Q K^T) V with respect to Q, K and V."""
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - np.sum(P * dP, axis=1, keepdims=True))
    return s * (dS @ K), s * (dS.T @ Q), dV


def _rms_backward(x, g, eps=NORM_EPS):
    """Gradient through the row-wise RMS normalisation xh = x r,
    r = (mean_d x^2 + eps)^(-1/2), for the gradient g of xh: by the chain rule
    (dr/dx_j = -r^3 x_j / D) dx = r (g - xh <g, xh> / D), row by row."""
    D = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xh = x * r
    return r * (g - xh * np.sum(g * xh, axis=-1, keepdims=True) / D)


def flarepp_backward(q0, q_fixed, gate, k0, k, v, dy, scale: float = 0.0, norm_synthesis: bool = False):
    """Gradients of the gated mixer (gate open).  Returns a dict with
    dq0, dq_fixed [H,M,D], dgate [H], dk0, dk, dv [B,H,N,D], the forward's
    y [B,H,N,D], and the intermediates q_dyn and dq = dL/dq [B,H,M,D] (fp64).
    ``norm_synthesis``: the synthesis reads RMS-normalised q0 and k0 rows
    (physicsnemo issue #2024, "Normalizing the synthesis call"; the reading of
    ``rms_normalise``), and dq0, dk0 are taken through that step."""
    q0, q_fixed, gate = _f64(q0), _f64(q_fixed), _f64(gate).reshape(-1)
    k0, k, v, dy = _f64(k0), _f64(k), _f64(v), _f64(dy)
    if norm_synthesis:
        q0_raw, k0_raw = q0, k0
        q0 = q0_raw / np.sqrt(np.mean(q0_raw * q0_raw, axis=-1, keepdims=True) + NORM_EPS)
        k0 = k0_raw / np.sqrt(np.mean(k0_raw * k0_raw, axis=-1, keepdims=True) + NORM_EPS)
    B, H, N, D = k.shape
    M = q_fixed.shape[1]
    s = scale if scale > 0 else 1.0 / np.sqrt(D)
    g = {name: np.zeros_like(a) for name, a in
         (("dq0", q0), ("dq_fixed", q_fixed), ("dgate", gate), ("dk0", k0), ("dk", k), ("dv", v))}
    y = np.empty_like(k)
    q_dyn_all = np.empty((B, H, M, D))
    dq_all = np.empty((B, H, M, D))
    for b in range(B):
        for h in range(H):
            # forward, keeping the weights
            P_syn, q_dyn = _sdpa_fwd(q0[h], k0[b, h], k0[b, h], s)
            q = q_fixed[h] + gate[h] * q_dyn
            P_enc, z = _sdpa_fwd(q, k[b, h], v[b, h], s)
            P_dec, y[b, h] = _sdpa_fwd(k[b, h], q, z, s)
            # decode: y = SDPA(k, q, z)
            dk_a, dq_a, dz = _sdpa_bwd(k[b, h], q, z, P_dec, dy[b, h], s)
            # encode: z = SDPA(q, k, v)
            dq_b, dk_b, dv = _sdpa_bwd(q, k[b, h], v[b, h], P_enc, dz, s)
            dq = dq_a + dq_b
            q_dyn_all[b, h], dq_all[b, h] = q_dyn, dq
            # gate: q = q_fixed + gate * q_dyn
            g["dq_fixed"][h] += dq
            g["dgate"][h] += np.sum(dq * q_dyn)
            dq_dyn = gate[h] * dq
            # synthesis: q_dyn = SDPA(q0, k0, k0)
            dq0, dk0_keys, dk0_values = _sdpa_bwd(q0[h], k0[b, h], k0[b, h], P_syn, dq_dyn, s)
            g["dq0"][h] += dq0
            g["dk0"][b, h] = dk0_keys + dk0_values
            g["dk"][b, h] = dk_a + dk_b
            g["dv"][b, h] = dv
    if norm_synthesis:
        g["dq0"] = _rms_backward(q0_raw, g["dq0"])
        g["dk0"] = _rms_backward(k0_raw, g["dk0"])
    g["y"] = y
    g["q_dyn"], g["dq"] = q_dyn_all, dq_all
    return g
