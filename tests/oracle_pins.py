"""Pins for the fp64 oracle: checks that tie it to something other than itself.

Each check takes ``plant`` (0 = the oracle as committed, n > 0 = a build of
the oracle with planted mistake n) and returns True when the oracle passes it.
The committed oracle must pass every check; every planted mistake must fail at
least one (tests/test_oracle_mutations.py).

What each check pins the oracle to:

* torch's ``scaled_dot_product_attention`` in fp64 on the CPU -- the library
  routine the FLARE.py README's FLARE++ and FLARE blocks are written in;
* an independent numpy brute force that materialises each attention matrix,
  checks it is row-stochastic, and multiplies explicitly;
* closed forms of the definition: a two-token synthesis reduces to tanh,
  identical keys give the mean of the values, identical synthesis keys give
  q = q_fixed + gate * key, one token gives its value, one latent gives every
  token that latent's value, constant values pass through;
* invariants: closed gate equals the two-call FLARE form (physicsnemo issue
  #2024, "Fixed reference and gate"), decode outputs lie in the convex hull of
  the latents, equivariance under token permutation, invariance under token
  duplication, independence of batch elements and heads.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle

RTOL = 1e-11


def _rng(seed):
    return np.random.default_rng(seed)


def _inputs(seed, B, H, N, M, D, key_scale=1.0):
    r = _rng(seed)
    q0 = r.standard_normal((H, M, D))
    qf = r.standard_normal((H, M, D))
    gate = 1.0 / (1.0 + np.exp(-r.standard_normal(H)))
    k0 = r.standard_normal((B, H, N, D)) * key_scale
    k = r.standard_normal((B, H, N, D)) * key_scale
    v = r.standard_normal((B, H, N, D))
    return q0, qf, gate, k0, k, v


def _close(a, b, tol=RTOL):
    a, b = np.asarray(a), np.asarray(b)
    if a.shape != b.shape or not np.all(np.isfinite(a)):
        return False
    return float(np.max(np.abs(a - b))) <= tol * max(1.0, float(np.max(np.abs(b))))


def _torch_mixer(q0, qf, gate, k0, k, v, flare=False, scale=None):
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    B, H, N, D = k.shape
    M = qf.shape[1]
    kw = {} if scale is None else {"scale": scale}
    if flare:
        q = T(qf).expand(B, H, M, D)
    else:
        q_dyn = F.scaled_dot_product_attention(T(q0).expand(B, H, M, D), T(k0), T(k0), **kw)
        q = T(qf) + T(gate).view(H, 1, 1) * q_dyn
    z = F.scaled_dot_product_attention(q, T(k), T(v), **kw)
    y = F.scaled_dot_product_attention(T(k), q, z, **kw)
    return y.numpy(), q.numpy(), z.numpy()


# --------------------------------------------------------------------------- library routine

def pin_sdpa_vs_torch(plant):
    r = _rng(1)
    Q, K, V = r.standard_normal((7, 16)), r.standard_normal((33, 16)), r.standard_normal((33, 16))
    T = torch.from_numpy
    ok = _close(oracle.sdpa(Q, K, V, plant=plant), F.scaled_dot_product_attention(T(Q), T(K), T(V)).numpy())
    ok &= _close(oracle.sdpa(Q, K, V, scale=1.0, plant=plant),
                 F.scaled_dot_product_attention(T(Q), T(K), T(V), scale=1.0).numpy())
    return bool(ok)


def pin_mixer_vs_torch(plant):
    args = _inputs(2, 2, 3, 40, 5, 16)
    y, q, z = oracle.flarepp(*args, plant=plant)
    ty, tq, tz = _torch_mixer(*args)
    ok = _close(y, ty) and _close(q, tq) and _close(z, tz)
    yf, _, _ = oracle.flarepp(*args, flare=True, plant=plant)
    ok = ok and _close(yf, _torch_mixer(*args, flare=True)[0])
    return bool(ok)


def pin_mixer_vs_torch_scale1(plant):
    """The FLARE block's printed scale=1.0, through the scale argument."""
    args = _inputs(3, 1, 2, 25, 4, 32)
    y, _, _ = oracle.flarepp(*args, scale=1.0, flare=True, plant=plant)
    return _close(y, _torch_mixer(*args, flare=True, scale=1.0)[0])


# --------------------------------------------------------------------------- brute force

def _bf_attention(Q, K, V, scale):
    S = (Q @ K.T) * scale
    A = np.exp(S - S.max(axis=1, keepdims=True))
    A = A / A.sum(axis=1, keepdims=True)
    assert np.all(A >= 0.0) and np.allclose(A.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    return A @ V


def pin_bruteforce(plant):
    q0, qf, gate, k0, k, v = _inputs(4, 2, 2, 23, 6, 16, key_scale=1.5)
    B, H, N, D = k.shape
    sc = 1.0 / math.sqrt(D)
    y_ref = np.empty_like(k)
    q_ref = np.empty((B, H, qf.shape[1], D))
    z_ref = np.empty_like(q_ref)
    for b in range(B):
        for h in range(H):
            qd = _bf_attention(q0[h], k0[b, h], k0[b, h], sc)
            q_ref[b, h] = qf[h] + gate[h] * qd
            z_ref[b, h] = _bf_attention(q_ref[b, h], k[b, h], v[b, h], sc)
            y_ref[b, h] = _bf_attention(k[b, h], q_ref[b, h], z_ref[b, h], sc)
    y, q, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    return bool(_close(y, y_ref) and _close(q, q_ref) and _close(z, z_ref))


# --------------------------------------------------------------------------- closed forms

def pin_two_token_tanh(plant):
    """q0 = [a,0,0,0], k0 = [+1,0,0,0], [-1,0,0,0]: scores are +-a/2 (scale 1/sqrt(4)),
    so the synthesised query is [tanh(a/2), 0, 0, 0]."""
    a = 1.7
    q0 = np.zeros((1, 1, 4)); q0[0, 0, 0] = a
    k0 = np.zeros((1, 1, 2, 4)); k0[0, 0, 0, 0] = 1.0; k0[0, 0, 1, 0] = -1.0
    qf = np.zeros((1, 1, 4))
    gate = np.array([1.0])
    k = np.ones((1, 1, 2, 4)); v = np.ones((1, 1, 2, 4))
    _, q, _ = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    return _close(q[0, 0, 0], np.array([math.tanh(a / 2), 0.0, 0.0, 0.0]))


def pin_identical_keys_mean(plant):
    q0, qf, gate, k0, k, v = _inputs(5, 1, 2, 31, 5, 16)
    k[:] = k[:, :, :1, :]                      # every key equal -> uniform encode weights
    _, _, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    expect = np.broadcast_to(v.mean(axis=2, keepdims=True), z.shape)
    return _close(z, expect, 1e-12)


def pin_identical_synthesis_keys(plant):
    q0, qf, gate, k0, k, v = _inputs(6, 2, 3, 17, 4, 16)
    k0[:] = k0[:, :, :1, :]                    # q_dyn = the shared key
    _, q, _ = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    expect = qf[None] + gate[None, :, None, None] * k0[:, :, :1, :]
    return _close(q, expect, 1e-12)


def pin_single_token(plant):
    q0, qf, gate, k0, k, v = _inputs(7, 2, 2, 1, 5, 16)
    y, q, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    ok = _close(q, qf[None] + gate[None, :, None, None] * k0)
    ok = ok and _close(z, np.broadcast_to(v, z.shape)) and _close(y, v)
    return bool(ok)


def pin_single_latent(plant):
    q0, qf, gate, k0, k, v = _inputs(8, 2, 2, 29, 1, 16)
    y, _, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    return _close(y, np.broadcast_to(z, y.shape), 1e-13)


def pin_constant_values(plant):
    q0, qf, gate, k0, k, v = _inputs(9, 1, 2, 21, 6, 16)
    v[:] = v[:, :, :1, :]
    y, _, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    return bool(_close(z, np.broadcast_to(v[:, :, :1, :], z.shape), 1e-12)
                and _close(y, np.broadcast_to(v[:, :, :1, :], y.shape), 1e-12))


# --------------------------------------------------------------------------- invariants

def pin_closed_gate_is_flare(plant):
    q0, qf, gate, k0, k, v = _inputs(10, 2, 2, 19, 5, 16)
    y0, _, _ = oracle.flarepp(q0, qf, np.zeros_like(gate), k0, k, v, plant=plant)
    yf, _, _ = oracle.flarepp(q0, qf, None, k0, k, v, flare=True, plant=plant)
    y1, _, _ = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    return bool(np.array_equal(y0, yf) and not _close(y1, yf, 1e-6))


def pin_convex_hull(plant):
    q0, qf, gate, k0, k, v = _inputs(11, 1, 3, 37, 6, 16, key_scale=2.0)
    y, _, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    lo = z.min(axis=2, keepdims=True) - 1e-12
    hi = z.max(axis=2, keepdims=True) + 1e-12
    return bool(np.all(y >= lo) and np.all(y <= hi))


def pin_permutation(plant):
    q0, qf, gate, k0, k, v = _inputs(12, 1, 2, 26, 4, 16)
    perm = _rng(99).permutation(k.shape[2])
    y, q, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    yp, qp, zp = oracle.flarepp(q0, qf, gate, k0[:, :, perm], k[:, :, perm], v[:, :, perm], plant=plant)
    return bool(_close(qp, q) and _close(zp, z) and _close(yp, y[:, :, perm]))


def pin_duplication(plant):
    q0, qf, gate, k0, k, v = _inputs(13, 1, 2, 15, 4, 16)
    idx = np.repeat(np.arange(k.shape[2]), 2)
    y, q, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    yd, qd, zd = oracle.flarepp(q0, qf, gate, k0[:, :, idx], k[:, :, idx], v[:, :, idx], plant=plant)
    return bool(_close(qd, q) and _close(zd, z) and _close(yd, y[:, :, idx]))


def pin_batch_head_independence(plant):
    q0, qf, gate, k0, k, v = _inputs(14, 3, 2, 18, 4, 16)
    y, q, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    ok = True
    for b in range(3):
        for h in range(2):
            ys, qs, zs = oracle.flarepp(q0[h:h + 1], qf[h:h + 1], gate[h:h + 1], k0[b:b + 1, h:h + 1],
                                        k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], plant=plant)
            ok = ok and _close(ys[0, 0], y[b, h]) and _close(qs[0, 0], q[b, h]) and _close(zs[0, 0], z[b, h])
    return bool(ok)


def pin_head_slice_entry(plant):
    """The sampled entry (one head, chosen tokens) agrees with the full entry."""
    q0, qf, gate, k0, k, v = _inputs(15, 2, 2, 33, 5, 16)
    y, q, z = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    toks = [0, 7, 32, 7]
    ys, qs, zs = oracle.flarepp_head(q0[1], qf[1], gate[1], k0[1, 1], k[1, 1], v[1, 1], toks, plant=plant)
    return bool(_close(ys, y[1, 1, toks]) and _close(qs, q[1, 1]) and _close(zs, z[1, 1]))


def _unit_rows(seed, shape):
    """Rows of +-1 entries: mean of squares exactly 1 (RMS 1) in any dimension."""
    return np.where(_rng(seed).standard_normal(shape) < 0, -1.0, 1.0)


def pin_norm_scale_invariance(plant):
    """Normalised seeds and synthesis keys/values do not depend on the scale of
    q0 and k0 (inputs far from the epsilon)."""
    q0, qf, gate, k0, k, v = _inputs(21, 2, 2, 40, 6, 16)
    q0, k0 = q0 * 100.0, k0 * 100.0
    _, qa, _ = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant, norm_synthesis=True)
    _, qb, _ = oracle.flarepp(q0 * 3.0, qf, gate, k0 * 11.0, k, v, plant=plant, norm_synthesis=True)
    return _close(qa, qb, 1e-8)


def pin_norm_identical_keys(plant):
    """Every synthesis key equal to c*u with u of RMS 1: the values are the
    normalised key u, so q = q_fixed + gate * u."""
    q0, qf, gate, k0, k, v = _inputs(22, 2, 3, 17, 4, 16)
    u = _unit_rows(23, (2, 3, 1, 16))
    k0 = np.broadcast_to(1000.0 * u, k0.shape).copy()
    _, q, _ = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant, norm_synthesis=True)
    return _close(q, qf[None] + gate[None, :, None, None] * u, 1e-10)


def pin_norm_of_unit_rows(plant):
    """Seeds and keys whose rows already have RMS 1 pass the normalisation
    unchanged up to the epsilon (a factor 1/sqrt(1 + 1e-6))."""
    q0, qf, gate, k0, k, v = _inputs(24, 1, 2, 33, 5, 32)
    q0, k0 = _unit_rows(25, q0.shape), _unit_rows(26, k0.shape)
    ya, qa, za = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant, norm_synthesis=True)
    yb, qb, zb = oracle.flarepp(q0, qf, gate, k0, k, v, plant=plant)
    return _close(qa, qb, 1e-5) and _close(ya, yb, 1e-5)


PINS = {name[4:]: fn for name, fn in sorted(globals().items()) if name.startswith("pin_") and callable(fn)}
