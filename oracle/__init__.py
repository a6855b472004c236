"""fp64 CPU oracle for the FLARE++ mixer forward.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference leg may import this package.  The
product path (``rank_latent_attention_mixer_b200``) never imports it and shares
no code with it.

The arithmetic lives in ``flarepp_oracle.c`` (plain C, fp64, libm ``exp``, no
fast-math), which restates the FLARE++ block of the FLARE.py README ("FLARE++"
code block: three scaled-dot-product-attention calls) and the FLARE block of
the same README.  This module only compiles it, marshals numpy arrays and
returns fp64 results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flarepp_oracle.c")
_LOCK = threading.Lock()
_LIBS: dict[int, ctypes.CDLL] = {}

_i64 = ctypes.c_int64
_dp = ctypes.POINTER(ctypes.c_double)


def library_path(plant: int = 0) -> str:
    name = "liboracle_flarepp.so" if plant == 0 else f"liboracle_flarepp_plant{plant}.so"
    return os.path.join(_HERE, name)


def build(plant: int = 0, force: bool = False) -> str:
    """Compile the oracle (``plant`` > 0 compiles a variant with a planted mistake,
    used only by the test that checks that the pins catch such mistakes)."""
    out = library_path(plant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           f"-DORACLE_PLANT={plant}", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _lib(plant: int = 0) -> ctypes.CDLL:
    with _LOCK:
        if plant not in _LIBS:
            lib = ctypes.CDLL(build(plant))
            lib.oracle_sdpa.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, ctypes.c_double]
            lib.oracle_sdpa.restype = ctypes.c_int
            lib.oracle_flarepp.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                           _i64, _i64, _i64, _i64, _i64, ctypes.c_double, ctypes.c_int]
            lib.oracle_flarepp.restype = ctypes.c_int
            lib.oracle_flarepp_head.argtypes = [_dp, _dp, ctypes.c_double, _dp, _dp, _dp,
                                                ctypes.POINTER(ctypes.c_int64), _i64, _dp, _dp, _dp,
                                                _i64, _i64, _i64, ctypes.c_double, ctypes.c_int]
            lib.oracle_flarepp_head.restype = ctypes.c_int
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_plant.restype = ctypes.c_int
            _LIBS[plant] = lib
        return _LIBS[plant]


def _f64(a) -> np.ndarray:
    """Contiguous fp64 numpy copy of an array-like (torch tensors included; bf16 widens exactly)."""
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu", torch.float64).contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def sdpa(Q, K, V, scale: float = 0.0, plant: int = 0) -> np.ndarray:
    """SDPA(Q[Lq,D], K[Lk,D], V[Lk,D]) for one slice, fp64.  scale <= 0 means 1/sqrt(D)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Lq, D = Q.shape
    Lk = K.shape[0]
    assert K.shape == (Lk, D) and V.shape == (Lk, D)
    O = np.empty((Lq, D), np.float64)
    rc = _lib(plant).oracle_sdpa(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), Lq, Lk, D, float(scale))
    if rc:
        raise ValueError(f"oracle_sdpa failed with code {rc}")
    return O


NORM_EPS = 1e-6


def rms_normalise(x, eps: float = NORM_EPS, plant: int = 0) -> np.ndarray:
    """Head-wise normalisation of the synthesis seeds and keys/values
    (physicsnemo issue #2024, FLARE++ list: "Normalizing the synthesis call"),
    read as RMS over the head dimension without a learned scale:
    x / sqrt(mean_d x^2 + eps), row by row, in fp64.
    Planted mistakes (test use): 11 divides by the row's L2 norm instead."""
    x = _f64(x)
    if plant == 11:
        return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def flarepp(q0, q_fixed, gate, k0, k, v, scale: float = 0.0, flare: bool = False,
            plant: int = 0, norm_synthesis: bool = False):
    """Full mixer in fp64.  Returns (y [B,H,N,D], q [B,H,M,D], z [B,H,M,D]).

    ``gate`` is sigmoid(g) per head ([H]); ``gate=None`` or ``flare=True`` is the
    closed gate, i.e. FLARE with q = q_fixed.  ``norm_synthesis`` applies
    rms_normalise to the seeds q0 and the synthesis keys/values k0 first.
    Planted mistakes (test use): 12 normalises the seeds but not k0.
    """
    q_fixed, k, v = _f64(q_fixed), _f64(k), _f64(v)
    B, H, N, D = k.shape
    M = q_fixed.shape[1]
    assert q_fixed.shape == (H, M, D) and v.shape == (B, H, N, D)
    closed = flare or gate is None
    q0a = None if closed else _f64(q0)
    k0a = None if closed else _f64(k0)
    if norm_synthesis and not closed:
        q0a = np.ascontiguousarray(rms_normalise(q0a, plant=plant))
        if plant != 12:
            k0a = np.ascontiguousarray(rms_normalise(k0a, plant=plant))
    plant = plant if plant <= 10 else 0          # 11, 12 live above, not in the C build
    ga = None if closed else _f64(gate).reshape(H)
    if not closed:
        assert q0a.shape == (H, M, D) and k0a.shape == (B, H, N, D)
    y = np.empty((B, H, N, D), np.float64)
    q = np.empty((B, H, M, D), np.float64)
    z = np.empty((B, H, M, D), np.float64)
    rc = _lib(plant).oracle_flarepp(_ptr(q0a), _ptr(q_fixed), _ptr(ga), _ptr(k0a), _ptr(k), _ptr(v),
                                    _ptr(y), _ptr(q), _ptr(z), B, H, N, M, D, float(scale),
                                    1 if closed else 0)
    if rc:
        raise ValueError(f"oracle_flarepp failed with code {rc}")
    return y, q, z


def flarepp_head(q0_h, q_fixed_h, gate_h, k0_bh, k_bh, v_bh, tokens, scale: float = 0.0,
                 flare: bool = False, plant: int = 0):
    """One (b, h) slice: q and z [M,D] in full, y at the listed tokens [len(tokens), D]."""
    q_fixed_h, k_bh, v_bh = _f64(q_fixed_h), _f64(k_bh), _f64(v_bh)
    N, D = k_bh.shape
    M = q_fixed_h.shape[0]
    q0a = None if flare else _f64(q0_h)
    k0a = None if flare else _f64(k0_bh)
    tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
    y = np.empty((tok.size, D), np.float64)
    q = np.empty((M, D), np.float64)
    z = np.empty((M, D), np.float64)
    rc = _lib(plant).oracle_flarepp_head(
        _ptr(q0a), _ptr(q_fixed_h), float(0.0 if flare else gate_h), _ptr(k0a), _ptr(k_bh), _ptr(v_bh),
        tok.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), tok.size, _ptr(y), _ptr(q), _ptr(z),
        N, M, D, float(scale), 1 if flare else 0)
    if rc:
        raise ValueError(f"oracle_flarepp_head failed with code {rc}")
    return y, q, z
