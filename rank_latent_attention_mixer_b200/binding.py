"""Thin ctypes binding of the C ABI in include/flarepp.h.

Argument marshalling only: every step of the mixer runs in the CUDA library
``libflarepp.so`` built in this directory.  PyTorch provides device memory,
the current stream and scratch from its caching allocator.  There is no CPU
fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflarepp.so")

F32, BF16, F16 = 0, 1, 2
PATH_AUTO, PATH_SIMT, PATH_TCGEN05 = 0, 1, 2
LAYOUTS = {"bhnd": 0, "bnhd": 1}
STATUS = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED", 3: "ERR_CUDA",
          4: "ERR_WORKSPACE", 5: "ERR_TIMEOUT"}
EXPORTS = ["flarepp_mixer_fwd", "flare_fwd", "flarepp_mixer_fwd_ex", "flarepp_workspace_bytes",
           "flarepp_mixer_fwd_host", "flarepp_selected_path", "flarepp_check_device_status",
           "flarepp_status_string", "flarepp_abi_version", "flarepp_launches_per_call",
           "flarepp_mixer_bwd", "flarepp_mixer_bwd_workspace_bytes", "flarepp_mixer_bwd_launches",
           "flarepp_train_context_bytes", "flarepp_mixer_fwd_train", "flarepp_mixer_bwd_ctx",
           "flarepp_set_workspace", "flarepp_mixer_fwd_debug"]


class FlareppError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


class Options(ctypes.Structure):
    """flarepp_options_t."""
    _fields_ = [("scale", ctypes.c_float), ("path", ctypes.c_int), ("force_chunks", ctypes.c_int),
                ("n_stage_events", ctypes.c_int), ("q_out", ctypes.c_void_p), ("z_out", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("stage_events", ctypes.POINTER(ctypes.c_void_p)), ("layout", ctypes.c_int),
                ("norm_synthesis", ctypes.c_int)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m rank_latent_attention_mixer_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i = ctypes.c_void_p, ctypes.c_int
    sig = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i]
    lib.flarepp_mixer_fwd.argtypes = sig + [vp]
    lib.flarepp_mixer_fwd_ex.argtypes = sig + [ctypes.POINTER(Options), vp]
    lib.flarepp_mixer_fwd_host.argtypes = sig + [vp]
    lib.flare_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.flarepp_workspace_bytes.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(Options)]
    lib.flarepp_workspace_bytes.restype = ctypes.c_size_t
    lib.flarepp_selected_path.argtypes = [i, i, i, i, i, i]
    lib.flarepp_check_device_status.argtypes = [vp]
    lib.flarepp_status_string.argtypes = [i]
    lib.flarepp_status_string.restype = ctypes.c_char_p
    lib.flarepp_launches_per_call.argtypes = [i]
    lib.flarepp_mixer_bwd.argtypes = [vp] * 13 + [i] * 6 + [ctypes.POINTER(Options), vp]
    lib.flarepp_mixer_bwd_workspace_bytes.argtypes = [i] * 6 + [ctypes.POINTER(Options)]
    lib.flarepp_mixer_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.flarepp_mixer_bwd_launches.argtypes = [i, i]
    lib.flarepp_train_context_bytes.argtypes = [i] * 6
    lib.flarepp_train_context_bytes.restype = ctypes.c_size_t
    lib.flarepp_mixer_fwd_train.argtypes = sig + [ctypes.POINTER(Options), vp, ctypes.c_size_t, vp]
    lib.flarepp_mixer_bwd_ctx.argtypes = [vp] * 14 + [i] * 6 + [ctypes.POINTER(Options), vp, ctypes.c_size_t, vp]
    lib.flarepp_set_workspace.argtypes = [vp, ctypes.c_size_t]
    lib.flarepp_mixer_fwd_debug.argtypes = sig + [vp, vp, i, vp]
    for name in ("flarepp_mixer_fwd", "flarepp_mixer_fwd_ex", "flarepp_mixer_fwd_host", "flare_fwd",
                 "flarepp_selected_path", "flarepp_check_device_status", "flarepp_abi_version",
                 "flarepp_launches_per_call", "flarepp_mixer_bwd", "flarepp_mixer_bwd_launches",
                 "flarepp_mixer_fwd_train", "flarepp_mixer_bwd_ctx", "flarepp_set_workspace",
                 "flarepp_mixer_fwd_debug"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load()
ABI_VERSION = 5
if lib.flarepp_abi_version() != ABI_VERSION:
    raise ImportError(f"{LIB_PATH} has ABI version {lib.flarepp_abi_version()}, this binding needs {ABI_VERSION}: "
                      "rebuild it")


def status_string(status: int) -> str:
    return lib.flarepp_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return F16
    raise TypeError(f"unsupported dtype {t.dtype}; the mixer takes float32, bfloat16 or float16")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(rc: int, where: str):
    if rc != 0:
        raise FlareppError(rc, where)


def _shapes(q_fixed: torch.Tensor, k: torch.Tensor, layout: str = "bhnd"):
    if k.dim() != 4 or q_fixed.dim() != 3:
        raise ValueError(f"expected q_fixed [H,M,D] and k [{','.join(layout.upper())}]")
    if layout == "bhnd":
        B, H, N, D = k.shape
    elif layout == "bnhd":
        B, N, H, D = k.shape
    else:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}")
    if q_fixed.shape[0] != H or q_fixed.shape[2] != D:
        raise ValueError(f"q_fixed {tuple(q_fixed.shape)} does not match k {tuple(k.shape)}")
    return B, H, N, q_fixed.shape[1], D


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous (the mixer reads row-major [.., D] rows)")


def launches_per_call(gated: bool = True) -> int:
    return int(lib.flarepp_launches_per_call(int(gated)))


def workspace_bytes(B, H, N, M, D, dtype=BF16, gated=True, path=PATH_AUTO, force_chunks=0, layout="bhnd",
                    norm_synthesis=False) -> int:
    o = Options(0.0, path, force_chunks, 0, None, None, None, 0, None, LAYOUTS[layout], int(norm_synthesis))
    return int(lib.flarepp_workspace_bytes(B, H, N, M, D, dtype, int(gated), ctypes.byref(o)))


def selected_path(B, H, N, M, D, dtype=BF16) -> int:
    return int(lib.flarepp_selected_path(B, H, N, M, D, dtype))


def mixer_fwd(q0, q_fixed, gate, k0, k, v, y=None, *, scale: float = 0.0, path: int = PATH_AUTO,
              force_chunks: int = 0, return_qz: bool = False, workspace: Optional[torch.Tensor] = None,
              stage_events=None, layout: str = "bhnd", norm_synthesis: bool = False):
    """FLARE++ mixer forward on the current CUDA stream.  ``gate=None`` is FLARE.

    q0, q_fixed [H,M,D]; gate fp32 [H] (sigmoid already applied); k0, k, v and y
    [B,H,N,D] (``layout="bhnd"``) or [B,N,H,D] (``layout="bnhd"``, read and
    written in place); all on the same CUDA device, contiguous, fp32, bf16 or
    fp16.  Returns y (and q, z fp32 [B,H,M,D] when ``return_qz``).
    ``stage_events``: torch.cuda.Event objects (created with enable_timing)
    recorded before the first launch and after each launch on the current stream.
    ``norm_synthesis``: RMS-normalise the q0 and k0 rows inside the synthesis pass."""
    B, H, N, M, D = _shapes(q_fixed, k, layout)
    _contig(q0, q_fixed, gate, k0, k, v, y)
    dt = _dtype_code(k)
    if y is None:
        y = torch.empty_like(k)
    q_out = z_out = None
    if return_qz:
        q_out = torch.empty((B, H, M, D), dtype=torch.float32, device=k.device)
        z_out = torch.empty((B, H, M, D), dtype=torch.float32, device=k.device)
    if gate is not None and gate.dtype != torch.float32:
        raise TypeError("gate must be float32 [H]")
    need = workspace_bytes(B, H, N, M, D, dt, gate is not None, path, force_chunks, layout, norm_synthesis)
    if need == 0:
        ws_ptr, ws_len = None, 0
    else:
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
        ws_ptr, ws_len = workspace.data_ptr(), workspace.numel()
    ev_arr, n_ev = None, 0
    if stage_events:
        handles = []
        for e in stage_events:
            if e.cuda_event == 0:          # torch creates the CUDA event lazily
                e.record()
            handles.append(e.cuda_event)
        n_ev = len(handles)
        ev_arr = (ctypes.c_void_p * n_ev)(*handles)
    o = Options(float(scale), int(path), int(force_chunks), n_ev, _ptr(q_out), _ptr(z_out), ws_ptr, ws_len,
                ctypes.cast(ev_arr, ctypes.POINTER(ctypes.c_void_p)) if ev_arr is not None else None,
                LAYOUTS[layout], int(norm_synthesis))
    rc = lib.flarepp_mixer_fwd_ex(_ptr(q0) if gate is not None else None, _ptr(q_fixed), _ptr(gate),
                                  _ptr(k0) if gate is not None else None, _ptr(k), _ptr(v), _ptr(y),
                                  B, H, N, M, D, dt, ctypes.byref(o), _stream(k.device))
    _check(rc, "flarepp_mixer_fwd_ex")
    return (y, q_out, z_out) if return_qz else y


def _event_array(stage_events):
    if not stage_events:
        return None, 0
    handles = []
    for e in stage_events:
        if e.cuda_event == 0:          # torch creates the CUDA event lazily
            e.record()
        handles.append(e.cuda_event)
    return (ctypes.c_void_p * len(handles))(*handles), len(handles)


def bwd_launches(gated: bool = True, path: int = PATH_SIMT) -> int:
    """Launches of one backward call whose forward runs on kernel family ``path`` (SIMT or TCGEN05)."""
    return int(lib.flarepp_mixer_bwd_launches(int(gated), int(path)))


def bwd_workspace_bytes(B, H, N, M, D, dtype=BF16, path=PATH_AUTO, force_chunks=0, layout="bhnd",
                        norm_synthesis=False) -> int:
    o = Options(0.0, path, force_chunks, 0, None, None, None, 0, None, LAYOUTS[layout], int(norm_synthesis))
    return int(lib.flarepp_mixer_bwd_workspace_bytes(B, H, N, M, D, dtype, ctypes.byref(o)))


def train_context_bytes(B, H, N, M, D, dtype=BF16) -> int:
    return int(lib.flarepp_train_context_bytes(B, H, N, M, D, dtype))


def mixer_fwd_train(q0, q_fixed, gate, k0, k, v, y=None, *, ctx: Optional[torch.Tensor] = None, scale: float = 0.0,
                    path: int = PATH_AUTO, force_chunks: int = 0, layout: str = "bhnd", norm_synthesis: bool = False,
                    workspace: Optional[torch.Tensor] = None):
    """flarepp_mixer_fwd_train: the forward, also saving the state its backward
    needs into ``ctx`` (a uint8 device tensor, allocated if None).  Returns (y, ctx)."""
    B, H, N, M, D = _shapes(q_fixed, k, layout)
    _contig(q0, q_fixed, gate, k0, k, v, y)
    dt = _dtype_code(k)
    if y is None:
        y = torch.empty_like(k)
    need = train_context_bytes(B, H, N, M, D, dt)
    if ctx is None or ctx.numel() < need:
        ctx = torch.empty(need, dtype=torch.uint8, device=k.device)
    wneed = workspace_bytes(B, H, N, M, D, dt, gate is not None, path, force_chunks, layout, norm_synthesis)
    if workspace is None or workspace.numel() < wneed:
        workspace = torch.empty(max(wneed, 1), dtype=torch.uint8, device=k.device)
    o = Options(float(scale), int(path), int(force_chunks), 0, None, None, workspace.data_ptr(), workspace.numel(),
                None, LAYOUTS[layout], int(norm_synthesis))
    rc = lib.flarepp_mixer_fwd_train(_ptr(q0) if gate is not None else None, _ptr(q_fixed), _ptr(gate),
                                     _ptr(k0) if gate is not None else None, _ptr(k), _ptr(v), _ptr(y),
                                     B, H, N, M, D, dt, ctypes.byref(o), ctx.data_ptr(), ctx.numel(),
                                     _stream(k.device))
    _check(rc, "flarepp_mixer_fwd_train")
    return y, ctx


def mixer_bwd(q0, q_fixed, gate, k0, k, v, dy, *, scale: float = 0.0, path: int = PATH_AUTO,
              force_chunks: int = 0, layout: str = "bhnd", workspace: Optional[torch.Tensor] = None,
              stage_events=None, out: Optional[dict] = None, norm_synthesis: bool = False,
              ctx: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None) -> dict:
    """Gradients of the FLARE++ mixer (flarepp_mixer_bwd) for the upstream gradient dy of y.

    Inputs as for ``mixer_fwd`` plus dy (the layout and dtype of k).  Returns a
    dict with dk, dv (and dk0 when gated) in the I/O dtype and token layout,
    dq_fixed (and dq0) fp32 [H,M,D], and dgate fp32 [H] (the gradient with
    respect to the gate value, not its logit).  ``gate=None`` is FLARE.
    ``out`` may supply preallocated gradient tensors under the same names.
    ``norm_synthesis``: the synthesis reads RMS-normalised q0, k0 rows, as in
    ``mixer_fwd``, and dq0, dk0 are taken through that step.
    ``ctx``, ``y``: the context and output of ``mixer_fwd_train`` on the same
    inputs and options (flarepp_mixer_bwd_ctx: no recomputed forward passes)."""
    B, H, N, M, D = _shapes(q_fixed, k, layout)
    _contig(q0, q_fixed, gate, k0, k, v, dy)
    dt = _dtype_code(k)
    gated = gate is not None
    if gated and gate.dtype != torch.float32:
        raise TypeError("gate must be float32 [H]")
    g = dict(out or {})
    dev = k.device
    g.setdefault("dk", torch.empty_like(k))
    g.setdefault("dv", torch.empty_like(v))
    g.setdefault("dq_fixed", torch.empty((H, M, D), dtype=torch.float32, device=dev))
    if gated:
        g.setdefault("dk0", torch.empty_like(k0))
        g.setdefault("dq0", torch.empty((H, M, D), dtype=torch.float32, device=dev))
        g.setdefault("dgate", torch.empty((H,), dtype=torch.float32, device=dev))
    need = bwd_workspace_bytes(B, H, N, M, D, dt, path, force_chunks, layout, norm_synthesis)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ev_arr, n_ev = _event_array(stage_events)
    o = Options(float(scale), int(path), int(force_chunks), n_ev, None, None,
                workspace.data_ptr() if need else None, workspace.numel() if need else 0,
                ctypes.cast(ev_arr, ctypes.POINTER(ctypes.c_void_p)) if ev_arr is not None else None,
                LAYOUTS[layout], int(norm_synthesis))
    grads = (_ptr(g.get("dq0")) if gated else None, _ptr(g["dq_fixed"]), _ptr(g.get("dgate")) if gated else None,
             _ptr(g.get("dk0")) if gated else None, _ptr(g["dk"]), _ptr(g["dv"]))
    ins = (_ptr(q0) if gated else None, _ptr(q_fixed), _ptr(gate), _ptr(k0) if gated else None, _ptr(k), _ptr(v))
    if ctx is not None:
        if y is None:
            raise ValueError("the context backward needs the forward's output y")
        rc = lib.flarepp_mixer_bwd_ctx(*ins, _ptr(y), _ptr(dy), *grads, B, H, N, M, D, dt, ctypes.byref(o),
                                       ctx.data_ptr(), ctx.numel(), _stream(dev))
        _check(rc, "flarepp_mixer_bwd_ctx")
        return g
    rc = lib.flarepp_mixer_bwd(*ins, _ptr(dy), *grads, B, H, N, M, D, dt, ctypes.byref(o), _stream(dev))
    _check(rc, "flarepp_mixer_bwd")
    return g


def mixer_fwd_plain(q0, q_fixed, gate, k0, k, v, y):
    """flarepp_mixer_fwd exactly as a C caller would make it (library-managed scratch)."""
    B, H, N, M, D = _shapes(q_fixed, k)
    _contig(q0, q_fixed, gate, k0, k, v, y)
    rc = lib.flarepp_mixer_fwd(_ptr(q0), _ptr(q_fixed), _ptr(gate), _ptr(k0), _ptr(k), _ptr(v), _ptr(y),
                               B, H, N, M, D, _dtype_code(k), _stream(k.device))
    _check(rc, "flarepp_mixer_fwd")
    return y


def mixer_fwd_debug(q0, q_fixed, gate, k0, k, v, y=None, *, force_chunks: int = 0):
    """flarepp_mixer_fwd_debug: y and the fp32 intermediates q, z [B,H,M,D]."""
    B, H, N, M, D = _shapes(q_fixed, k)
    _contig(q0, q_fixed, gate, k0, k, v, y)
    if y is None:
        y = torch.empty_like(k)
    q_out = torch.empty((B, H, M, D), dtype=torch.float32, device=k.device)
    z_out = torch.empty((B, H, M, D), dtype=torch.float32, device=k.device)
    rc = lib.flarepp_mixer_fwd_debug(_ptr(q0), _ptr(q_fixed), _ptr(gate), _ptr(k0), _ptr(k), _ptr(v), _ptr(y),
                                     B, H, N, M, D, _dtype_code(k), q_out.data_ptr(), z_out.data_ptr(),
                                     force_chunks, _stream(k.device))
    _check(rc, "flarepp_mixer_fwd_debug")
    return y, q_out, z_out


def set_workspace(buf: Optional[torch.Tensor]):
    """flarepp_set_workspace on the current device: a uint8 CUDA tensor the
    forward entries without an options workspace then use (None unregisters).
    The caller keeps the tensor alive while it is registered."""
    if buf is None:
        rc = lib.flarepp_set_workspace(None, 0)
    else:
        if not buf.is_cuda or not buf.is_contiguous():
            raise ValueError("the registered workspace must be a contiguous CUDA tensor")
        rc = lib.flarepp_set_workspace(buf.data_ptr(), buf.numel() * buf.element_size())
    _check(rc, "flarepp_set_workspace")


def flare_fwd(q, k, v, y=None):
    """FLARE (closed gate): z = SDPA(q,k,v), y = SDPA(k,q,z); q [H,M,D]."""
    B, H, N, M, D = _shapes(q, k)
    _contig(q, k, v, y)
    if y is None:
        y = torch.empty_like(k)
    rc = lib.flare_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(y), B, H, N, M, D, _dtype_code(k), _stream(k.device))
    _check(rc, "flare_fwd")
    return y


def mixer_fwd_host(q0, q_fixed, gate, k0, k, v, y, stream: Optional[torch.cuda.Stream] = None):
    """End-to-end form on HOST tensors (pinned for full copy speed): the library
    copies inputs in, runs, copies y out and synchronises the stream."""
    B, H, N, M, D = _shapes(q_fixed, k)
    _contig(q0, q_fixed, gate, k0, k, v, y)
    for t in (q0, q_fixed, gate, k0, k, v, y):
        if t is not None and t.is_cuda:
            raise ValueError("mixer_fwd_host takes host tensors")
    st = (stream or torch.cuda.current_stream()).cuda_stream
    rc = lib.flarepp_mixer_fwd_host(_ptr(q0), _ptr(q_fixed), _ptr(gate), _ptr(k0), _ptr(k), _ptr(v), _ptr(y),
                                    B, H, N, M, D, _dtype_code(k), st)
    _check(rc, "flarepp_mixer_fwd_host")
    return y


def mixer_fwd_noalloc(q0, q_fixed, gate, k0, k, v, y):
    """flarepp_mixer_fwd_noalloc: the mixer with no device allocation during
    the call (scratch comes from a fixed array inside the library; calls that
    overlap on the GPU race on it).  Same arguments and result as mixer_fwd_plain."""
    fn = lib.flarepp_mixer_fwd_noalloc
    if fn.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
        fn.restype = ctypes.c_int
    B, H, N, M, D = _shapes(q_fixed, k)
    _contig(q0, q_fixed, gate, k0, k, v, y)
    rc = fn(_ptr(q0), _ptr(q_fixed), _ptr(gate), _ptr(k0), _ptr(k), _ptr(v), _ptr(y),
            B, H, N, M, D, _dtype_code(k), _stream(k.device))
    _check(rc, "flarepp_mixer_fwd_noalloc")
    return y


# ---------------------------------------------------------------- token-sharded stages

def cp_triple_bytes(B, H, M, D) -> int:
    fn = lib.flarepp_cp_triple_bytes
    fn.argtypes = [ctypes.c_int] * 4
    fn.restype = ctypes.c_size_t
    return int(fn(B, H, M, D))


def cp_latent_bytes(B, H, M, D, dtype) -> int:
    fn = lib.flarepp_cp_latent_bytes
    fn.argtypes = [ctypes.c_int] * 5
    fn.restype = ctypes.c_size_t
    return int(fn(B, H, M, D, dtype))


def _cp_options(path, scale, force_chunks, layout, workspace=None, norm=False):
    ws_ptr, ws_len = (workspace.data_ptr(), workspace.numel()) if workspace is not None else (None, 0)
    return Options(float(scale), int(path), int(force_chunks), 0, None, None, ws_ptr, ws_len, None, LAYOUTS[layout],
                   int(norm))


def cp_partials(q, q_shared: bool, k, v, triple, *, B, H, N, M, D, path=PATH_AUTO, scale=0.0, force_chunks=0,
                layout="bhnd", norm_synthesis=False):
    """flarepp_cp_partials: this rank's split pass reduced to one triple per latent row
    (``norm_synthesis``: RMS-normalise this pass's q and k rows first)."""
    fn = lib.flarepp_cp_partials
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, i, vp, vp, vp, i, i, i, i, i, i, ctypes.POINTER(Options), vp]
    fn.restype = i
    o = _cp_options(path, scale, force_chunks, layout, norm=norm_synthesis)
    rc = fn(_ptr(q), int(q_shared), _ptr(k), _ptr(v), _ptr(triple), B, H, N, M, D, _dtype_code(k),
            ctypes.byref(o), _stream(k.device))
    _check(rc, "flarepp_cp_partials")
    return triple


def cp_merge(gathered, ranks: int, q_fixed, gate, state, *, B, H, M, D, dtype, lse_out=None, pregate_out=None):
    """flarepp_cp_merge: log-sum-exp merge of the gathered triples into a latent state
    (flarepp_cp_merge_ex when ``lse_out`` [B,H,M] or ``pregate_out`` [B,H,M,D], fp32, are given)."""
    vp, i = ctypes.c_void_p, ctypes.c_int
    if lse_out is None and pregate_out is None:
        fn = lib.flarepp_cp_merge
        fn.argtypes = [vp, i, vp, vp, vp, i, i, i, i, i, vp]
        fn.restype = i
        rc = fn(_ptr(gathered), int(ranks), _ptr(q_fixed), _ptr(gate), _ptr(state), B, H, M, D, dtype,
                _stream(gathered.device))
        _check(rc, "flarepp_cp_merge")
        return state
    fn = lib.flarepp_cp_merge_ex
    fn.argtypes = [vp, i, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    fn.restype = i
    rc = fn(_ptr(gathered), int(ranks), _ptr(q_fixed), _ptr(gate), _ptr(state), _ptr(lse_out), _ptr(pregate_out),
            B, H, M, D, dtype, _stream(gathered.device))
    _check(rc, "flarepp_cp_merge_ex")
    return state


class CpBwdLayout(ctypes.Structure):
    """flarepp_cp_bwd_layout_t."""
    _fields_ = [("bytes", ctypes.c_size_t), ("reduce_offset", ctypes.c_size_t * 3),
                ("reduce_bytes", ctypes.c_size_t * 3)]


def cp_bwd_layout(B, H, N, M, D, dtype, *, path=PATH_AUTO, scale=0.0, force_chunks=0, layout="bhnd",
                  norm_synthesis=False) -> CpBwdLayout:
    """flarepp_cp_bwd_layout: the per-rank state of the token-sharded backward and the
    regions to sum over the ranks after stages 1, 2, 3."""
    fn = lib.flarepp_cp_bwd_layout
    i = ctypes.c_int
    fn.argtypes = [i] * 6 + [ctypes.POINTER(Options), ctypes.POINTER(CpBwdLayout)]
    fn.restype = i
    out = CpBwdLayout()
    o = _cp_options(path, scale, force_chunks, layout, norm=norm_synthesis)
    _check(fn(B, H, N, M, D, dtype, ctypes.byref(o), ctypes.byref(out)), "flarepp_cp_bwd_layout")
    return out


def cp_bwd_stage(stage: int, q0, q_fixed, gate, q_state, z_state, lse_syn, lse_enc, qdyn, k0, k, v, dy, grads: dict,
                 state, *, B, H, N, M, D, path=PATH_AUTO, scale=0.0, force_chunks=0, layout="bhnd",
                 norm_synthesis=False):
    """flarepp_cp_bwd_stage: one stage of the token-sharded backward on this rank's tokens."""
    fn = lib.flarepp_cp_bwd_stage
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [i] + [vp] * 19 + [i] * 6 + [ctypes.POINTER(Options), vp]
    fn.restype = i
    o = _cp_options(path, scale, force_chunks, layout, norm=norm_synthesis)
    gated = gate is not None
    rc = fn(int(stage), _ptr(q0) if gated else None, _ptr(q_fixed), _ptr(gate), _ptr(q_state) if gated else None,
            _ptr(z_state), _ptr(lse_syn) if gated else None, _ptr(lse_enc), _ptr(qdyn) if gated else None,
            _ptr(k0) if gated else None, _ptr(k), _ptr(v), _ptr(dy),
            _ptr(grads.get("dq0")) if gated else None, _ptr(grads["dq_fixed"]),
            _ptr(grads.get("dgate")) if gated else None, _ptr(grads.get("dk0")) if gated else None,
            _ptr(grads["dk"]), _ptr(grads["dv"]), _ptr(state), B, H, N, M, D, _dtype_code(k), ctypes.byref(o),
            _stream(k.device))
    _check(rc, f"flarepp_cp_bwd_stage({stage})")


def cp_decode(q, q_shared: bool, z_state, k, y, *, B, H, N, M, D, path=PATH_AUTO, scale=0.0, layout="bhnd"):
    """flarepp_cp_decode: this rank's tokens decoded against the merged latents."""
    fn = lib.flarepp_cp_decode
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, i, vp, vp, vp, i, i, i, i, i, i, ctypes.POINTER(Options), vp]
    fn.restype = i
    o = _cp_options(path, scale, 0, layout)
    rc = fn(_ptr(q), int(q_shared), _ptr(z_state), _ptr(k), _ptr(y), B, H, N, M, D, _dtype_code(k),
            ctypes.byref(o), _stream(k.device))
    _check(rc, "flarepp_cp_decode")
    return y


def selftest_wait_timeout(limit_us: int = 20000, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Launches the bounded-wait self-test (a wait nothing satisfies); returns the launch status."""
    fn = lib.flarepp_selftest_wait_timeout
    fn.argtypes = [ctypes.c_void_p, ctypes.c_uint]
    fn.restype = ctypes.c_int
    st = (stream or torch.cuda.current_stream()).cuda_stream
    return int(fn(st, int(limit_us)))


def check_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    st = (stream or torch.cuda.current_stream()).cuda_stream
    return int(lib.flarepp_check_device_status(st))


def raw_call(name: str, *args) -> int:
    """Calls an exported entry with already-marshalled arguments (tests)."""
    return int(getattr(lib, name)(*args))
