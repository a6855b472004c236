"""Token-sharded (context-parallel) FLARE++ mixer forward over torch.distributed.

Each rank holds its own slice of the N tokens (k0, k, v and y of this rank's
tokens) and the replicated latent inputs (q0, q_fixed, gate).  The split
softmax passes run on the local tokens and are reduced to one triple per latent
row; the ranks' triples are all-gathered (NCCL over NVLink on GPUs) and merged
by log-sum-exp, which rebuilds the globally normalised attention exactly up to
rounding; the decode stays local (physicsnemo issue #2024, section 2).  Two
all-gathers per call (synthesis and encode; one for the closed gate), each of
B*H*M*(D+2) fp32 per rank: the exchange depends on M and D, not on N.

The stages are the C entries flarepp_cp_partials / flarepp_cp_merge /
flarepp_cp_decode; this module only allocates buffers and calls the
collective between them.

The backward (``mixer_bwd_cp``) runs the forward's sharded passes again,
keeping the per-latent log-sum-exps, then the four stages of
flarepp_cp_bwd_stage with an all-reduce (sum) of a latent-sized fp32 region
of the per-rank state after each of the first three: every sum over tokens
in the backward is a sum of per-rank sums.
"""

import torch
import torch.distributed as dist

from . import binding as _b


def shard_bounds(N: int, ranks: int, rank: int):
    """Token range [lo, hi) of `rank` when N tokens are split over `ranks` as
    evenly as possible (the first N % ranks ranks take one token more)."""
    if ranks < 1 or not 0 <= rank < ranks:
        raise ValueError("rank must lie in [0, ranks)")
    if N < ranks:
        raise ValueError(f"{N} tokens cannot give each of {ranks} ranks at least one")
    base, extra = divmod(N, ranks)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def _all_gather(t: torch.Tensor, group) -> torch.Tensor:
    """The ranks' buffers back to back in rank order, flat: one
    all_gather_into_tensor, the same call on NCCL (device buffers) and on gloo
    (host buffers, as in the multi-process tests)."""
    if not dist.is_initialized():
        return t.reshape(-1)
    ranks = dist.get_world_size(group)
    out = torch.empty(ranks * t.numel(), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous().reshape(-1), group=group)
    return out


def _all_reduce(t: torch.Tensor, group) -> torch.Tensor:
    """In-place sum over the ranks (one collective)."""
    if dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def mixer_bwd_cp(q0, q_fixed, gate, k0, k, v, dy, *, group=None, layout: str = "bhnd", path: int = _b.PATH_AUTO,
                 scale: float = 0.0, force_chunks: int = 0, norm_synthesis: bool = False, _ops=None, _gather=None,
                 _reduce=None) -> dict:
    """Gradients of the FLARE++ mixer with the tokens sharded over the ranks of `group`.

    Inputs as for ``mixer_fwd_cp`` plus dy (this rank's tokens, the layout of k).
    Returns dk, dv (and dk0) for this rank's tokens and dq_fixed (and dq0,
    dgate), the same on every rank.  ``_ops``, ``_gather`` and ``_reduce``
    replace the library stages and the collectives (tests)."""
    ops = _ops or _b
    gather = _gather or _all_gather
    reduce = _reduce or _all_reduce
    B, H, N, M, D = _b._shapes(q_fixed, k, layout)
    if N < 1:
        raise ValueError("every rank needs at least one token")
    dt = _b._dtype_code(k)
    dev = k.device
    gated = gate is not None
    ranks = dist.get_world_size(group) if dist.is_initialized() else 1
    common = dict(B=B, H=H, M=M, D=D)
    tok = dict(N=N, path=path, scale=scale, layout=layout)
    f32 = dict(dtype=torch.float32, device=dev)
    # the forward's sharded passes, keeping the log-sum-exps and the pre-gate synthesis output
    triple = torch.empty(ops.cp_triple_bytes(B, H, M, D) // 4, **f32)
    lat_bytes = ops.cp_latent_bytes(B, H, M, D, dt)
    lse_enc = torch.empty((B, H, M), **f32)
    lse_syn = qdyn = qs = None
    if gated:
        lse_syn = torch.empty((B, H, M), **f32)
        qdyn = torch.empty((B, H, M, D), **f32)
        ops.cp_partials(q0, True, k0, k0, triple, force_chunks=force_chunks, norm_synthesis=norm_synthesis,
                        **common, **tok)
        qs = torch.empty(lat_bytes, dtype=torch.uint8, device=dev)
        ops.cp_merge(gather(triple, group), ranks, q_fixed, gate, qs, dtype=dt, lse_out=lse_syn, pregate_out=qdyn,
                     **common)
        ops.cp_partials(qs, False, k, v, triple, force_chunks=force_chunks, **common, **tok)
    else:
        ops.cp_partials(q_fixed, True, k, v, triple, force_chunks=force_chunks, **common, **tok)
    zs = torch.empty(lat_bytes, dtype=torch.uint8, device=dev)
    ops.cp_merge(gather(triple, group), ranks, None, None, zs, dtype=dt, lse_out=lse_enc, **common)

    grads = {"dk": torch.empty_like(k), "dv": torch.empty_like(v), "dq_fixed": torch.empty((H, M, D), **f32)}
    if gated:
        grads.update(dk0=torch.empty_like(k0), dq0=torch.empty((H, M, D), **f32), dgate=torch.empty((H,), **f32))
    lay = ops.cp_bwd_layout(B, H, N, M, D, dt, path=path, scale=scale, force_chunks=force_chunks, layout=layout,
                            norm_synthesis=norm_synthesis)
    state = torch.empty(lay.bytes, dtype=torch.uint8, device=dev)
    for stage in (1, 2, 3, 4):
        ops.cp_bwd_stage(stage, q0, q_fixed, gate, qs, zs, lse_syn, lse_enc, qdyn, k0, k, v, dy, grads, state,
                         N=N, path=path, scale=scale, force_chunks=force_chunks, layout=layout,
                         norm_synthesis=norm_synthesis, **common)
        if stage < 4 and (gated or stage < 3):
            off, nbytes = lay.reduce_offset[stage - 1], lay.reduce_bytes[stage - 1]
            reduce(state[off:off + nbytes].view(torch.float32), group)
    return grads


def mixer_fwd_cp(q0, q_fixed, gate, k0, k, v, y=None, *, group=None, layout: str = "bhnd",
                 path: int = _b.PATH_AUTO, scale: float = 0.0, force_chunks: int = 0,
                 return_qz: bool = False, norm_synthesis: bool = False, _ops=None, _gather=None):
    """FLARE++ mixer forward with the tokens sharded over the ranks of `group`.

    q0, q_fixed [H,M,D] and gate fp32 [H] (or None: FLARE) are the same on every
    rank; k0, k, v are this rank's tokens, [B,H,N_r,D] or [B,N_r,H,D]
    (``layout``).  Returns this rank's y (and the merged q, z as fp32
    [B,H,M,D] when ``return_qz``; identical on every rank).  ``norm_synthesis``
    RMS-normalises the q0 and k0 rows in the synthesis pass.

    ``_ops`` and ``_gather`` replace the library stages and the collective
    (tests of the orchestration on CPU ranks); the default is the CUDA library
    and torch.distributed."""
    ops = _ops or _b
    gather = _gather or _all_gather
    B, H, N, M, D = _b._shapes(q_fixed, k, layout)
    if N < 1:
        raise ValueError("every rank needs at least one token")
    dt = _b._dtype_code(k)
    dev = k.device
    gated = gate is not None
    ranks = dist.get_world_size(group) if dist.is_initialized() else 1
    common = dict(B=B, H=H, M=M, D=D)
    tok = dict(N=N, path=path, scale=scale, layout=layout)
    triple = torch.empty(ops.cp_triple_bytes(B, H, M, D) // 4, dtype=torch.float32, device=dev)
    lat_bytes = ops.cp_latent_bytes(B, H, M, D, dt)
    if gated:
        ops.cp_partials(q0, True, k0, k0, triple, force_chunks=force_chunks, norm_synthesis=norm_synthesis,
                        **common, **tok)
        qs = torch.empty(lat_bytes, dtype=torch.uint8, device=dev)
        ops.cp_merge(gather(triple, group), ranks, q_fixed, gate, qs, dtype=dt, **common)
        ops.cp_partials(qs, False, k, v, triple, force_chunks=force_chunks, **common, **tok)
    else:
        qs = None
        ops.cp_partials(q_fixed, True, k, v, triple, force_chunks=force_chunks, **common, **tok)
    zs = torch.empty(lat_bytes, dtype=torch.uint8, device=dev)
    ops.cp_merge(gather(triple, group), ranks, None, None, zs, dtype=dt, **common)
    if y is None:
        y = torch.empty_like(k)
    ops.cp_decode(qs if gated else q_fixed, not gated, zs, k, y, **common, **tok)
    if not return_qz:
        return y
    n = B * H * M * D
    z32 = zs.view(torch.float32)[:n].view(B, H, M, D)
    if gated:
        q32 = qs.view(torch.float32)[:n].view(B, H, M, D)
    else:
        q32 = q_fixed.float().unsqueeze(0).expand(B, H, M, D).contiguous()
    return y, q32, z32
