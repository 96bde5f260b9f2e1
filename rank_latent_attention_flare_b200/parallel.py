"""Context parallelism over torch.distributed: every rank holds an equal
shard of each sequence's tokens (the FLARE++ page: the input tokens sharded
across devices, never gathered).

Forward: each rank encodes its shard into chunk records, the records are
all-gathered (the only exchange), every rank merges them into the whole
sequence's Z and decodes its own tokens.  Backward: each rank's part of dZ
is all-reduced between the decode and the encode stage, and the parts of dQ
at the end.  Argument marshalling and collectives only: the math runs in
libflare.so.  ``ops`` defaults to this package's stage calls; the
multi-process CPU tests pass stand-ins with the same signatures.
"""
from __future__ import annotations

import importlib
from typing import Optional

import torch
import torch.distributed as dist

# the binding module (the package's `flare` attribute is the autograd function)
_f = importlib.import_module(__package__ + ".flare")


def _encode_and_merge(ops, Q, K, V, s, ws, group, **outs):
    """Encodes this rank's shard, all-gathers every rank's records (rank
    order) and merges them into the whole sequence's Z in ``ws``."""
    B, H, N, M, D, _ = _f._dims(Q, K)
    ops.flare_encode(Q, K, V, s, workspace=ws)
    ml, acc = ops.encode_records(ws, B, H, N, M, D, K.dtype)
    G = dist.get_world_size(group)
    # gathered along the first dimension (rank order), then viewed as [shards, ...]
    gml = torch.empty((G * ml.shape[0],) + tuple(ml.shape[1:]), dtype=ml.dtype, device=ml.device)
    gacc = torch.empty((G * acc.shape[0],) + tuple(acc.shape[1:]), dtype=acc.dtype,
                       device=acc.device)
    dist.all_gather_into_tensor(gml, ml.contiguous(), group=group)
    dist.all_gather_into_tensor(gacc, acc.contiguous(), group=group)
    ops.flare_combine_shards(gml.view((G,) + tuple(ml.shape)), gacc.view((G,) + tuple(acc.shape)),
                             B, H, N, M, D, K.dtype, workspace=ws, **outs)


def cp_flare_fwd(Q, K, V, scale: Optional[float] = None, *, group=None, save: bool = False,
                 ops=_f):
    """K, V: this rank's shard [B,H,N_r,D] of every sequence (the same N_r on
    every rank; shards in rank order).  Returns this rank's Y shard, or
    (Y, Z, lse) of the whole sequence when ``save``."""
    B, H, N, M, D, _ = _f._dims(Q, K)
    s = _f.default_scale(D) if scale is None else float(scale)
    ws = ops.alloc_workspace(_f._lib.FLARE_OP_FWD, B, H, N, M, D, K.dtype, K.device)
    Z = torch.empty((B, H, M, D), dtype=torch.float32, device=K.device)
    lse = torch.empty((B, H, M), dtype=torch.float32, device=K.device)
    _encode_and_merge(ops, Q, K, V, s, ws, group, Z_save=Z, lse_save=lse)
    Y = ops.flare_decode(Q, K, s, workspace=ws)
    return (Y, Z, lse) if save else Y


def cp_flare_bwd(Q, K, V, dY, Z, lse, scale: Optional[float] = None, *, group=None, ops=_f,
                 workspace=None):
    """Gradients for this rank's shard (Z, lse: the whole sequence's, from
    cp_flare_fwd(save=True)).  Returns (dQ summed over the shards, in Q's
    dtype; this shard's dK, dV)."""
    dQ, dK, dV = _cp_bwd32(Q, K, V, dY, Z, lse, scale, group, ops, workspace)
    return dQ.to(Q.dtype), dK, dV


def _cp_bwd32(Q, K, V, dY, Z, lse, scale, group, ops, ws):
    B, H, N, M, D, _ = _f._dims(Q, K)
    s = _f.default_scale(D) if scale is None else float(scale)
    if ws is None:
        ws = ops.alloc_workspace(_f._lib.FLARE_OP_BWD, B, H, N, M, D, K.dtype, K.device)
    dZ = ops.flare_bwd_shard_dz(Q, K, V, dY, Z, lse, s, workspace=ws)
    dist.all_reduce(dZ, group=group)
    dQ, dK, dV = ops.flare_bwd_shard_finish(Q, K, V, dY, Z, lse, dZ, s, workspace=ws)
    dist.all_reduce(dQ, group=group)
    return dQ, dK, dV


def cp_flare_pp_fwd(Q, K, V, scale: Optional[float] = None, *, group=None, save: bool = False,
                    ops=_f):
    """FLARE++ with learned latents Q [H,M,D] over token shards: two record
    exchanges (the first encode, which gives Q_dyn = Q + Z1, and the second
    with Q_dyn).  Returns (Y shard, Q_dyn), or (Y, Q_dyn, Z, lse) when
    ``save`` (Z, lse: the second encode's, whole sequence)."""
    B, H, N, M, D, qbs = _f._dims(Q, K)
    if qbs != 0:
        raise ValueError("FLARE++ takes learned latents Q of shape [H,M,D]")
    s = _f.default_scale(D) if scale is None else float(scale)
    ws = ops.alloc_workspace(_f._lib.FLARE_OP_FWD, B, H, N, M, D, K.dtype, K.device)
    Qd = torch.empty((B, H, M, D), dtype=K.dtype, device=K.device)
    _encode_and_merge(ops, Q, K, V, s, ws, group, Q_learned=Q, Q_dyn_out=Qd)
    Z = torch.empty((B, H, M, D), dtype=torch.float32, device=K.device)
    lse = torch.empty((B, H, M), dtype=torch.float32, device=K.device)
    _encode_and_merge(ops, Qd, K, V, s, ws, group, Z_save=Z, lse_save=lse)
    Y = ops.flare_decode(Qd, K, s, workspace=ws)
    return (Y, Qd, Z, lse) if save else (Y, Qd)


def cp_flare_pp_bwd(Q, K, V, dY, Q_dyn, Z, lse, scale: Optional[float] = None, *, group=None,
                    ops=_f):
    """FLARE++ gradients for this rank's shard (Q_dyn, Z, lse from
    cp_flare_pp_fwd(save=True)).  Returns (dQ [H,M,D] in Q's dtype; this
    shard's dK, dV)."""
    B, H, N, M, D, _ = _f._dims(Q, K)
    s = _f.default_scale(D) if scale is None else float(scale)
    # the first encode, recomputed: Z1, lse1 of the whole sequence
    wsf = ops.alloc_workspace(_f._lib.FLARE_OP_FWD, B, H, N, M, D, K.dtype, K.device)
    Z1 = torch.empty((B, H, M, D), dtype=torch.float32, device=K.device)
    lse1 = torch.empty((B, H, M), dtype=torch.float32, device=K.device)
    _encode_and_merge(ops, Q, K, V, s, wsf, group, Z_save=Z1, lse_save=lse1)
    # FLARE's backward with the per-batch latents Q_dyn, then the first encode's
    ws = ops.alloc_workspace(_f._lib.FLARE_OP_PP_BWD, B, H, N, M, D, K.dtype, K.device)
    dQd, dK, dV = _cp_bwd32(Q_dyn, K, V, dY, Z, lse, s, group, ops, ws)
    # rank 0's part also carries the sum over the batch of dQ_dyn, so the
    # all-reduced parts are the whole dQ
    dQp = ops.flare_pp_bwd_shard_tail(Q, K, V, Z1, lse1, dQd.to(K.dtype), dK, dV, s, workspace=ws,
                                      add_dq_dyn=dist.get_rank(group) == 0)
    dist.all_reduce(dQp, group=group)
    return dQp.to(Q.dtype), dK, dV
