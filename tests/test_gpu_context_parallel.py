"""Context parallelism on one GPU: the shards of each sequence are processed
one after another through the stage calls, their exchanges done by stacking
(the all-gather of the encode records) and summing (the all-reduces of dZ
and dQ).  The result must match the single-device call and the oracle."""
import math
import os

import pytest
import torch
import torch.distributed as dist

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import TOL_F32_GRAD_REL, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    (2, 2, 1536, 128, 32, torch.bfloat16, 2, False),   # tensor-core fwd and bwd, 2 shards
    (1, 2, 1536, 256, 32, torch.bfloat16, 3, False),   # tensor cores, M = 256
    (2, 2, 1536, 128, 16, torch.bfloat16, 4, True),    # per-batch latents
    (2, 2, 600, 32, 16, torch.float32, 3, False),      # CUDA-core fp32
]
IDS = ["tc_2", "tc_M256_3", "tc_D16_batchQ_4", "simt_f32_3"]


def _shards(t, G):
    return [c.contiguous() for c in t.chunk(G, dim=2)]


@pytest.mark.parametrize("B,H,N,M,D,dtype,G,batch_q", CASES, ids=IDS)
def test_sharded_forward_and_backward(B, H, N, M, D, dtype, G, batch_q):
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=101 + G, per_batch_q=batch_q, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Q = g["Q"]
    Ks, Vs, dYs = _shards(g["K"], G), _shards(g["V"], G), _shards(g["dY"], G)
    Nr = N // G
    # forward: encode each shard, stack the records, merge, decode each shard
    wss = [fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, Nr, M, D, dtype, DEV) for _ in range(G)]
    recs = []
    for r in range(G):
        fl.flare_encode(Q, Ks[r], Vs[r], s, workspace=wss[r])
        recs.append([t.clone() for t in fl.encode_records(wss[r], B, H, Nr, M, D, dtype)])
    gml = torch.stack([ml for ml, _ in recs])
    gacc = torch.stack([acc for _, acc in recs])
    Ys, Z, lse = [], None, None
    for r in range(G):
        Zr = torch.empty((B, H, M, D), dtype=torch.float32, device=DEV)
        lr = torch.empty((B, H, M), dtype=torch.float32, device=DEV)
        fl.flare_combine_shards(gml, gacc, B, H, Nr, M, D, dtype, workspace=wss[r], Z_save=Zr,
                                lse_save=lr)
        Ys.append(fl.flare_decode(Q, Ks[r], s, workspace=wss[r]))
        if Z is None:
            Z, lse = Zr, lr
        else:   # every shard merges the same records in the same order
            assert torch.equal(Zr, Z) and torch.equal(lr, lse)
    Y = torch.cat(Ys, dim=2)
    Y1, Z1, l1 = fl.flare_fwd(Q, g["K"], g["V"], s, save=True)
    Yo, Zo, lo = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Y, Yo, dtype, "Y (sharded)")
    assert_close(Z, Zo, dtype, "Z (sharded)")
    assert_close(Y, Y1.float(), dtype, "Y (sharded vs one device)")
    # backward: each shard's dZ part, their sum, then each shard's rows and dQ part
    wsb = [fl.alloc_workspace(fl.FLARE_OP_BWD, B, H, Nr, M, D, dtype, DEV) for _ in range(G)]
    dZ = sum(fl.flare_bwd_shard_dz(Q, Ks[r], Vs[r], dYs[r], Z, lse, s, workspace=wsb[r])
             for r in range(G))
    dQ = torch.zeros(Q.shape, dtype=torch.float32, device=DEV)
    dKs, dVs = [], []
    for r in range(G):
        dq, dk, dv = fl.flare_bwd_shard_finish(Q, Ks[r], Vs[r], dYs[r], Z, lse, dZ, s,
                                               workspace=wsb[r])
        dQ += dq
        dKs.append(dk)
        dVs.append(dv)
    for w in wss + wsb:
        assert fl.device_status(w) == 0
    dK, dV = torch.cat(dKs, dim=2), torch.cat(dVs, dim=2)
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    assert_close(dV, dVo, dtype, "dV (sharded)", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dK, dKo, dtype, "dK (sharded)", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dQ, dQo, dtype, "dQ (sharded)", rel_f32=TOL_F32_GRAD_REL)


def test_parallel_module_with_one_rank():
    # the collective module itself, on a one-rank NCCL group: equals the
    # single-device calls
    B, H, N, M, D = 2, 2, 1000, 128, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=107, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29533")
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        Y, Z, lse = fl.parallel.cp_flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
        dQ, dK, dV = fl.parallel.cp_flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    Y1, Z1, l1 = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    r1 = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z1, l1, s)
    assert torch.equal(Y, Y1) and torch.equal(Z, Z1)
    assert torch.equal(dK, r1[1]) and torch.equal(dV, r1[2])
    assert_close(dQ, r1[0].float(), torch.bfloat16, "dQ")


def _merge(Qx, Ks, Vs, s, wss, dims, dtype, **outs_per_shard):
    """Encode every shard, stack the records, merge them on every shard's
    workspace; outs_per_shard(r) gives the output tensors of shard r."""
    B, H, Nr, M, D = dims
    recs = []
    for r, (K, V) in enumerate(zip(Ks, Vs)):
        fl.flare_encode(Qx, K, V, s, workspace=wss[r])
        recs.append([t.clone() for t in fl.encode_records(wss[r], B, H, Nr, M, D, dtype)])
    gml = torch.stack([a for a, _ in recs])
    gacc = torch.stack([b for _, b in recs])
    for r in range(len(Ks)):
        fl.flare_combine_shards(gml, gacc, B, H, Nr, M, D, dtype, workspace=wss[r],
                                **{k: f(r) for k, f in outs_per_shard.items()})


@pytest.mark.parametrize("B,H,N,M,D,dtype,G", [(2, 2, 1536, 128, 32, torch.bfloat16, 2),
                                               (2, 2, 600, 32, 16, torch.float32, 3)],
                         ids=["tc_2", "simt_f32_3"])
def test_sharded_flare_pp(B, H, N, M, D, dtype, G):
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=111 + G, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Q = g["Q"]
    Ks, Vs, dYs = _shards(g["K"], G), _shards(g["V"], G), _shards(g["dY"], G)
    Nr = N // G
    dims = (B, H, Nr, M, D)
    new = lambda *shape, dt=torch.float32: torch.empty(shape, dtype=dt, device=DEV)
    wss = [fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, Nr, M, D, dtype, DEV) for _ in range(G)]
    # first encode: Q_dyn = Q + Z1 (and Z1, lse1 for the backward)
    Qds = [new(B, H, M, D, dt=dtype) for _ in range(G)]
    Z1s = [new(B, H, M, D) for _ in range(G)]
    l1s = [new(B, H, M) for _ in range(G)]
    _merge(Q, Ks, Vs, s, wss, dims, dtype, Q_learned=lambda r: Q, Q_dyn_out=lambda r: Qds[r],
           Z_save=lambda r: Z1s[r], lse_save=lambda r: l1s[r])
    for r in range(1, G):
        assert torch.equal(Qds[r], Qds[0])
    Qd, Z1, lse1 = Qds[0], Z1s[0], l1s[0]
    # second encode with Q_dyn, then each shard's decode
    Zs = [new(B, H, M, D) for _ in range(G)]
    ls = [new(B, H, M) for _ in range(G)]
    _merge(Qd, Ks, Vs, s, wss, dims, dtype, Z_save=lambda r: Zs[r], lse_save=lambda r: ls[r])
    Z, lse = Zs[0], ls[0]
    Y = torch.cat([fl.flare_decode(Qd, Ks[r], s, workspace=wss[r]) for r in range(G)], dim=2)
    Y1, Qd1, Zo1, _ = fl.flare_pp_fwd(Q, g["K"], g["V"], s, save=True)
    Yo, Qdo, _, _ = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Qd, Qdo, dtype, "Q_dyn (sharded)")
    assert_close(Y, Yo, dtype, "Y (sharded)")
    # backward: FLARE's with Q_dyn, then the first encode's, shard by shard
    wsb = [fl.alloc_workspace(fl.FLARE_OP_PP_BWD, B, H, Nr, M, D, dtype, DEV) for _ in range(G)]
    dZ = sum(fl.flare_bwd_shard_dz(Qd, Ks[r], Vs[r], dYs[r], Z, lse, s, workspace=wsb[r])
             for r in range(G))
    parts = [fl.flare_bwd_shard_finish(Qd, Ks[r], Vs[r], dYs[r], Z, lse, dZ, s, workspace=wsb[r])
             for r in range(G)]
    dQd = sum(p[0] for p in parts)
    dQ = sum(fl.flare_pp_bwd_shard_tail(Q, Ks[r], Vs[r], Z1, lse1, dQd.to(dtype), parts[r][1],
                                        parts[r][2], s, workspace=wsb[r], add_dq_dyn=(r == 0))
             for r in range(G))
    for w in wss + wsb:
        assert fl.device_status(w) == 0
    dK = torch.cat([p[1] for p in parts], dim=2)
    dV = torch.cat([p[2] for p in parts], dim=2)
    dQo, dKo, dVo = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    assert_close(dV, dVo, dtype, "dV (sharded)", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dK, dKo, dtype, "dK (sharded)", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dQ, dQo, dtype, "dQ (sharded)", rel_f32=TOL_F32_GRAD_REL)
