"""Context parallelism's host logic on CPU (gloo, world size 2 and 3), for
FLARE and FLARE++.

rank_latent_attention_flare_b200.parallel runs the collectives: the
all-gather of the encode records and the all-reduces of dZ and dQ.  Here its
stage calls are replaced by float64 torch stand-ins written from the shard
math below (the CUDA library is not available on CPU), so the test checks
the exchanges -- which rank's data lands where, what is summed -- against
the oracle on the whole sequence.

Shard math per (b, h), tokens n in this rank's shard, logits in log2 units
x = s log2(e) q.k: a record is (m, l, acc) = (max x, sum 2^(x-m),
sum 2^(x-m) v); records merge by the log-sum-exp rule; the decode is per
token; dZ = sum over tokens of P_d^T dY is summed over the shards, and so
is dQ.
"""
import math
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LOG2E = 1.0 / math.log(2.0)


class _Stand:
    """Stage calls with the library's signatures, in float64 torch."""

    class _WS(dict):
        pass

    @staticmethod
    def alloc_workspace(op, B, H, N, M, D, dtype, device):
        return _Stand._WS()

    @staticmethod
    def _q(Q, B):
        return Q.double() if Q.dim() == 4 else Q.double().unsqueeze(0).expand(B, -1, -1, -1)

    @staticmethod
    def flare_encode(Q, K, V, s, *, workspace):
        B = K.shape[0]
        x = torch.einsum("bhmd,bhnd->bhmn", _Stand._q(Q, B), K.double()) * s * LOG2E
        m = x.amax(-1)
        w = torch.exp2(x - m[..., None])
        workspace["rec"] = (m, w.sum(-1), torch.einsum("bhmn,bhnd->bhmd", w, V.double()))

    @staticmethod
    def encode_records(ws, B, H, N, M, D, dtype):
        m, l, acc = ws["rec"]
        ml = torch.stack([m, l], -1).reshape(B * H, 1, M, 2)
        return ml, acc.reshape(B * H, 1, M, D)

    @staticmethod
    def flare_combine_shards(gml, gacc, B, H, N, M, D, dtype, *, workspace, Z_save=None,
                             lse_save=None, Q_learned=None, Q_dyn_out=None):
        m, l = gml[..., 0], gml[..., 1]                        # [G, BH, R, M]
        mstar = m.amax(dim=(0, 2))                             # [BH, M]
        f = torch.exp2(m - mstar[None, :, None, :])
        L = (f * l).sum(dim=(0, 2))
        Z = (f[..., None] * gacc).sum(dim=(0, 2)) / L[..., None]
        workspace["Z"] = Z.reshape(B, H, M, D)
        if Z_save is not None:
            Z_save.copy_(workspace["Z"])
            lse_save.copy_(((mstar + torch.log2(L)) / LOG2E).reshape(B, H, M))
        if Q_dyn_out is not None:   # FLARE++: Q_dyn = Q + Z1
            Q_dyn_out.copy_(Q_learned.double().unsqueeze(0) + workspace["Z"])

    @staticmethod
    def _pd(Q, K, s):
        return torch.softmax(s * torch.einsum("bhnd,bhmd->bhnm", K.double(),
                                              _Stand._q(Q, K.shape[0])), -1)

    @staticmethod
    def flare_decode(Q, K, s, *, workspace):
        return torch.einsum("bhnm,bhmd->bhnd", _Stand._pd(Q, K, s), workspace["Z"])

    @staticmethod
    def flare_bwd_shard_dz(Q, K, V, dY, Z, lse, s, *, workspace):
        Pd = _Stand._pd(Q, K, s)
        dPd = torch.einsum("bhnd,bhmd->bhnm", dY.double(), Z.double())
        dAd = Pd * (dPd - (Pd * dPd).sum(-1, keepdim=True))
        workspace["dk"] = s * torch.einsum("bhnm,bhmd->bhnd", dAd, _Stand._q(Q, K.shape[0]))
        workspace["dq"] = s * torch.einsum("bhnm,bhnd->bhmd", dAd, K.double())
        return torch.einsum("bhnm,bhnd->bhmd", Pd, dY.double())

    @staticmethod
    def flare_bwd_shard_finish(Q, K, V, dY, Z, lse, dZ, s, *, workspace):
        Qb = _Stand._q(Q, K.shape[0])
        Pe = torch.exp(s * torch.einsum("bhmd,bhnd->bhmn", Qb, K.double()) - lse.double()[..., None])
        dPe = torch.einsum("bhmd,bhnd->bhmn", dZ, V.double())
        dAe = Pe * (dPe - (dZ * Z.double()).sum(-1)[..., None])
        dK = workspace["dk"] + s * torch.einsum("bhmn,bhmd->bhnd", dAe, Qb)
        dV = torch.einsum("bhmn,bhmd->bhnd", Pe, dZ)
        dq = workspace["dq"] + s * torch.einsum("bhmn,bhnd->bhmd", dAe, K.double())
        return (dq.sum(0) if Q.dim() == 3 else dq), dK, dV

    @staticmethod
    def flare_pp_bwd_shard_tail(Q, K, V, Z1, lse1, dQd, dK, dV, s, *, workspace, add_dq_dyn=False):
        # the first encode's gradient with upstream dZ1 = dQ_dyn, over the shard
        Qb = _Stand._q(Q, K.shape[0])
        P = torch.exp(s * torch.einsum("bhmd,bhnd->bhmn", Qb, K.double()) - lse1.double()[..., None])
        dP = torch.einsum("bhmd,bhnd->bhmn", dQd.double(), V.double())
        dA = P * (dP - (dQd.double() * Z1.double()).sum(-1)[..., None])
        dV += torch.einsum("bhmn,bhmd->bhnd", P, dQd.double())
        dK += s * torch.einsum("bhmn,bhmd->bhnd", dA, Qb)
        part = (s * torch.einsum("bhmn,bhnd->bhmd", dA, K.double())).sum(0)
        return part + dQd.double().sum(0) if add_dq_dyn else part


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, batch_q, pp, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist

    from flare_inputs import make_inputs
    from rank_latent_attention_flare_b200 import parallel
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, M, D = 2, 2, 24 * world, 5, 4
        s = 0.5
        x = make_inputs(B, H, N, M, D, dtype=torch.float64, seed=7, per_batch_q=batch_q,
                        with_dy=True)
        sh = {k: x[k].chunk(world, dim=2)[rank].contiguous() for k in ("K", "V", "dY")}
        if pp:
            Y, Qd, Z, lse = parallel.cp_flare_pp_fwd(x["Q"], sh["K"], sh["V"], s, save=True,
                                                     ops=_Stand)
            dQ, dK, dV = parallel.cp_flare_pp_bwd(x["Q"], sh["K"], sh["V"], sh["dY"], Qd, Z, lse,
                                                  s, ops=_Stand)
        else:
            Y, Z, lse = parallel.cp_flare_fwd(x["Q"], sh["K"], sh["V"], s, save=True, ops=_Stand)
            dQ, dK, dV = parallel.cp_flare_bwd(x["Q"], sh["K"], sh["V"], sh["dY"], Z, lse, s,
                                               ops=_Stand)
        out[rank] = (Y.numpy(), Z.numpy(), dQ.numpy(), dK.numpy(), dV.numpy())
    finally:
        dist.destroy_process_group()


def _run(world, batch_q, pp=False):
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from flare_inputs import make_inputs
    out = mp.Manager().dict()
    mp.start_processes(_worker, args=(world, _free_port(), batch_q, pp, out), nprocs=world,
                       join=True, start_method="spawn")
    B, H, N, M, D = 2, 2, 24 * world, 5, 4
    x = make_inputs(B, H, N, M, D, dtype=torch.float64, seed=7, per_batch_q=batch_q, with_dy=True)
    if pp:
        Yo, _, Zo, _ = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], 0.5)
        dQo, dKo, dVo = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], 0.5)
    else:
        Yo, Zo, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], 0.5)
        dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], 0.5)
    n = N // world
    for r in range(world):
        Y, Z, dQ, dK, dV = out[r]
        rows = slice(r * n, (r + 1) * n)
        np.testing.assert_allclose(Y, Yo[:, :, rows], rtol=1e-10, atol=1e-12)
        # Z and lse are kept in float32 (as the library keeps them), and the
        # backward starts from them
        np.testing.assert_allclose(Z, Zo, rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(dK, dKo[:, :, rows], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(dV, dVo[:, :, rows], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(dQ, dQo, rtol=1e-5, atol=1e-6)


def test_two_ranks_shared_latents():
    _run(2, False)


def test_three_ranks_per_batch_latents():
    _run(3, True)


def test_flare_pp_two_ranks():
    _run(2, False, pp=True)
