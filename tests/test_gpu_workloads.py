"""Parity on the five benchmark workloads at their full sizes.

Each runs the library exactly as bench.py does.  Where the oracle cannot
finish the whole workload in seconds it checks complete (b, h) heads: Z and
lse over all N tokens, and Y at sampled tokens (first, last and random).
"""
import numpy as np
import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import WORKLOADS, make_workload_inputs
from gpu_util import TOL_F32_GRAD_REL, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _stage_fwd(g, w, ws, Z, lse):
    """The forward as bench.py launches it: encode, combine, decode."""
    fl.flare_encode(g["Q"], g["K"], g["V"], w.scale, workspace=ws)
    fl.flare_combine(w.B, w.H, w.N, w.M, w.D, w.torch_dtype, workspace=ws, Z_save=Z, lse_save=lse)
    return fl.flare_decode(g["Q"], g["K"], w.scale, workspace=ws)


def _sample_rows(N, k, seed):
    rng = np.random.default_rng(seed)
    r = np.concatenate([np.arange(min(64, N)), np.arange(max(0, N - 64), N),
                        rng.integers(0, N, size=k)])
    return np.unique(r)


def test_c1_fp32_tiny_full():
    w = WORKLOADS["c1_fwd_f32_tiny"]
    x = make_workload_inputs(w)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, DEV)
    Z = torch.empty((w.B, w.H, w.M, w.D), device=DEV)
    lse = torch.empty((w.B, w.H, w.M), device=DEV)
    Y = _stage_fwd(g, w, ws, Z, lse)
    torch.cuda.synchronize()
    Yo, Zo, lo = oracle.flare_fwd(x["Q"], x["K"], x["V"], w.scale)
    assert_close(Z, Zo, torch.float32, "Z")
    assert_close(lse, lo, torch.float32, "lse")
    assert_close(Y, Yo, torch.float32, "Y")


def test_c2_bf16_mesh256_full():
    w = WORKLOADS["c2_fwd_bf16_mesh256"]
    x = make_workload_inputs(w)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, DEV)
    Z = torch.empty((w.B, w.H, w.M, w.D), device=DEV)
    lse = torch.empty((w.B, w.H, w.M), device=DEV)
    Y = _stage_fwd(g, w, ws, Z, lse)
    assert fl.device_status(ws) == 0
    Yo, Zo, lo = oracle.flare_fwd(x["Q"], x["K"], x["V"], w.scale)
    assert_close(Z, Zo, w.torch_dtype, "Z")
    assert_close(Y, Yo, w.torch_dtype, "Y")


def test_c3_bf16_1M_headline_sampled():
    w = WORKLOADS["c3_fwd_bf16_1M"]
    x = make_workload_inputs(w)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, DEV)
    Z = torch.empty((w.B, w.H, w.M, w.D), device=DEV)
    lse = torch.empty((w.B, w.H, w.M), device=DEV)
    Y = _stage_fwd(g, w, ws, Z, lse)
    assert fl.device_status(ws) == 0
    Yc, Zc, lc = Y.cpu(), Z.cpu(), lse.cpu()
    del g, Y
    for h in (0, 11):
        Qh = x["Q"][h:h + 1]
        Kh = x["K"][0:1, h:h + 1]
        Vh = x["V"][0:1, h:h + 1]
        Zo, lo = oracle.encode(Qh, Kh, Vh, w.scale)
        assert_close(Zc[0, h], Zo[0, 0], w.torch_dtype, f"Z head {h}")
        assert_close(lc[0, h], lo[0, 0], w.torch_dtype, f"lse head {h}")
        rows = _sample_rows(w.N, 4096, seed=h)
        Yo = oracle.decode_rows(Qh, Kh, Zo, w.scale, rows)
        assert_close(Yc[0, h][rows], Yo, w.torch_dtype, f"Y head {h}")


def test_c4_flare_pp_sampled_heads():
    w = WORKLOADS["c4_ppfwd_bf16_256k"]
    x = make_workload_inputs(w)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], w.scale, save=True)
    torch.cuda.synchronize()
    Yc, Qdc, Zc = Y.cpu(), Qd.cpu(), Z.cpu()
    del g, Y
    for b, h in ((0, 0), (1, 7)):
        Yo, Qdo, Zo, _ = oracle.flare_pp_fwd(x["Q"][h:h + 1], x["K"][b:b + 1, h:h + 1],
                                             x["V"][b:b + 1, h:h + 1], w.scale)
        assert_close(Qdc[b, h], Qdo[0, 0], w.torch_dtype, f"Q_dyn {b},{h}")
        assert_close(Zc[b, h], Zo[0, 0], w.torch_dtype, f"Z {b},{h}")
        assert_close(Yc[b, h], Yo[0, 0], w.torch_dtype, f"Y {b},{h}")


def test_c5_fwd_bwd_full_fwd_sampled_bwd():
    w = WORKLOADS["c5_fwdbwd_bf16_16k"]
    x = make_workload_inputs(w)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], w.scale, save=True)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, w.scale)
    torch.cuda.synchronize()
    Yo, _, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], w.scale)
    assert_close(Y, Yo, w.torch_dtype, "Y")
    dQc, dKc, dVc = dQ.cpu(), dK.cpu(), dV.cpu()
    for h in (0, 5):
        # dQ[h] sums over the whole batch (shared latents): take every b of head h
        dQo, dKo, dVo = oracle.flare_bwd(x["Q"][h:h + 1], x["K"][:, h:h + 1],
                                         x["V"][:, h:h + 1], x["dY"][:, h:h + 1], w.scale)
        assert_close(dVc[:, h:h + 1], dVo, w.torch_dtype, f"dV head {h}")
        assert_close(dKc[:, h:h + 1], dKo, w.torch_dtype, f"dK head {h}")
        assert_close(dQc[h:h + 1], dQo, w.torch_dtype, f"dQ head {h}")
