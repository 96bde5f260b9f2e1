"""Token tensors in other layouts than contiguous [B,H,N,D].

A fused projection produces K and V as [B,N,H,D] (or interleaved
[B,N,3,H,D]); the *_ex entry points read and write such layouts in
place.  The arithmetic is the same as for contiguous tensors, so the results
must equal the contiguous call's bit for bit, and the contiguous call is
compared with the oracle elsewhere; one case per op is also compared with the
oracle here.
"""
import math

import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import TOL_F32_GRAD_REL, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (B, H, N, M, D, dtype): tensor-core and CUDA-core forward / backward shapes
CASES = [
    (2, 3, 1000, 128, 32, torch.bfloat16),    # tensor-core fwd and bwd
    (1, 2, 777, 256, 16, torch.bfloat16),     # tensor cores, M = 256 (B = 1: 3-D maps)
    (2, 2, 1000, 256, 32, torch.bfloat16),    # tensor cores, M = 256, 4-D maps
    (2, 2, 300, 64, 32, torch.bfloat16),      # CUDA-core fwd and bwd
    (2, 2, 257, 32, 16, torch.float32),       # CUDA-core, fp32
]
IDS = ["tc", "tc_M256", "tc_M256_4d", "simt_bf16", "simt_f32"]


def _bnhd(x: torch.Tensor) -> torch.Tensor:
    """The same values as x [B,H,N,D], stored as [B,N,H,D]; returns the
    [B,H,N,D] view."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


def _fused(*xs: torch.Tensor):
    """The tensors xs [B,H,N,D] interleaved in one [B,N,len(xs),H,D] buffer,
    as [B,H,N,D] views (not dense: rows len(xs)*H*D apart); and the buffer."""
    B, H, N, D = xs[0].shape
    buf = torch.empty((B, N, len(xs), H, D), dtype=xs[0].dtype, device=xs[0].device)
    for i, x in enumerate(xs):
        buf[:, :, i] = x.transpose(1, 2)
    return [buf[:, :, i].transpose(1, 2) for i in range(len(xs))], buf


def _inputs(B, H, N, M, D, dtype, seed, **kw):
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=seed, **kw)
    return x, {k: v.to(DEV) for k, v in x.items()}


@pytest.mark.parametrize("B,H,N,M,D,dtype", CASES, ids=IDS)
def test_fwd_strided_equals_contiguous(B, H, N, M, D, dtype):
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, dtype, seed=71 + N)
    Y0, Z0, l0 = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    # [B,N,H,D] K and V; Y comes back in K's layout
    Kt, Vt = _bnhd(g["K"]), _bnhd(g["V"])
    assert not Kt.is_contiguous()
    Y1, Z1, l1 = fl.flare_fwd(g["Q"], Kt, Vt, s, save=True)
    assert Y1.stride() == Kt.stride()
    # interleaved [B,N,3,H,D]: Y written into slot 0 of the same buffer
    (Yf, Kf, Vf), buf = _fused(torch.zeros_like(g["K"]), g["K"], g["V"])
    before = buf[:, :, 1:].clone()
    fl.flare_fwd(g["Q"], Kf, Vf, s, out=Yf)
    torch.cuda.synchronize()
    assert torch.equal(buf[:, :, 1:], before)        # K and V slots untouched
    for Y in (Y1, Yf):
        assert torch.equal(Y, Y0)
    assert torch.equal(Z1, Z0) and torch.equal(l1, l0)
    if N == 1000 or dtype == torch.float32:
        Yo, _, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
        assert_close(Y1, Yo, dtype, "Y (strided)")


@pytest.mark.parametrize("B,H,N,M,D,dtype", CASES, ids=IDS)
def test_bwd_strided_equals_contiguous(B, H, N, M, D, dtype):
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, dtype, seed=72 + N, with_dy=True)
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    r0 = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    Kt, Vt, dYt = _bnhd(g["K"]), _bnhd(g["V"]), _bnhd(g["dY"])
    r1 = fl.flare_bwd(g["Q"], Kt, Vt, dYt, Z, lse, s)
    assert r1[1].stride() == Kt.stride() and r1[2].stride() == Vt.stride()
    (Kf, Vf, dYf), _ = _fused(g["K"], g["V"], g["dY"])
    r2 = fl.flare_bwd(g["Q"], Kf, Vf, dYf, Z, lse, s)
    torch.cuda.synchronize()
    for r in (r1, r2):
        for a, b in zip(r, r0):
            assert torch.equal(a, b)
    if N == 1000 or dtype == torch.float32:
        dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
        assert_close(r1[2], dVo, dtype, "dV", rel_f32=TOL_F32_GRAD_REL)
        assert_close(r1[1], dKo, dtype, "dK", rel_f32=TOL_F32_GRAD_REL)
        assert_close(r1[0], dQo, dtype, "dQ", rel_f32=TOL_F32_GRAD_REL)


@pytest.mark.parametrize("B,H,N,M,D,dtype", [CASES[0], CASES[2], CASES[3]],
                         ids=["tc", "tc_M256_4d", "simt_bf16"])
def test_pp_fwd_bwd_strided_equals_contiguous(B, H, N, M, D, dtype):
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, dtype, seed=73 + N, with_dy=True)
    Y0, Qd0, Z0, l0 = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    r0 = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd0, Z0, l0, s)
    (Kf, Vf, dYf), _ = _fused(g["K"], g["V"], g["dY"])
    Y1, Qd1, Z1, l1 = fl.flare_pp_fwd(g["Q"], Kf, Vf, s, save=True)
    r1 = fl.flare_pp_bwd(g["Q"], Kf, Vf, dYf, Qd1, Z1, l1, s)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y0) and torch.equal(Qd1, Qd0)
    for a, b in zip(r1, r0):
        assert torch.equal(a, b)
    if N == 1000:
        dQo, dKo, dVo = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
        assert_close(r1[2], dVo, dtype, "dV")
        assert_close(r1[1], dKo, dtype, "dK")
        assert_close(r1[0], dQo, dtype, "dQ")


def test_strided_rejects_overlapping_output():
    B, H, N, M, D = 1, 2, 64, 32, 16
    x, g = _inputs(B, H, N, M, D, torch.bfloat16, seed=74)
    Y = torch.empty(B * H * N * D, dtype=torch.bfloat16, device=DEV)
    # every head's rows on top of each other
    Yv = Y.as_strided((B, H, N, D), (H * N * D, 0 + 8, D, 1))
    with pytest.raises(fl.FlareError):
        fl.flare_fwd(g["Q"], g["K"], g["V"], out=Yv)
