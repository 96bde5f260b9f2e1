"""Variable sequence lengths (key-padding mask) on the GPU against the oracle.

Batch element b has seq_lens[b] valid tokens; the rest is padding, filled
here with NaN in K, V and dY so that any read of it would show.  Lengths
cover the empty sequence, one token, and both sides of the tensor-core
encode (48-token) and decode / backward (128-token) tile boundaries.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import TOL_F32_GRAD_REL, assert_close, max_abs, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (B, H, N, M, D, dtype, lens)
CASES = [
    (6, 2, 400, 128, 32, torch.bfloat16, [400, 0, 1, 47, 129, 256]),   # tensor-core fwd + bwd
    (4, 2, 300, 128, 16, torch.bfloat16, [49, 128, 127, 300]),         # tensor-core, D = 16
    (3, 2, 500, 256, 32, torch.bfloat16, [96, 500, 5]),                # tensor cores, M = 256
    (3, 2, 200, 64, 16, torch.bfloat16, [0, 65, 200]),                 # CUDA-core bf16
    (3, 2, 150, 32, 16, torch.float32, [1, 150, 64]),                  # CUDA-core fp32
]
IDS = ["tc_D32", "tc_D16", "tc_M256", "simt_bf16", "simt_f32"]


def _inputs(B, H, N, M, D, dtype, lens, seed, with_dy=True):
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=seed, with_dy=with_dy)
    for b, L in enumerate(lens):   # padding: never read
        for k in ("K", "V", "dY"):
            if k in x:
                x[k][b, :, L:] = float("nan")
    g = {k: v.to(DEV) for k, v in x.items()}
    g["lens"] = torch.tensor(lens, dtype=torch.int32, device=DEV)
    return x, g


def _check_padding_zero(t, lens, what):
    for b, L in enumerate(lens):
        assert not torch.any(t[b, :, L:] != 0), f"{what}: padding of batch {b} not zero"


def _close_valid(got, ref, lens, dtype, what, **kw):
    # compare only the valid rows (the padding is checked to be exactly 0).  A
    # one-token sequence has dK = 0 exactly (its encode and decode weights are
    # constant 1), so a relative error there is meaningless: absolute bound.
    for b, L in enumerate(lens):
        if L == 1:
            tol = 1e-5 if dtype == torch.float32 else 3e-2
            assert max_abs(got[b, :, :1], ref[b, :, :1]) <= tol, f"{what} batch {b} (one token)"
        elif L > 1:
            assert_close(got[b, :, :L], ref[b, :, :L], dtype, f"{what} batch {b}", **kw)


@pytest.mark.parametrize("B,H,N,M,D,dtype,lens", CASES, ids=IDS)
def test_varlen_fwd_matches_oracle(B, H, N, M, D, dtype, lens):
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, dtype, lens, seed=81 + N, with_dy=False)
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, dtype, DEV)
    ws.fill_(0xFF)
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, seq_lens=g["lens"],
                             workspace=ws)
    assert fl.device_status(ws) == 0
    Yo, Zo, lo = oracle.flare_fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)
    assert torch.isfinite(Y).all()
    _check_padding_zero(Y, lens, "Y")
    _close_valid(Y, Yo, lens, dtype, "Y")
    assert_close(Z, Zo, dtype, "Z")
    lse_c = lse.cpu().numpy()
    empty = np.array(lens) == 0
    assert np.all(lse_c[empty] == -np.inf)
    np.testing.assert_allclose(lse_c[~empty], lo[~empty], rtol=0,
                               atol=1e-5 if dtype == torch.float32 else 2e-2)


@pytest.mark.parametrize("B,H,N,M,D,dtype,lens", CASES, ids=IDS)
def test_varlen_bwd_matches_oracle(B, H, N, M, D, dtype, lens):
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, dtype, lens, seed=82 + N)
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, seq_lens=g["lens"])
    ws = fl.alloc_workspace(fl.FLARE_OP_BWD, B, H, N, M, D, dtype, DEV)
    ws.fill_(0xFF)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s, seq_lens=g["lens"],
                              workspace=ws)
    assert fl.device_status(ws) == 0
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens)
    for t in (dQ, dK, dV):
        assert torch.isfinite(t).all()
    _check_padding_zero(dK, lens, "dK")
    _check_padding_zero(dV, lens, "dV")
    _close_valid(dV, dVo, lens, dtype, "dV", rel_f32=TOL_F32_GRAD_REL)
    _close_valid(dK, dKo, lens, dtype, "dK", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dQ, dQo, dtype, "dQ", rel_f32=TOL_F32_GRAD_REL)


@pytest.mark.parametrize("B,H,N,M,D,dtype,lens", [CASES[0], CASES[3]], ids=["tc", "simt_bf16"])
def test_varlen_pp_fwd_bwd_matches_oracle(B, H, N, M, D, dtype, lens):
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, dtype, lens, seed=83 + N)
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True, seq_lens=g["lens"])
    dQ, dK, dV = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s,
                                 seq_lens=g["lens"])
    torch.cuda.synchronize()
    Yo, Qdo, _, _ = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)
    dQo, dKo, dVo = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens)
    _check_padding_zero(Y, lens, "Y")
    _close_valid(Y, Yo, lens, dtype, "Y")
    assert_close(Qd, Qdo, dtype, "Q_dyn")
    _check_padding_zero(dK, lens, "dK")
    _check_padding_zero(dV, lens, "dV")
    _close_valid(dV, dVo, lens, dtype, "dV")
    _close_valid(dK, dKo, lens, dtype, "dK")
    assert_close(dQ, dQo, dtype, "dQ")


@pytest.mark.parametrize("N", [1152, 1000])
def test_full_lengths_equal_the_unmasked_call(N):
    # seq_lens = N for every batch element computes the plain call: bit for
    # bit when N is a multiple of every tile (48, 128 and 256 tokens); with a
    # partial last tile the two place it differently (the plain call reads
    # rows past N as zeros, the length-aware one right-aligns the tile), so
    # they agree to rounding.
    B, H, M, D = 2, 2, 128, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=84, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    lens = torch.full((B,), N, dtype=torch.int32, device=DEV)
    a = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    b = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, seq_lens=lens)
    ra = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], a[1], a[2], s)
    rb = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], a[1], a[2], s, seq_lens=lens)
    torch.cuda.synchronize()
    for u, v, what in zip(a + ra, b + rb, ("Y", "Z", "lse", "dQ", "dK", "dV")):
        if N % 384 == 0:
            assert torch.equal(u, v), what
        else:
            assert_close(v, u, torch.bfloat16, what)


def test_varlen_with_strided_layout():
    # lengths and a [B,N,H,D] layout together
    B, H, N, M, D = 3, 2, 333, 128, 32
    lens = [333, 100, 0]
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, torch.bfloat16, lens, seed=85)
    t = {k: g[k].transpose(1, 2).contiguous().transpose(1, 2) for k in ("K", "V", "dY")}
    Y, Z, lse = fl.flare_fwd(g["Q"], t["K"], t["V"], s, save=True, seq_lens=g["lens"])
    dQ, dK, dV = fl.flare_bwd(g["Q"], t["K"], t["V"], t["dY"], Z, lse, s, seq_lens=g["lens"])
    torch.cuda.synchronize()
    Yo, _, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens)
    _check_padding_zero(Y, lens, "Y")
    _close_valid(Y, Yo, lens, torch.bfloat16, "Y")
    _check_padding_zero(dK, lens, "dK")
    _close_valid(dK, dKo, lens, torch.bfloat16, "dK")
    _close_valid(dV, dVo, lens, torch.bfloat16, "dV")
    assert_close(dQ, dQo, torch.bfloat16, "dQ")


def test_out_of_range_lengths_are_clamped_and_reported():
    B, H, N, M, D = 2, 2, 100, 128, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=86)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, torch.bfloat16, DEV)
    bad = torch.tensor([N + 5, -3], dtype=torch.int32, device=DEV)
    Y = fl.flare_fwd(g["Q"], g["K"], g["V"], s, seq_lens=bad, workspace=ws)
    with pytest.raises(fl.FlareError):
        fl.device_status(ws)
    # clamped to [N, 0]
    Yc = fl.flare_fwd(g["Q"], g["K"], g["V"], s,
                      seq_lens=torch.tensor([N, 0], dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert torch.equal(Y, Yc)


def _plan_lens(B, N, seed):
    r = np.random.default_rng(seed)
    lens = r.integers(0, N + 1, size=B)
    lens[0], lens[-1] = N, 0
    return [int(v) for v in lens]


# Length-proportional work plans: one long sequence among short ones (its
# tiles split into many units, the short heads into one each), and a batch
# larger than the plan kernel's thread count (its scan over the batch takes
# several elements per thread).
PLAN_CASES = [
    (4, 8, 20000, 128, 32, [20000, 3000, 0, 17]),
    (2, 4, 9000, 256, 32, [9000, 1]),
    (1100, 1, 64, 128, 16, _plan_lens(1100, 64, 87)),
]
PLAN_IDS = ["skewed_M128", "skewed_M256", "batch1100"]


@pytest.mark.parametrize("B,H,N,M,D,lens", PLAN_CASES, ids=PLAN_IDS)
def test_varlen_work_plan_matches_oracle(B, H, N, M, D, lens):
    dtype = torch.bfloat16
    s = 1.0 / math.sqrt(D)
    x, g = _inputs(B, H, N, M, D, dtype, lens, seed=88 + B)
    wsf = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, dtype, DEV)
    wsb = fl.alloc_workspace(fl.FLARE_OP_BWD, B, H, N, M, D, dtype, DEV)
    wsf.fill_(0xFF)
    wsb.fill_(0xFF)
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, seq_lens=g["lens"],
                             workspace=wsf)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s, seq_lens=g["lens"],
                              workspace=wsb)
    assert fl.device_status(wsf) == 0 and fl.device_status(wsb) == 0
    Yo, Zo, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens)
    for t in (Y, Z, dQ, dK, dV):
        assert torch.isfinite(t).all()
    _check_padding_zero(Y, lens, "Y")
    _check_padding_zero(dK, lens, "dK")
    _check_padding_zero(dV, lens, "dV")
    if B > 64:   # many short heads: compare all valid rows at once
        mask = np.zeros(tuple(Y.shape), dtype=bool)
        for b, L in enumerate(lens):
            mask[b, :, :L] = True
        for got, ref, what in ((Y, Yo, "Y"), (dK, dKo, "dK"), (dV, dVo, "dV")):
            assert_close(to64(got)[mask], np.asarray(ref)[mask], dtype, what)
    else:
        _close_valid(Y, Yo, lens, dtype, "Y")
        _close_valid(dK, dKo, lens, dtype, "dK")
        _close_valid(dV, dVo, lens, dtype, "dV")
    assert_close(Z, Zo, dtype, "Z")
    assert_close(dQ, dQo, dtype, "dQ")
