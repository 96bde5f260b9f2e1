"""GPU parity of FLARE++ forward and of the FLARE backward against the oracle."""
import math

import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import TOL_F32_GRAD_REL, assert_close, assert_close_scaled

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("B,H,N,M,D", [(2, 2, 1000, 256, 32), (1, 3, 129, 128, 16),
                                       (2, 1, 500, 32, 16), (1, 1, 1, 16, 32)])
def test_pp_fwd_matches_oracle(B, H, N, M, D, dtype):
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=31 + N)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    torch.cuda.synchronize()
    Yo, Qdo, Zo, lo = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Qd, Qdo, dtype, "Q_dyn")
    assert_close(Z, Zo, dtype, "Z")
    assert_close(Y, Yo, dtype, "Y")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("per_batch_q", [False, True], ids=["sharedQ", "batchQ"])
@pytest.mark.parametrize("B,H,N,M,D", [(2, 2, 600, 128, 32), (1, 2, 257, 256, 16),
                                       (3, 1, 64, 32, 16)])
def test_bwd_matches_oracle(B, H, N, M, D, dtype, per_batch_q):
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=41 + N, per_batch_q=per_batch_q,
                    with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    torch.cuda.synchronize()
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    assert_close(dV, dVo, dtype, "dV", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dK, dKo, dtype, "dK", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dQ, dQo, dtype, "dQ", rel_f32=TOL_F32_GRAD_REL)


def test_bwd_is_bitwise_deterministic():
    B, H, N, M, D = 2, 2, 3000, 128, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=3, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    a = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    b = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_bwd_single_token_closed_form(dtype):
    # With one token every latent encodes Z[m] = V[0] and the decode returns
    # Y[0] = V[0] whatever K and Q are: dQ = 0, dK = 0 and dV = dY exactly.
    B, H, N, M, D = 2, 2, 1, 32, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=4, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    torch.cuda.synchronize()
    assert torch.equal(Y, g["V"]) or float((Y.float() - g["V"].float()).abs().max()) <= 1e-6 * 4
    tol = 1e-5 if dtype == torch.float32 else 3e-2
    assert float(dQ.float().abs().max()) <= tol
    assert float(dK.float().abs().max()) <= tol
    assert float((dV.float() - g["dY"].float()).abs().max()) <= tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("B,H,N,M,D", [(2, 2, 600, 128, 32), (1, 2, 257, 256, 16),
                                       (2, 1, 300, 32, 16), (2, 2, 1000, 128, 16)])
def test_pp_bwd_matches_oracle(B, H, N, M, D, dtype):
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=51 + N, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    ws = fl.alloc_workspace(fl.FLARE_OP_PP_BWD, B, H, N, M, D, dtype, DEV)
    ws.fill_(0xFF)   # NaN in every float the kernels might read unwritten
    dQ, dK, dV = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s, workspace=ws)
    assert fl.device_status(ws) == 0
    dQo, dKo, dVo = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    assert_close(dV, dVo, dtype, "dV", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dK, dKo, dtype, "dK", rel_f32=TOL_F32_GRAD_REL)
    assert_close(dQ, dQo, dtype, "dQ", rel_f32=TOL_F32_GRAD_REL)


def test_pp_bwd_is_bitwise_deterministic():
    B, H, N, M, D = 2, 2, 2000, 128, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=52, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    a = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s)
    b = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_pp_bwd_single_token_closed_form(dtype):
    # One token: both encodes return V[0] for every latent and the decode
    # returns Y = V[0] whatever Q and K are, so dQ = dK = 0 and dV = dY.
    B, H, N, M, D = 1, 3, 1, 16, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=53, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    dQ, dK, dV = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s)
    torch.cuda.synchronize()
    tol = 1e-5 if dtype == torch.float32 else 3e-2
    assert float(dQ.float().abs().max()) <= tol
    assert float(dK.float().abs().max()) <= tol
    assert float((dV.float() - g["dY"].float()).abs().max()) <= tol


# The tensor-core form (bf16, M = 128, D in {16, 32}): FLARE's backward with
# Q_dyn and the first encode's gradient both run on tcgen05 kernels.
@pytest.mark.parametrize("B,H,N,D", [(2, 2, 127, 32), (1, 2, 129, 16), (2, 1, 383, 32),
                                     (1, 2, 40000, 32)])
def test_pp_bwd_tensor_core_sizes(B, H, N, D):
    M, dtype = 128, torch.bfloat16
    assert fl.bwd_path(B, H, N, M, D, dtype) == 1
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=61 + N, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    ws = fl.alloc_workspace(fl.FLARE_OP_PP_BWD, B, H, N, M, D, dtype, DEV)
    ws.fill_(0xFF)
    dQ, dK, dV = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s, workspace=ws)
    assert fl.device_status(ws) == 0
    dQo, dKo, dVo = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    assert_close(dV, dVo, dtype, "dV")
    assert_close(dK, dKo, dtype, "dK")
    assert_close(dQ, dQo, dtype, "dQ")


@pytest.mark.parametrize("D", [16, 32])
def test_pp_bwd_tensor_core_single_token(D):
    B, H, N, M = 2, 2, 1, 128
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=62, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    dQ, dK, dV = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s)
    torch.cuda.synchronize()
    assert float(dQ.float().abs().max()) <= 3e-2
    assert float(dK.float().abs().max()) <= 3e-2
    assert float((dV.float() - g["dY"].float()).abs().max()) <= 3e-2


def test_pp_bwd_tensor_core_mixed_heads_fast_and_exact():
    # Head 1's latent queries are scaled up so that the first encode's lse
    # spreads far beyond 64 (log2 units): its gradient takes the exact form
    # while head 0 takes the one-exponential form, in the same launches.
    # Head 1's gradient is so sensitive to Q_dyn that rounding Q_dyn to bf16
    # alone moves it by about 2% (relative Frobenius), so the expected values
    # are the gradient at the bf16 Q_dyn the forward stores (reading C15):
    # the oracle's own Q_dyn, rounded to bf16 (round to nearest even) on the
    # host; FLARE's gradient at that Q_dyn plus the first encode's gradient
    # with upstream dQ_dyn.  No value computed on the GPU enters them.
    B, H, N, M, D = 2, 2, 1500, 128, 32
    dtype = torch.bfloat16
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=63, with_dy=True)
    x["Q"][1] = (x["Q"][1].float() * 40.0).to(dtype)
    # the premise: the first encode's lse spread (log2 units) per head
    lg = s * torch.einsum("hmd,bhnd->bhmn", x["Q"].double(), x["K"].double())
    spread = lg.logsumexp(-1).amax(-1) - lg.logsumexp(-1).amin(-1)
    spread = spread * math.log2(math.e)
    assert float(spread[:, 1].min()) > 64.0 and float(spread[:, 0].max()) < 64.0
    _, Qd_o, _, _ = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s)
    Qd_b = torch.from_numpy(Qd_o).to(dtype)          # RNE rounding on the host
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd, Z, lse = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s, save=True)
    ws = fl.alloc_workspace(fl.FLARE_OP_PP_BWD, B, H, N, M, D, dtype, DEV)
    ws.fill_(0xFF)
    dQ, dK, dV = fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, s, workspace=ws)
    assert fl.device_status(ws) == 0
    dQd, dKa, dVa = oracle.flare_bwd(Qd_b, x["K"], x["V"], x["dY"], s)
    dQe, dKe, dVe = oracle.encode_bwd(x["Q"], x["K"], x["V"], dQd, s)
    dKo, dVo, dQo = dKa + dKe, dVa + dVe, dQd.sum(0) + dQe
    for hh in (0, 1):
        chk = assert_close if hh == 0 else (lambda a, b, dt, w: assert_close_scaled(a, b, w))
        chk(dV[:, hh], dVo[:, hh], dtype, f"dV head {hh}")
        chk(dK[:, hh], dKo[:, hh], dtype, f"dK head {hh}")
        chk(dQ[hh], dQo[hh], dtype, f"dQ head {hh}")
