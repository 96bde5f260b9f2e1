"""GPU parity of the tensor-core backward (bf16, M in {128, 256}, D in
{16, 32}) against the double-precision oracle.  With M = 256 the decode
stage runs as the statistics pass (decode pipeline) and the dZ pass (encode
pipeline, 48-token tiles), and pass B once per half of the latents.

Covers single tokens, one tile, ragged tails, many tiles and several chunks
per (b, h), shared and per-batch latents, both forms of the encode weights
(the one-exponential form and, for heads whose lse spread is large, the
exact form), near-uniform softmaxes (small latents), the device error word,
poisoned workspaces and bitwise reproducibility.
"""
import math

import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import assert_close, assert_close_scaled

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF16 = torch.bfloat16


def _run(B, H, N, M, D, seed, per_batch_q=False, scale_mul=1.0, q_std=1.0, poison=False):
    s = scale_mul / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=BF16, seed=seed, per_batch_q=per_batch_q,
                    with_dy=True, q_std=q_std)
    g = {k: v.to(DEV) for k, v in x.items()}
    assert fl.bwd_path(B, H, N, M, D, BF16) == 1
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    ws = fl.alloc_workspace(fl.FLARE_OP_BWD, B, H, N, M, D, BF16, DEV)
    if poison:
        ws.fill_(0xFF)   # NaN in every float the kernels might read unwritten
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s, workspace=ws)
    assert fl.device_status(ws) == 0
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    if scale_mul == 1.0:
        assert_close(dV, dVo, BF16, "dV")
        assert_close(dK, dKo, BF16, "dK")
        assert_close(dQ, dQo, BF16, "dQ")
    else:   # sharper softmax: gradients well above unit scale
        assert_close_scaled(dV, dVo, "dV")
        assert_close_scaled(dK, dKo, "dK")
        assert_close_scaled(dQ, dQo, "dQ")
    return dQ, dK, dV


@pytest.mark.parametrize("D", [32, 16])
@pytest.mark.parametrize("N", [2, 127, 128, 129, 383, 1000])
def test_tc_bwd_sizes(N, D):
    _run(2, 2, N, 128, D, seed=100 + N)


@pytest.mark.parametrize("D", [32, 16])
@pytest.mark.parametrize("N", [2, 47, 48, 49, 129, 1000])
def test_tc_bwd_sizes_m256(N, D):
    # both tile sizes of the M = 256 path: 48 tokens (dZ pass), 128 (the
    # rest); one token (dK = 0 exactly) is the closed-form test below
    _run(2, 2, N, 256, D, seed=200 + N)


@pytest.mark.parametrize("M", [128, 256])
@pytest.mark.parametrize("D", [32, 16])
def test_tc_bwd_single_token_closed_form(D, M):
    # One token: every latent encodes Z[m] = V[0] and the decode returns
    # Y[0] = V[0] whatever K and Q are, so dQ = dK = 0 and dV = dY.  The
    # kernels take every derived sum with the bf16 operands the tensor cores
    # use, so the zeros come out at float32 rounding level.
    B, H, N = 2, 2, 1
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=BF16, seed=4, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    torch.cuda.synchronize()
    assert float(dQ.float().abs().max()) <= 1e-3
    assert float(dK.float().abs().max()) <= 1e-3
    assert float((dV.float() - g["dY"].float()).abs().max()) <= 3e-2


@pytest.mark.parametrize("M", [128, 256])
@pytest.mark.parametrize("D", [32, 16])
def test_tc_bwd_per_batch_latents(D, M):
    _run(3, 2, 700, M, D, seed=7, per_batch_q=True)


@pytest.mark.parametrize("M", [128, 256])
@pytest.mark.parametrize("D", [32, 16])
def test_tc_bwd_many_tiles_and_chunks(D, M):
    # 40,000 tokens per head: 313 tiles, split over several CTAs per head
    _run(1, 2, 40000, M, D, seed=9)


@pytest.mark.parametrize("M", [128, 256])
@pytest.mark.parametrize("scale_mul", [4.0, 100.0])
def test_tc_bwd_sharp_softmax_exact_form(scale_mul, M):
    # Large logits spread the lse over more than 64 (log2 units) on some heads:
    # those heads take the exact form of the encode weights.
    _run(2, 2, 900, M, 32, seed=11, scale_mul=scale_mul)


@pytest.mark.parametrize("M", [128, 256])
def test_tc_bwd_near_uniform_softmax(M):
    _run(2, 2, 3000, M, 32, seed=12, q_std=0.02)


@pytest.mark.parametrize("M", [128, 256])
def test_tc_bwd_poisoned_workspace(M):
    _run(1, 3, 517, M, 32, seed=13, poison=True)


@pytest.mark.parametrize("M", [128, 256])
def test_tc_bwd_bitwise_reproducible(M):
    B, H, N, D = 2, 2, 5000, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=BF16, seed=14, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    a = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    b = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("M", [128, 256])
def test_tc_bwd_mixed_heads_fast_and_exact(M):
    # Head 1's latents are scaled up so its lse spreads far beyond 64 (log2
    # units) and it takes the exact form, while head 0 takes the
    # one-exponential form, in the same launch.
    B, H, N, D = 2, 2, 1500, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=BF16, seed=15, with_dy=True)
    x["Q"][1] = (x["Q"][1].float() * 40.0).to(BF16)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    spread = (lse.float().amax(-1) - lse.float().amin(-1)) * math.log2(math.e)
    assert float(spread[:, 1].min()) > 64.0 and float(spread[:, 0].max()) < 64.0
    ws = fl.alloc_workspace(fl.FLARE_OP_BWD, B, H, N, M, D, BF16, DEV)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s, workspace=ws)
    assert fl.device_status(ws) == 0
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    for hh in (0, 1):
        chk = assert_close if hh == 0 else (lambda a, b, dt, w: assert_close_scaled(a, b, w))
        chk(dV[:, hh], dVo[:, hh], BF16, f"dV head {hh}")
        chk(dK[:, hh], dKo[:, hh], BF16, f"dK head {hh}")
        chk(dQ[hh], dQo[hh], BF16, f"dQ head {hh}")
