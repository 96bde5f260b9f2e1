"""GPU parity of the FLARE forward (through the C ABI) against the oracle.

Shapes span several 128-token tiles with a ragged tail, single-token and
single-tile heads, every supported M class and both D, shared and per-batch
latents, float32 (CUDA-core kernels) and bf16 (tensor-core kernels where the
shape is covered).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda"

SHAPES = [
    # B, H, N, M, D
    (1, 1, 1, 16, 16),
    (1, 2, 7, 32, 16),
    (2, 3, 129, 64, 32),
    (1, 2, 1000, 128, 16),
    (2, 2, 1000, 128, 32),
    (1, 2, 1000, 256, 32),
    (1, 1, 4097, 256, 16),
    (3, 1, 385, 256, 32),
    (1, 2, 300, 48, 32),
    (2, 1, 2049, 128, 32),
]


def _run(x, s, dtype, per_batch_q=False, save=True):
    g = {k: v.to(DEV) for k, v in x.items()}
    return fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=save)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("B,H,N,M,D", SHAPES)
def test_fwd_matches_oracle(B, H, N, M, D, dtype):
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=N + M + D)
    Y, Z, lse = _run(x, s, dtype)
    torch.cuda.synchronize()
    Yo, Zo, lo = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Z, Zo, dtype, "Z")
    assert_close(Y, Yo, dtype, "Y")
    assert_close(lse, lo, torch.float32 if dtype == torch.float32 else dtype, "lse")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("M,D", [(128, 16), (256, 32), (32, 16)])
def test_fwd_per_batch_latents(M, D, dtype):
    B, H, N = 3, 2, 700
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=77, per_batch_q=True)
    Y, Z, lse = _run(x, s, dtype)
    torch.cuda.synchronize()
    Yo, Zo, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Z, Zo, dtype, "Z")
    assert_close(Y, Yo, dtype, "Y")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_fwd_large_scale_stable(dtype):
    # scale 100x the usual 1/sqrt(D): softmaxes are sharply peaked, the
    # running max must keep every exponential finite.
    B, H, N, M, D = 1, 2, 900, 128, 32
    s = 100.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=5)
    Y, Z, lse = _run(x, s, dtype)
    torch.cuda.synchronize()
    assert torch.isfinite(Y.float()).all() and torch.isfinite(Z).all()
    Yo, Zo, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Z, Zo, dtype, "Z")
    assert_close(Y, Yo, dtype, "Y")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_fwd_writes_every_output_and_is_deterministic(dtype):
    B, H, N, M, D = 2, 2, 1537, 256, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=9)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, dtype, DEV)
    ws.fill_(0xFF)  # poison: NaN bit patterns everywhere in the workspace
    Y1 = torch.full_like(g["K"], float("nan"))
    fl.flare_fwd(g["Q"], g["K"], g["V"], s, workspace=ws, out=Y1)
    Y2 = torch.full_like(g["K"], float("nan"))
    fl.flare_fwd(g["Q"], g["K"], g["V"], s, workspace=ws, out=Y2)
    assert fl.device_status(ws) == 0
    assert not torch.isnan(Y1.float()).any()
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_stage_calls_equal_fused_call(dtype):
    B, H, N, M, D = 1, 3, 2000, 128, 16
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=dtype, seed=10)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, dtype, DEV)
    Y1, Z1, l1 = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, workspace=ws)
    Z2 = torch.empty_like(Z1)
    l2 = torch.empty_like(l1)
    fl.flare_encode(g["Q"], g["K"], g["V"], s, workspace=ws)
    fl.flare_combine(B, H, N, M, D, dtype, workspace=ws, Z_save=Z2, lse_save=l2)
    Y2 = fl.flare_decode(g["Q"], g["K"], s, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(Z1, Z2) and torch.equal(l1, l2)


def test_gpu_rejects_invalid_arguments_without_side_effects():
    B, H, N, M, D = 1, 2, 100, 32, 16
    x = {k: v.to(DEV) for k, v in make_inputs(B, H, N, M, D, dtype=torch.float32).items()}
    Y = torch.zeros_like(x["K"])
    with pytest.raises(fl.FlareError) as e:
        fl.flare_fwd(x["Q"], x["K"], x["V"], scale=-1.0, out=Y)
    assert e.value.status == 1
    small = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(fl.FlareError) as e:
        fl.flare_fwd(x["Q"], x["K"], x["V"], workspace=small, out=Y)
    assert e.value.status == 3
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y) == 0


@pytest.mark.parametrize("M", [128, 256])
@pytest.mark.parametrize("regime", ["spiky", "growing"])
def test_encode_running_max_over_many_tiles(M, regime):
    # One head of 262,144 tokens: every encode CTA walks many 48-token tiles,
    # so the running-max machinery is exercised.  "spiky": scale x100 makes
    # tile maxima jump by far more than 2^64 (tiles recomputed with the exact
    # max); "growing": keys grow steadily along the sequence, so the running
    # max keeps rising by more than 2^8 (deferred rescales).
    B, H, N, D = 1, 1, 262144, 32
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=21 + M)
    if regime == "spiky":
        s = 100.0 / math.sqrt(D)
    else:
        s = 1.0 / math.sqrt(D)
        ramp = torch.linspace(0.25, 4.0, N).view(1, 1, N, 1)
        x["K"] = (x["K"].float() * ramp).to(torch.bfloat16)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, torch.bfloat16, DEV)
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, workspace=ws)
    assert fl.device_status(ws) == 0
    assert torch.isfinite(Z).all() and torch.isfinite(Y.float()).all()
    Zo, lo = oracle.encode(x["Q"], x["K"], x["V"], s)
    rows = np.unique(np.concatenate([np.arange(64), np.arange(N - 64, N),
                                     np.random.default_rng(0).integers(0, N, 2048)]))
    Yo = oracle.decode_rows(x["Q"], x["K"], Zo, s, rows)
    assert_close(Z, Zo, torch.bfloat16, "Z")
    assert_close(lse, lo, torch.bfloat16, "lse")
    assert_close(Y.float().cpu().reshape(-1, D)[rows], Yo, torch.bfloat16, "Y")


def test_decode_row_reference_mixed_within_warps():
    # M = 256: each token row takes the first 32-logit chunk's max as its
    # reference when c |k| max |q| is within 2^64 of it, else the warp
    # computes the exact max.  Every 7th key scaled x40 puts rows of both
    # kinds in every warp of a tile.
    B, H, N, M, D = 1, 2, 3000, 256, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=27)
    x["K"][:, :, ::7] = (x["K"][:, :, ::7].float() * 40.0).to(torch.bfloat16)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, torch.bfloat16, DEV)
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, workspace=ws)
    assert fl.device_status(ws) == 0
    Yo, Zo, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert torch.isfinite(Y.float()).all()
    for sel, what in ((slice(0, None, 7), "scaled rows"), (slice(1, None, 7), "plain rows")):
        assert_close(Y[:, :, sel], Yo[:, :, sel], torch.bfloat16, what)
    assert_close(Y, Yo, torch.bfloat16, "Y")
    assert_close(Z, Zo, torch.bfloat16, "Z")


@pytest.mark.parametrize("M", [16, 48, 64, 80, 112, 144, 192, 240])
@pytest.mark.parametrize("D", [16, 32])
def test_fwd_tensor_core_padded_latents(M, D):
    # Latent counts other than 128 and 256 run on the tensor-core kernels
    # with the latent tile padded by zero rows: never stored by the encode,
    # never weighted by the decode.
    B, H, N = 2, 2, 1000
    s = 1.0 / math.sqrt(D)
    assert fl.fwd_path(B, H, N, M, D, torch.bfloat16) == 1
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=100 + M + D)
    g = {k: v.to(DEV) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, B, H, N, M, D, torch.bfloat16, DEV)
    ws.fill_(0xFF)
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True, workspace=ws)
    assert fl.device_status(ws) == 0
    Yo, Zo, lo = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Z, Zo, torch.bfloat16, f"Z M={M}")
    assert_close(lse, lo, torch.bfloat16, f"lse M={M}")
    assert_close(Y, Yo, torch.bfloat16, f"Y M={M}")


@pytest.mark.parametrize("M", [64, 192])
def test_padded_latents_per_batch_flare_pp_and_backward(M):
    # per-batch latents (FLARE++'s Q_dyn path) and the backward (CUDA cores
    # for these M) from the tensor-core forward's saved Z and lse
    B, H, N, D = 2, 2, 777, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=200 + M, with_dy=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    Y, Qd = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], s)
    Yo, Qdo, _, _ = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Qd, Qdo, torch.bfloat16, "Q_dyn")
    assert_close(Y, Yo, torch.bfloat16, "Y (FLARE++)")
    Y, Z, lse = fl.flare_fwd(g["Q"], g["K"], g["V"], s, save=True)
    dQ, dK, dV = fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, s)
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    assert_close(dV, dVo, torch.bfloat16, "dV")
    assert_close(dK, dKo, torch.bfloat16, "dK")
    assert_close(dQ, dQo, torch.bfloat16, "dQ")
