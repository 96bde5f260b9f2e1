"""flare_fwd_noalloc -- the forward for callers that cannot allocate device
memory (a plugin whose host framework owns all device allocations and gives
it no workspace, or a running loop where cudaMalloc is not allowed) -- must
give the same results as flare_fwd with a caller workspace.

This file is collected last on purpose, so that a run stopping at the
first failure has already run every other test.  It calls the C entry point
directly through ctypes and makes two calls in a row on each case: the
shared scratch array keeps the previous call's contents, which must not
leak into the next result.
"""
import ctypes
import math

import pytest
import torch

import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import assert_close

pytestmark = pytest.mark.gpu


def _noalloc_c_call(g, Y, s):
    lib = fl.load()
    B, H, N, D = g["K"].shape
    M = g["Q"].shape[-2]
    qbs = 0 if g["Q"].dim() == 3 else H * M * D
    dt = fl.FLARE_F32 if g["K"].dtype == torch.float32 else fl.FLARE_BF16
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.flare_fwd_noalloc(p(g["Q"]), qbs, p(g["K"]), p(g["V"]), p(Y), B, H, N, M, D, dt,
                                 s, None, None, stream)


@pytest.mark.parametrize("dtype,B,H,N,M,D,per_batch_q", [
    (torch.bfloat16, 1, 2, 5000, 256, 32, False),   # tensor-core kernels
    (torch.bfloat16, 2, 3, 777, 128, 16, True),
    (torch.float32, 1, 4, 1024, 32, 16, False),     # CUDA-core kernels
])
def test_noalloc_matches_workspace_entry_point(dtype, B, H, N, M, D, per_batch_q):
    s = 1.0 / math.sqrt(D)
    for seed in (11, 12):   # two calls in a row with different inputs
        x = make_inputs(B, H, N, M, D, dtype=dtype, seed=seed, per_batch_q=per_batch_q)
        g = {k: v.cuda() for k, v in x.items()}
        ref = fl.flare_fwd(g["Q"], g["K"], g["V"], s)
        Y = torch.full_like(g["K"], float("nan"))
        assert _noalloc_c_call(g, Y, s) == 0
        torch.cuda.synchronize()
        assert not torch.isnan(Y.float()).any()
        assert_close(Y, ref.float().cpu().double().numpy(), dtype, f"Y seed {seed}")
    assert fl.noalloc_device_status() == 0   # no bounded wait ran out


def test_noalloc_large_then_small_call():
    # A large call fills more of the shared scratch array (more chunk
    # records, other offsets) than a small one reads: the small call after
    # it must not pick up the large call's leftovers.
    cases = [(torch.bfloat16, 1, 2, 5000, 256, 32), (torch.bfloat16, 1, 1, 777, 128, 32),
             (torch.bfloat16, 1, 2, 5000, 256, 32), (torch.bfloat16, 2, 1, 300, 128, 16)]
    for i, (dtype, B, H, N, M, D) in enumerate(cases):
        s = 1.0 / math.sqrt(D)
        x = make_inputs(B, H, N, M, D, dtype=dtype, seed=30 + i)
        g = {k: v.cuda() for k, v in x.items()}
        ref = fl.flare_fwd(g["Q"], g["K"], g["V"], s)
        Y = torch.full_like(g["K"], float("nan"))
        assert _noalloc_c_call(g, Y, s) == 0
        torch.cuda.synchronize()
        assert_close(Y, ref.float().cpu().double().numpy(), dtype, f"Y case {i}")
    assert fl.noalloc_device_status() == 0


def test_noalloc_rejects_sizes_beyond_the_scratch_array():
    # 1024 heads: Z alone takes 1024 x 256 x 32 x 4 B = 32 MiB of scratch.
    B, H, N, M, D = 64, 16, 65536, 256, 32
    need = fl.workspace_size(fl.FLARE_OP_FWD, B, H, N, M, D, torch.bfloat16)
    assert need > fl.NOALLOC_SCRATCH_BYTES   # checked before any call: nothing is launched
    small = make_inputs(1, 1, 8, M, D, dtype=torch.bfloat16)
    q = small["Q"].cuda()
    big = torch.empty((1, 1, 1, D), dtype=torch.bfloat16, device="cuda")   # never touched
    lib = fl.load()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.flare_fwd_noalloc(p(q), 0, p(big), p(big), p(big), B, H, N, M, D, fl.FLARE_BF16,
                               0.1, None, None, None)
    assert st == 3
    assert b"scratch" in lib.flare_last_error_detail()
