"""The autograd functions: gradients through a graph equal the library's
backward and the oracle's gradient."""
import math

import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("pp", [False, True], ids=["flare", "flare_pp"])
def test_autograd_matches_library_and_oracle(pp):
    B, H, N, M, D = 2, 2, 700, 128, 32
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=91, with_dy=True)
    g = {k: v.to(DEV).requires_grad_(k != "dY") for k, v in x.items()}
    fn = fl.flare_pp if pp else fl.flare
    Y = fn(g["Q"], g["K"], g["V"], s)
    (Y.float() * g["dY"].float()).sum().backward()
    if pp:
        _, Qd, Z, lse = fl.flare_pp_fwd(g["Q"].detach(), g["K"].detach(), g["V"].detach(), s,
                                        save=True)
        ref = fl.flare_pp_bwd(g["Q"].detach(), g["K"].detach(), g["V"].detach(), g["dY"], Qd, Z,
                              lse, s)
        orc = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    else:
        _, Z, lse = fl.flare_fwd(g["Q"].detach(), g["K"].detach(), g["V"].detach(), s, save=True)
        ref = fl.flare_bwd(g["Q"].detach(), g["K"].detach(), g["V"].detach(), g["dY"], Z, lse, s)
        orc = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    torch.cuda.synchronize()
    for name, r, o in zip(("Q", "K", "V"), ref, orc):
        assert torch.equal(g[name].grad, r), name
        assert_close(g[name].grad, o, torch.bfloat16, "d" + name)


def test_autograd_broadcast_gradient_and_lengths():
    # sum() hands the backward a zero-stride gradient; lengths pass through
    B, H, N, M, D = 2, 2, 300, 128, 16
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=92)
    lens = [300, 131]
    g = {k: v.to(DEV).requires_grad_() for k, v in x.items()}
    Y = fl.flare(g["Q"], g["K"], g["V"], s,
                 seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV))
    Y.float().sum().backward()
    ones = torch.ones(B, H, N, D)
    dQo, dKo, dVo = oracle.flare_bwd(x["Q"], x["K"], x["V"], ones, s, seq_lens=lens)
    assert_close(g["Q"].grad, dQo, torch.bfloat16, "dQ")
    for b, L in enumerate(lens):
        assert_close(g["K"].grad[b, :, :L], dKo[b, :, :L], torch.bfloat16, "dK")
        assert_close(g["V"].grad[b, :, :L], dVo[b, :, :L], torch.bfloat16, "dV")
        assert not g["K"].grad[b, :, L:].any() and not g["V"].grad[b, :, L:].any()
