"""The forward from and to host memory (flare_fwd_host): chunked copies on
a second stream overlapped with the compute, against the oracle and the
device-buffer call."""
import math

import pytest
import torch

import oracle
import rank_latent_attention_flare_b200 as fl
from flare_inputs import make_inputs
from gpu_util import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


# (B, H, N, M, D, per-batch latents): heads per chunk 1 (6 heads), and 2
# with a last chunk of one head (17 heads); shared and per-batch Q
CASES = [(2, 3, 1000, 128, 32, False), (1, 17, 700, 256, 16, False), (2, 3, 500, 64, 32, True)]


@pytest.mark.parametrize("B,H,N,M,D,per_batch", CASES)
def test_fwd_host_matches_oracle_and_device_call(B, H, N, M, D, per_batch):
    s = 1.0 / math.sqrt(D)
    x = make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=91 + H)
    if per_batch:   # per-batch latents: the shared ones, perturbed per batch element
        g = torch.Generator().manual_seed(92)
        x["Q"] = (x["Q"].float().unsqueeze(0) +
                  0.1 * torch.randn((B,) + tuple(x["Q"].shape), generator=g)).to(torch.bfloat16)
    hx = {k: x[k].contiguous().pin_memory() for k in ("Q", "K", "V")}
    cs = torch.cuda.Stream()
    Y = fl.flare_fwd_host(hx["Q"], hx["K"], hx["V"], s, copy_stream=cs)
    torch.cuda.synchronize()
    assert not Y.is_cuda and torch.isfinite(Y.float()).all()
    Yo, _, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert_close(Y, Yo, torch.bfloat16, "Y (host call)")
    Yd = fl.flare_fwd(x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV), s)
    torch.cuda.synchronize()
    assert_close(Y, Yd.cpu(), torch.bfloat16, "Y (host call vs device call)")


def test_fwd_host_reuses_buffers_and_orders_after_the_stream():
    # two calls into the same device buffers and workspace, the second on new
    # inputs: the second's copies must wait for the first call's work
    B, H, N, M, D = 1, 4, 800, 128, 32
    s = 1.0 / math.sqrt(D)
    xs = [make_inputs(B, H, N, M, D, dtype=torch.bfloat16, seed=93 + i) for i in range(2)]
    bufs = {"Q": torch.empty(xs[0]["Q"].shape, dtype=torch.bfloat16, device=DEV),
            **{k: torch.empty((B, H, N, D), dtype=torch.bfloat16, device=DEV)
               for k in ("K", "V", "Y")}}
    cs = torch.cuda.Stream()
    outs = []
    for x in xs:
        hx = {k: x[k].contiguous().pin_memory() for k in ("Q", "K", "V")}
        outs.append(fl.flare_fwd_host(hx["Q"], hx["K"], hx["V"], s, device_buffers=bufs,
                                      copy_stream=cs))
    torch.cuda.synchronize()
    for x, Y in zip(xs, outs):
        Yo, _, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
        assert_close(Y, Yo, torch.bfloat16, "Y")
