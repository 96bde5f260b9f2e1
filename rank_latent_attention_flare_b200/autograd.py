"""torch.autograd functions over the library's forward and backward calls.

Argument marshalling only: the forward saves what the library's backward
needs (Z and lse, and FLARE++'s Q_dyn), and the backward calls flare_bwd /
flare_pp_bwd.  Both directions run in libflare.so.
"""
from __future__ import annotations

import importlib
from typing import Optional

import torch

# the binding module (the package's `flare` attribute is the autograd function)
_f = importlib.import_module(__package__ + ".flare")


def _token_grad(t: torch.Tensor) -> torch.Tensor:
    """An upstream gradient the library can read in place ([B,H,N,D] with D
    contiguous and 16-byte row strides), else a contiguous copy (autograd
    hands out broadcast gradients with zero strides, e.g. after a sum)."""
    esz = t.element_size()
    ok = t.dim() == 4 and t.stride(-1) == 1 and all(
        s > 0 and (s * esz) % 16 == 0 for s in t.stride()[:3])
    return t if ok and t.data_ptr() % 16 == 0 else t.contiguous()


class FlareFunction(torch.autograd.Function):
    """Y = FLARE(Q, K, V): encode then decode (see flare_fwd)."""

    @staticmethod
    def forward(ctx, Q, K, V, scale, seq_lens):
        Y, Z, lse = _f.flare_fwd(Q, K, V, scale, save=True, seq_lens=seq_lens)
        ctx.save_for_backward(Q, K, V, Z, lse)
        ctx.scale = scale
        ctx.seq_lens = seq_lens
        return Y

    @staticmethod
    def backward(ctx, dY):
        Q, K, V, Z, lse = ctx.saved_tensors
        dQ, dK, dV = _f.flare_bwd(Q, K, V, _token_grad(dY), Z, lse, ctx.scale,
                                  seq_lens=ctx.seq_lens)
        return dQ, dK, dV, None, None


class FlarePPFunction(torch.autograd.Function):
    """Y = FLARE++(Q, K, V) with learned latents Q [H,M,D] (see flare_pp_fwd)."""

    @staticmethod
    def forward(ctx, Q, K, V, scale, seq_lens):
        Y, Qd, Z, lse = _f.flare_pp_fwd(Q, K, V, scale, save=True, seq_lens=seq_lens)
        ctx.save_for_backward(Q, K, V, Qd, Z, lse)
        ctx.scale = scale
        ctx.seq_lens = seq_lens
        return Y

    @staticmethod
    def backward(ctx, dY):
        Q, K, V, Qd, Z, lse = ctx.saved_tensors
        dQ, dK, dV = _f.flare_pp_bwd(Q, K, V, _token_grad(dY), Qd, Z, lse, ctx.scale,
                                     seq_lens=ctx.seq_lens)
        return dQ, dK, dV, None, None


def flare(Q, K, V, scale: Optional[float] = None,
          seq_lens: Optional[torch.Tensor] = None) -> torch.Tensor:
    """FLARE token mixing with autograd: Q [H,M,D] or [B,H,M,D]; K, V
    [B,H,N,D] (D contiguous, any other strides); optional int32 seq_lens [B]."""
    s = _f.default_scale(K.shape[-1]) if scale is None else float(scale)
    return FlareFunction.apply(Q, K, V, s, seq_lens)


def flare_pp(Q, K, V, scale: Optional[float] = None,
             seq_lens: Optional[torch.Tensor] = None) -> torch.Tensor:
    """FLARE++ token mixing with autograd: learned latents Q [H,M,D]."""
    s = _f.default_scale(K.shape[-1]) if scale is None else float(scale)
    return FlarePPFunction.apply(Q, K, V, s, seq_lens)
