"""Seeded synthetic inputs for FLARE workloads.

This module is the only code shared by the CUDA path's tests/benchmark and
the CPU oracle.  It holds no part of the method's arithmetic: it draws
i.i.d. standard normal tensors in a fixed order (Q, K, V, then dY) from one
seeded CPU generator, and rounds them to the working dtype (round to nearest
even for bfloat16).  The oracle reads the rounded values widened exactly to
float64, so both sides see bit-identical inputs.

The shapes are the workloads the FLARE pages describe (PDE meshes of 256x256
points, million-point unstructured meshes, long-sequence classification);
no dataset is used.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    op: str          # "fwd", "pp_fwd" or "fwd_bwd"
    dtype: str       # "f32" or "bf16"
    B: int
    H: int
    N: int
    M: int
    D: int
    note: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads of the benchmark table (sizes as stated there).
WORKLOADS = {
    "c1_fwd_f32_tiny": Workload("c1_fwd_f32_tiny", "fwd", "f32", 1, 4, 1024, 32, 16,
                                "tiny fp32 case, checkable against the full N x N mixing matrix"),
    "c2_fwd_bf16_mesh256": Workload("c2_fwd_bf16_mesh256", "fwd", "bf16", 4, 8, 65536, 128, 16,
                                    "256x256 mesh-sized token count, hidden 128"),
    "c3_fwd_bf16_1M": Workload("c3_fwd_bf16_1M", "fwd", "bf16", 1, 16, 1048576, 256, 32,
                               "million-point unstructured mesh, hidden 512 (headline)"),
    "c4_ppfwd_bf16_256k": Workload("c4_ppfwd_bf16_256k", "pp_fwd", "bf16", 2, 8, 262144, 256, 32,
                                   "FLARE++ forward"),
    "c5_fwdbwd_bf16_16k": Workload("c5_fwdbwd_bf16_16k", "fwd_bwd", "bf16", 8, 8, 16384, 128, 32,
                                   "long-sequence classification shape, hidden 256"),
}


def make_inputs(B: int, H: int, N: int, M: int, D: int, dtype=torch.bfloat16, seed: int = 0,
                per_batch_q: bool = False, with_dy: bool = False, q_std: float = 1.0):
    """Return a dict of CPU tensors Q, K, V (and dY) in ``dtype``.

    Q is [H,M,D] (learned latents shared over the batch) unless
    ``per_batch_q``, then [B,H,M,D].  K, V, dY are [B,H,N,D].  Values are
    N(0,1) (Q optionally scaled by ``q_std``), drawn in the order Q, K, V, dY
    in float32 from ``torch.Generator('cpu').manual_seed(seed)``, then
    rounded to ``dtype``.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    qshape = (B, H, M, D) if per_batch_q else (H, M, D)
    out = {}
    out["Q"] = (torch.randn(qshape, generator=g, dtype=torch.float32) * q_std).to(dtype)
    out["K"] = torch.randn((B, H, N, D), generator=g, dtype=torch.float32).to(dtype)
    out["V"] = torch.randn((B, H, N, D), generator=g, dtype=torch.float32).to(dtype)
    if with_dy:
        out["dY"] = torch.randn((B, H, N, D), generator=g, dtype=torch.float32).to(dtype)
    return out


def make_workload_inputs(w: Workload, seed: int = 0):
    return make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed,
                       with_dy=(w.op == "fwd_bwd"))
