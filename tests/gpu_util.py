"""Helpers for the GPU parity tests (comparison metrics and tolerances)."""
import numpy as np
import torch

# Tolerances of the parity bar: float32 inputs -> relative Frobenius error
# <= 1e-5; bf16 inputs with float32 accumulation -> relative Frobenius error
# <= 1e-2 and max-abs error <= 3e-2.
TOL_F32_REL = 1e-5
TOL_BF16_REL = 1e-2
TOL_BF16_ABS = 3e-2
# Gradients computed in float32 from float32 inputs: the recompute adds a
# few more roundings than the forward; 1e-4 relative Frobenius.
TOL_F32_GRAD_REL = 1e-4


def to64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def rel_fro(a, b) -> float:
    a, b = to64(a), to64(b)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b) -> float:
    a, b = to64(a), to64(b)
    return float(np.abs(a - b).max()) if a.size else 0.0


def assert_close(got, ref, dtype, what="", rel_f32=TOL_F32_REL):
    r = rel_fro(got, ref)
    if dtype == torch.float32:
        assert r <= rel_f32, f"{what}: rel_fro {r:.3e} > {rel_f32}"
    else:
        m = max_abs(got, ref)
        assert r <= TOL_BF16_REL and m <= TOL_BF16_ABS, \
            f"{what}: rel_fro {r:.3e} (<= {TOL_BF16_REL}), max_abs {m:.3e} (<= {TOL_BF16_ABS})"
    return r
