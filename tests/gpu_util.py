"""Helpers for the GPU parity tests (comparison metrics and tolerances)."""
import os

import numpy as np
import torch

# Tolerances of the parity bar: float32 inputs -> relative Frobenius error
# <= 1e-5; bf16 inputs with float32 accumulation -> relative Frobenius error
# <= 1e-2 and max-abs error <= 3e-2.
TOL_F32_REL = 1e-5
TOL_BF16_REL = 1e-2
TOL_BF16_ABS = 3e-2
# Gradients from float32 inputs carry the same bar as the forward.
TOL_F32_GRAD_REL = 1e-5

# Every comparison made through the helpers below, as
# (test, what, dtype, rel_fro, max_abs): written out at the end of the
# session when FLARE_PARITY_LOG names a file (see conftest.py), so that the
# measured errors behind each bar can be quoted.
RECORDS = []


def _record(what, dtype, r, m):
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    RECORDS.append({"test": test, "what": what, "dtype": str(dtype).replace("torch.", ""),
                    "rel_fro": r, "max_abs": m})


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
    _record(what, dtype, r, max_abs(got, ref))
    if dtype == torch.float32:
        assert r <= rel_f32, f"{what}: rel_fro {r:.3e} > {rel_f32}"
    else:
        m = max_abs(got, ref)
        assert r <= TOL_BF16_REL and m <= TOL_BF16_ABS, \
            f"{what}: rel_fro {r:.3e} (<= {TOL_BF16_REL}), max_abs {m:.3e} (<= {TOL_BF16_ABS})"
    return r


def assert_close_scaled(got, ref, what=""):
    """bf16 parity for outputs that are not of unit scale: relative Frobenius
    error <= 1e-2 and max-abs error <= 3e-2 x max(1, max |ref|).  A bf16
    number of magnitude >= 8 has a rounding step of 1/16 or more, so an
    absolute 3e-2 bound cannot hold for it even after one correct rounding."""
    r = rel_fro(got, ref)
    m = max_abs(got, ref)
    _record(what, "scaled", r, m)
    big = float(np.abs(to64(ref)).max()) if to64(ref).size else 0.0
    bound = TOL_BF16_ABS * max(1.0, big)
    assert r <= TOL_BF16_REL and m <= bound, \
        f"{what}: rel_fro {r:.3e} (<= {TOL_BF16_REL}), max_abs {m:.3e} (<= {bound:.3e}, max|ref| {big:.3e})"
    return r
