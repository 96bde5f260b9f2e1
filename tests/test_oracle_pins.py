"""Pins of the CPU oracle to facts other than itself (CPU only).

Each test checks the oracle against something the pages or the mathematics
fix independently of the oracle's own code:

* a hand-derived worked example (tests/golden/flare_tiny_2x2.json) and a
  closed-form FLARE++ example;
* the full N x N mixing matrix W = softmax(s K Q^T) softmax(s Q K^T) of the
  FLARE abstract: row-stochastic, rank <= M, and W V = Y;
* closed forms (M = 1, constant V, Q = 0, identical latents) and the
  hard-max limit of a large scale, which pins indices and transposes;
* invariants (token permutation, linearity in V, key shift for the encode);
* the float64 SDPA library routine, since the abstracts state that each
  stage is one standard SDPA call;
* for the gradient: central finite differences of the oracle's forward,
  torch float64 autograd through the SDPA composition, and the identity
  sum_n dV[n] = sum_n dY[n] (W is row-stochastic).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from flare_inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _x(B, H, N, M, D, seed=0, per_batch_q=False, with_dy=False, q_std=1.0):
    return {k: v.double().numpy() for k, v in
            make_inputs(B, H, N, M, D, dtype=torch.float64, seed=seed,
                        per_batch_q=per_batch_q, with_dy=with_dy, q_std=q_std).items()}


def _softmax(a, axis):
    a = a - a.max(axis=axis, keepdims=True)
    e = np.exp(a)
    return e / e.sum(axis=axis, keepdims=True)


# ---------------------------------------------------------------- golden ---

def test_golden_hand_derived_2x2():
    g = json.load(open(os.path.join(GOLDEN, "flare_tiny_2x2.json")))
    Q = np.array(g["Q"])[None]            # [H=1, M=2, D=1]
    K = np.array(g["K"])[None, None]      # [B=1, H=1, N=2, D=1]
    V = np.array(g["V"])[None, None]
    Y, Z, lse = oracle.flare_fwd(Q, K, V, g["scale"])
    np.testing.assert_allclose(Z[0, 0], np.array(g["Z"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.array(g["lse"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(Y[0, 0], np.array(g["Y"]), rtol=0, atol=1e-14)


def test_golden_flare_pp_closed_form():
    # Same tiny head as the golden file.  FLARE++ (FLARE++ abstract):
    # Z1 = (3, 4)  ->  Q_dyn = (3, ln3 + 4)
    # encode row 0: logits (0, 3)        -> Z0 = (1 + 5 e^3) / (1 + e^3)
    # encode row 1: logits (0, ln3 + 4)  -> Z1 = (1 + 15 e^4) / (1 + 3 e^4)
    # decode token 0 (k=0): logits (0, 0)            -> Y0 = (Z0 + Z1) / 2
    # decode token 1 (k=1): logits (3, ln3 + 4)      -> weights 1 : 3e
    #                                                -> Y1 = (Z0 + 3e Z1) / (1 + 3e)
    e = math.e
    Q = np.array([[[0.0], [math.log(3.0)]]])
    K = np.array([[[[0.0], [1.0]]]])
    V = np.array([[[[1.0], [5.0]]]])
    Y, Qd, Z, lse = oracle.flare_pp_fwd(Q, K, V, 1.0)
    z0 = (1 + 5 * e ** 3) / (1 + e ** 3)
    z1 = (1 + 15 * e ** 4) / (1 + 3 * e ** 4)
    np.testing.assert_allclose(Qd[0, 0, :, 0], [3.0, math.log(3.0) + 4.0], rtol=1e-14)
    np.testing.assert_allclose(Z[0, 0, :, 0], [z0, z1], rtol=1e-14)
    np.testing.assert_allclose(Y[0, 0, :, 0], [(z0 + z1) / 2, (z0 + 3 * e * z1) / (1 + 3 * e)],
                               rtol=1e-14)


# ------------------------------------------------- brute-force mixing matrix ---

@pytest.mark.parametrize("B,H,N,M,D", [(1, 2, 48, 8, 16), (2, 1, 64, 5, 4), (1, 4, 1024, 32, 16)])
def test_bruteforce_mixing_matrix(B, H, N, M, D):
    x = _x(B, H, N, M, D, seed=3)
    s = 1.0 / math.sqrt(D)
    Y, Z, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    for b in range(B):
        for h in range(H):
            q, k, v = x["Q"][h], x["K"][b, h], x["V"][b, h]
            Pe = _softmax(s * q @ k.T, axis=1)       # [M, N], softmax over tokens
            Pd = _softmax(s * k @ q.T, axis=1)       # [N, M], softmax over latents
            W = Pd @ Pe                              # [N, N]
            assert np.abs(W.sum(axis=1) - 1.0).max() <= 1e-12
            sv = np.linalg.svd(W, compute_uv=False)
            assert sv[M:].max(initial=0.0) <= 1e-10 * sv[0]
            err = np.linalg.norm(W @ v - Y[b, h]) / np.linalg.norm(Y[b, h])
            assert err <= 1e-12


# ------------------------------------------------------------ closed forms ---

def test_single_latent_every_row_is_weighted_mean():
    x = _x(2, 3, 200, 1, 8, seed=5)
    s = 0.35
    Y, Z, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    # decode over a single latent is the identity on Z[0]
    np.testing.assert_allclose(Y, np.broadcast_to(Z, Y.shape), rtol=0, atol=1e-14)
    # and Z[0] is the softmax-weighted mean of V
    for b in range(2):
        for h in range(3):
            w = np.exp(s * x["K"][b, h] @ x["Q"][h, 0])
            w /= w.sum()
            np.testing.assert_allclose(Z[b, h, 0], w @ x["V"][b, h], rtol=1e-12, atol=1e-14)


def test_constant_values_map_to_constant():
    x = _x(2, 2, 300, 16, 8, seed=6)
    c = np.linspace(-2.0, 3.0, 8)
    V = np.broadcast_to(c, x["V"].shape).copy()
    Y, Z, _ = oracle.flare_fwd(x["Q"], x["K"], V, 0.4)
    np.testing.assert_allclose(Z, np.broadcast_to(c, Z.shape), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Y, np.broadcast_to(c, Y.shape), rtol=1e-13, atol=1e-13)


def test_zero_latents_give_token_mean():
    x = _x(1, 2, 257, 8, 16, seed=7)
    Q = np.zeros_like(x["Q"])
    Y, Z, lse = oracle.flare_fwd(Q, x["K"], x["V"], 0.25)
    mean = x["V"].mean(axis=2)                      # [B,H,D]
    np.testing.assert_allclose(Z, np.broadcast_to(mean[:, :, None, :], Z.shape), atol=1e-13)
    np.testing.assert_allclose(Y, np.broadcast_to(mean[:, :, None, :], Y.shape), atol=1e-13)
    np.testing.assert_allclose(lse, math.log(257.0), rtol=1e-14)


def test_identical_latents_collapse_output():
    x = _x(1, 2, 100, 6, 8, seed=8)
    Q = np.broadcast_to(x["Q"][:, :1, :], x["Q"].shape).copy()
    Y, Z, _ = oracle.flare_fwd(Q, x["K"], x["V"], 0.3)
    np.testing.assert_allclose(Y, np.broadcast_to(Z[:, :, :1, :], Y.shape), atol=1e-14)


def test_hardmax_limit_pins_indices():
    # With a huge scale each softmax becomes a one-hot argmax: Z[m] is the
    # value of the key best aligned with latent m, and Y[n] is Z at the latent
    # best aligned with key n.  A transposed operand or a wrong softmax axis
    # fails this.
    x = _x(2, 2, 64, 12, 8, seed=9)
    s = 1e5
    Y, Z, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert np.isfinite(Y).all() and np.isfinite(Z).all()
    for b in range(2):
        for h in range(2):
            logits = x["Q"][h] @ x["K"][b, h].T     # [M, N]
            np.testing.assert_array_equal(Z[b, h], x["V"][b, h][logits.argmax(axis=1)])
            np.testing.assert_array_equal(Y[b, h], Z[b, h][logits.T.argmax(axis=1)])


def test_large_scale_is_stable():
    x = _x(1, 2, 512, 16, 16, seed=10)
    s = 100.0 / 4.0
    Y, Z, lse = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    assert np.isfinite(Y).all() and np.isfinite(Z).all() and np.isfinite(lse).all()
    assert np.abs(Y).max() <= np.abs(x["V"]).max() + 1e-12   # convex combinations


# ------------------------------------------------------------- invariants ---

def test_token_permutation_equivariance():
    x = _x(2, 2, 150, 8, 8, seed=11)
    perm = np.random.default_rng(0).permutation(150)
    Y, Z, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], 0.3)
    Yp, Zp, _ = oracle.flare_fwd(x["Q"], x["K"][:, :, perm], x["V"][:, :, perm], 0.3)
    np.testing.assert_allclose(Zp, Z, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(Yp, Y[:, :, perm], rtol=1e-12, atol=1e-14)


def test_linearity_in_values():
    x = _x(1, 2, 120, 8, 8, seed=12)
    V2 = _x(1, 2, 120, 8, 8, seed=13)["V"]
    a, b = 0.7, -1.3
    Y1, _, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], 0.3)
    Y2, _, _ = oracle.flare_fwd(x["Q"], x["K"], V2, 0.3)
    Y3, _, _ = oracle.flare_fwd(x["Q"], x["K"], a * x["V"] + b * V2, 0.3)
    np.testing.assert_allclose(Y3, a * Y1 + b * Y2, rtol=1e-11, atol=1e-13)


def test_encode_invariant_to_common_key_shift():
    x = _x(1, 2, 90, 8, 8, seed=14)
    c = np.linspace(-1, 1, 8)
    Z1, _ = oracle.encode(x["Q"], x["K"], x["V"], 0.3)
    Z2, _ = oracle.encode(x["Q"], x["K"] + c, x["V"], 0.3)
    np.testing.assert_allclose(Z2, Z1, rtol=1e-11, atol=1e-13)


def test_decode_rows_matches_full_decode():
    x = _x(2, 3, 77, 8, 8, seed=15)
    Z, _ = oracle.encode(x["Q"], x["K"], x["V"], 0.3)
    Y = oracle.decode(x["Q"], x["K"], Z, 0.3)
    rows = np.array([0, 5, 76, 77, 200, 2 * 3 * 77 - 1])
    Yr = oracle.decode_rows(x["Q"], x["K"], Z, 0.3, rows)
    np.testing.assert_array_equal(Yr, Y.reshape(-1, 8)[rows])


# ------------------------------------------------- SDPA library special case ---

def _sdpa_flare(Q, K, V, s):
    """The abstracts' two-SDPA-call form, float64, torch CPU."""
    Qb = Q if Q.dim() == 4 else Q.unsqueeze(0).expand(K.shape[0], -1, -1, -1)
    Z = F.scaled_dot_product_attention(Qb, K, V, scale=s)
    Y = F.scaled_dot_product_attention(K, Qb, Z, scale=s)
    return Y, Z


@pytest.mark.parametrize("per_batch_q", [False, True])
def test_sdpa_float64_crosscheck(per_batch_q):
    x = _x(2, 3, 333, 24, 16, seed=16, per_batch_q=per_batch_q)
    s = 0.25
    Y, Z, lse = oracle.flare_fwd(x["Q"], x["K"], x["V"], s)
    t = {k: torch.from_numpy(v) for k, v in x.items()}
    Yt, Zt = _sdpa_flare(t["Q"], t["K"], t["V"], s)
    np.testing.assert_allclose(Z, Zt.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Y, Yt.numpy(), rtol=1e-12, atol=1e-13)
    Qb = t["Q"] if per_batch_q else t["Q"].unsqueeze(0).expand(2, -1, -1, -1)
    lse_t = torch.logsumexp(s * Qb @ t["K"].transpose(-1, -2), dim=-1)
    np.testing.assert_allclose(lse, lse_t.numpy(), rtol=1e-13)


def test_flare_pp_sdpa_composition():
    x = _x(2, 2, 200, 16, 8, seed=17)
    s = 1.0 / math.sqrt(8)
    Y, Qd, Z, lse = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s)
    t = {k: torch.from_numpy(v) for k, v in x.items()}
    Qb = t["Q"].unsqueeze(0).expand(2, -1, -1, -1)
    Qdt = Qb + F.scaled_dot_product_attention(Qb, t["K"], t["V"], scale=s)
    Yt, Zt = _sdpa_flare(Qdt, t["K"], t["V"], s)
    np.testing.assert_allclose(Qd, Qdt.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Z, Zt.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Y, Yt.numpy(), rtol=1e-12, atol=1e-13)


def test_flare_pp_constant_values():
    # constant V: Z1 = c for every latent, Q_dyn = Q + c, and Y = c
    x = _x(1, 2, 64, 8, 4, seed=18)
    c = np.array([0.5, -1.0, 2.0, 0.0])
    V = np.broadcast_to(c, x["V"].shape).copy()
    Y, Qd, Z, _ = oracle.flare_pp_fwd(x["Q"], x["K"], V, 0.5)
    np.testing.assert_allclose(Qd[0], x["Q"] + c, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Y, np.broadcast_to(c, Y.shape), rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------- gradient ---

def _loss(Q, K, V, dY, s):
    Y, _, _ = oracle.flare_fwd(Q, K, V, s)
    return float((Y * dY).sum())


@pytest.mark.parametrize("per_batch_q", [False, True])
def test_bwd_central_finite_differences(per_batch_q):
    # Every element of Q, K and V at N = 64 (the gradient check size of the
    # fwd+bwd workload), small M and D to keep it quick.
    B, H, N, M, D = 2, 1, 64, 4, 4
    x = _x(B, H, N, M, D, seed=19, per_batch_q=per_batch_q, with_dy=True)
    s = 1.0 / math.sqrt(D)
    dQ, dK, dV = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    eps = 1e-5
    for name, grad in (("Q", dQ), ("K", dK), ("V", dV)):
        base = x[name]
        fd = np.empty_like(base)
        flat = base.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(x["Q"], x["K"], x["V"], x["dY"], s)
            flat[i] = old - eps
            lm = _loss(x["Q"], x["K"], x["V"], x["dY"], s)
            flat[i] = old
            fd.reshape(-1)[i] = (lp - lm) / (2 * eps)
        scale_ref = np.abs(fd).max()
        assert np.abs(grad - fd).max() <= 1e-7 * max(scale_ref, 1.0), name


@pytest.mark.parametrize("per_batch_q", [False, True])
def test_bwd_float64_autograd_crosscheck(per_batch_q):
    x = _x(2, 2, 150, 16, 8, seed=20, per_batch_q=per_batch_q, with_dy=True)
    s = 0.3
    dQ, dK, dV = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    t = {k: torch.from_numpy(v.copy()).requires_grad_(k != "dY") for k, v in x.items()}
    Yt, _ = _sdpa_flare(t["Q"], t["K"], t["V"], s)
    (Yt * t["dY"]).sum().backward()
    np.testing.assert_allclose(dQ, t["Q"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, t["K"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, t["V"].grad.numpy(), rtol=1e-10, atol=1e-12)


def test_bwd_value_gradient_sums_to_output_gradient():
    x = _x(2, 2, 300, 16, 8, seed=21, with_dy=True)
    _, _, dV = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], 0.3)
    np.testing.assert_allclose(dV.sum(axis=2), x["dY"].sum(axis=2), rtol=1e-11, atol=1e-11)


# ------------------------------------------------------- FLARE++ gradient ---

def _pp_loss(Q, K, V, dY, s):
    Y, _, _, _ = oracle.flare_pp_fwd(Q, K, V, s)
    return float((Y * dY).sum())


def test_pp_bwd_central_finite_differences():
    # Every element of the learned latents Q, of K and of V; the chain runs
    # through both uses of Q_dyn and through the first encode.
    B, H, N, M, D = 2, 1, 40, 4, 4
    x = _x(B, H, N, M, D, seed=23, with_dy=True)
    s = 1.0 / math.sqrt(D)
    dQ, dK, dV = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    eps = 1e-5
    for name, grad in (("Q", dQ), ("K", dK), ("V", dV)):
        base = x[name]
        fd = np.empty_like(base)
        flat = base.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + eps
            lp = _pp_loss(x["Q"], x["K"], x["V"], x["dY"], s)
            flat[i] = old - eps
            lm = _pp_loss(x["Q"], x["K"], x["V"], x["dY"], s)
            flat[i] = old
            fd.reshape(-1)[i] = (lp - lm) / (2 * eps)
        scale_ref = np.abs(fd).max()
        assert np.abs(grad - fd).max() <= 1e-7 * max(scale_ref, 1.0), name


def test_pp_bwd_float64_autograd_crosscheck():
    # The abstracts' form written with torch SDPA in float64: Q_dyn = Q +
    # SDPA(Q, K, V), then the two-call FLARE with Q_dyn; autograd's gradients.
    x = _x(2, 2, 130, 16, 8, seed=24, with_dy=True)
    s = 0.3
    dQ, dK, dV = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    t = {k: torch.from_numpy(v.copy()).requires_grad_(k != "dY") for k, v in x.items()}
    Qb = t["Q"].unsqueeze(0).expand(t["K"].shape[0], -1, -1, -1)
    Qd = Qb + F.scaled_dot_product_attention(Qb, t["K"], t["V"], scale=s)
    Yt, _ = _sdpa_flare(Qd, t["K"], t["V"], s)
    (Yt * t["dY"]).sum().backward()
    np.testing.assert_allclose(dQ, t["Q"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, t["K"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, t["V"].grad.numpy(), rtol=1e-10, atol=1e-12)


def test_pp_bwd_reduces_to_flare_when_the_correction_is_removed():
    # With V = 0 the first encode returns Z1 = 0, so Q_dyn = Q and the FLARE++
    # forward equals FLARE's; the gradients w.r.t. Q and K then equal FLARE's
    # (Z1 = P V is linear in V, so no dQ or dK flows through it at V = 0),
    # and dV gains only the first encode's P^T dQ_dyn term.
    B, H, N, M, D = 2, 2, 70, 8, 8
    x = _x(B, H, N, M, D, seed=25, with_dy=True)
    x["V"][:] = 0.0
    s = 0.4
    dQ, dK, dV = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    dQf, dKf, dVf = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    np.testing.assert_allclose(dK, dKf, rtol=1e-11, atol=1e-12)
    # dQ: FLARE's dQ with per-batch Q_dyn = Q, summed over the batch, is
    # FLARE's shared-Q dQ
    np.testing.assert_allclose(dQ, dQf, rtol=1e-11, atol=1e-12)


def test_encode_bwd_central_finite_differences():
    # The encode's gradient alone: d/dX of sum(Z * dZ), Z = softmax_N(s Q K^T) V
    # with Q shared over the batch; every element of Q, K and V.
    B, H, N, M, D = 2, 1, 30, 5, 4
    x = _x(B, H, N, M, D, seed=26)
    dZ = np.random.default_rng(27).standard_normal((B, H, M, D))
    s = 0.7
    dQ, dK, dV = oracle.encode_bwd(x["Q"], x["K"], x["V"], dZ, s)

    def loss():
        Z, _ = oracle.encode(x["Q"], x["K"], x["V"], s)
        return float((Z * dZ).sum())

    eps = 1e-5
    for name, grad in (("Q", dQ), ("K", dK), ("V", dV)):
        flat = x[name].reshape(-1)
        fd = np.empty(flat.size)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + eps
            lp = loss()
            flat[i] = old - eps
            lm = loss()
            flat[i] = old
            fd[i] = (lp - lm) / (2 * eps)
        assert np.abs(grad.reshape(-1) - fd).max() <= 1e-7 * max(np.abs(fd).max(), 1.0), name


def test_encode_bwd_is_the_part_of_the_flare_pp_gradient_through_z1():
    # FLARE++'s gradient = FLARE's gradient at Q_dyn (per-batch latents) plus
    # the encode's gradient with upstream dQ_dyn; dQ also collects dQ_dyn
    # summed over the batch.
    B, H, N, M, D = 2, 2, 50, 6, 4
    x = _x(B, H, N, M, D, seed=28, with_dy=True)
    s = 0.5
    dQ, dK, dV = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    _, Qd, _, _ = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s)
    dQd, dKa, dVa = oracle.flare_bwd(Qd, x["K"], x["V"], x["dY"], s)
    dQe, dKe, dVe = oracle.encode_bwd(x["Q"], x["K"], x["V"], dQd, s)
    np.testing.assert_allclose(dK, dKa + dKe, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dV, dVa + dVe, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dQ, dQd.sum(0) + dQe, rtol=1e-11, atol=1e-13)


# -------------------------------------------- sequence lengths (padding) ---

def _trunc(x, b, L):
    return {k: (v[b:b + 1, :, :L] if k in ("K", "V", "dY") else v) for k, v in x.items()}


def test_varlen_equals_each_sequence_alone():
    # seq_lens = [N, 7, 1, 0]: every batch element's outputs must equal the
    # unmasked oracle on its first L_b tokens alone (already pinned above);
    # padding rows of Y, dK, dV are zero; shared dQ is the sum over b.
    B, H, N, M, D = 4, 2, 30, 6, 4
    lens = [N, 7, 1, 0]
    x = _x(B, H, N, M, D, seed=31, with_dy=True)
    s = 0.6
    Y, Z, lse = oracle.flare_fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)
    dQ, dK, dV = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens)
    Ypp, Qd, Zpp, _ = oracle.flare_pp_fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)
    pQ, pK, pV = oracle.flare_pp_bwd(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens)
    dQsum = np.zeros_like(dQ)
    pQsum = np.zeros_like(pQ)
    for b, L in enumerate(lens):
        assert not Y[b, :, L:].any() and not dK[b, :, L:].any() and not dV[b, :, L:].any()
        assert not Ypp[b, :, L:].any() and not pK[b, :, L:].any() and not pV[b, :, L:].any()
        if L == 0:
            assert not Z[b].any() and np.all(lse[b] == -np.inf)
            np.testing.assert_array_equal(Qd[b], x["Q"])      # Z1 = 0
            continue
        t = _trunc(x, b, L)
        Yt, Zt, lt = oracle.flare_fwd(t["Q"], t["K"], t["V"], s)
        np.testing.assert_allclose(Y[b:b + 1, :, :L], Yt, rtol=0, atol=1e-14)
        np.testing.assert_allclose(Z[b:b + 1], Zt, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[b:b + 1], lt, rtol=0, atol=1e-13)
        tQ, tK, tV = oracle.flare_bwd(t["Q"], t["K"], t["V"], t["dY"], s)
        np.testing.assert_allclose(dK[b:b + 1, :, :L], tK, rtol=0, atol=1e-13)
        np.testing.assert_allclose(dV[b:b + 1, :, :L], tV, rtol=0, atol=1e-13)
        dQsum += tQ
        Yt, Qdt, _, _ = oracle.flare_pp_fwd(t["Q"], t["K"], t["V"], s)
        np.testing.assert_allclose(Ypp[b:b + 1, :, :L], Yt, rtol=0, atol=1e-13)
        np.testing.assert_allclose(Qd[b:b + 1], Qdt, rtol=0, atol=1e-14)
        tQ, tK, tV = oracle.flare_pp_bwd(t["Q"], t["K"], t["V"], t["dY"], s)
        np.testing.assert_allclose(pK[b:b + 1, :, :L], tK, rtol=0, atol=1e-12)
        np.testing.assert_allclose(pV[b:b + 1, :, :L], tV, rtol=0, atol=1e-12)
        pQsum += tQ
    np.testing.assert_allclose(dQ, dQsum, rtol=0, atol=1e-12)
    np.testing.assert_allclose(pQ, pQsum, rtol=0, atol=1e-12)


def test_varlen_sdpa_key_mask_crosscheck():
    # torch float64 SDPA with a boolean key-padding mask for the encode, the
    # decode's SDPA per token, padded outputs multiplied by zero; autograd of
    # that composition for the gradient.
    B, H, N, M, D = 3, 2, 40, 8, 4
    lens = [40, 13, 1]
    x = _x(B, H, N, M, D, seed=32, with_dy=True)
    s = 0.45
    Y, Z, _ = oracle.flare_fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)
    dQ, dK, dV = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens)
    t = {k: torch.from_numpy(v.copy()).requires_grad_(k != "dY") for k, v in x.items()}
    keep = torch.arange(N)[None, :] < torch.tensor(lens)[:, None]          # [B, N]
    Qb = t["Q"].unsqueeze(0).expand(B, -1, -1, -1)
    Zt = F.scaled_dot_product_attention(Qb, t["K"], t["V"], attn_mask=keep[:, None, None, :],
                                        scale=s)
    Yt = F.scaled_dot_product_attention(t["K"], Qb, Zt, scale=s) * keep[:, None, :, None]
    np.testing.assert_allclose(Y, Yt.detach().numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(Z, Zt.detach().numpy(), rtol=1e-11, atol=1e-13)
    (Yt * t["dY"]).sum().backward()
    np.testing.assert_allclose(dQ, t["Q"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, t["K"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, t["V"].grad.numpy(), rtol=1e-10, atol=1e-12)


def test_varlen_padding_is_never_read():
    # NaN in every padded K, V, dY element changes nothing.
    B, H, N, M, D = 2, 2, 25, 8, 4
    lens = [9, 25]
    x = _x(B, H, N, M, D, seed=33, with_dy=True)
    y = {k: v.copy() for k, v in x.items()}
    for k in ("K", "V", "dY"):
        y[k][0, :, 9:] = np.nan
    s = 0.5
    for f in (oracle.flare_fwd, oracle.flare_pp_fwd):
        for a, b in zip(f(x["Q"], x["K"], x["V"], s, seq_lens=lens),
                        f(y["Q"], y["K"], y["V"], s, seq_lens=lens)):
            np.testing.assert_array_equal(a, b)
    for f in (oracle.flare_bwd, oracle.flare_pp_bwd):
        for a, b in zip(f(x["Q"], x["K"], x["V"], x["dY"], s, seq_lens=lens),
                        f(y["Q"], y["K"], y["V"], y["dY"], s, seq_lens=lens)):
            np.testing.assert_array_equal(a, b)


def test_varlen_gradient_central_finite_differences():
    B, H, N, M, D = 2, 1, 12, 3, 4
    lens = [5, 12]
    x = _x(B, H, N, M, D, seed=34, with_dy=True)
    s = 0.8
    for fwd, bwd in ((oracle.flare_fwd, oracle.flare_bwd),
                     (oracle.flare_pp_fwd, oracle.flare_pp_bwd)):
        grads = dict(zip(("Q", "K", "V"), bwd(x["Q"], x["K"], x["V"], x["dY"], s,
                                              seq_lens=lens)))

        def loss():
            return float((fwd(x["Q"], x["K"], x["V"], s, seq_lens=lens)[0] * x["dY"]).sum())

        eps = 1e-5
        for name in ("Q", "K", "V"):
            flat = x[name].reshape(-1)
            fd = np.empty(flat.size)
            for i in range(flat.size):
                old = flat[i]
                flat[i] = old + eps
                lp = loss()
                flat[i] = old - eps
                lm = loss()
                flat[i] = old
                fd[i] = (lp - lm) / (2 * eps)
            g = grads[name].reshape(-1)
            assert np.abs(g - fd).max() <= 1e-7 * max(np.abs(fd).max(), 1.0), name
