"""The factorisation the tensor-core backward computes, checked in float64 on
the CPU against the oracle's gradient (CPU only).

The kernels do not evaluate the chain rule term by term.  Per (b, h), with
c = scale * log2(e), S = K Q^T and all exponentials in base 2:

* decode statistics per token: its log-sum-exp mx'[n] = log2 sum_m
  2^(c S[n,m]), Y[n], delta_d[n] = dY[n] . Y[n];
* dZ[m] = sum_n P_d[n,m] dY[n] with the fixed weights P_d = 2^(c S - mx');
* with R = max_m lse2[m] (the forward's encode lse in log2 units),
  g[n] = 2^(mx'[n] - R), f[m] = 2^(R - lse2[m]), dY'' = dY / g,
  dZ'' = f dZ, delta'' = dY'' . Y, and e = 2^(c S - R) (the one
  exponential per pair):
    G  = e (dY''[n] . Z[m] + V[n] . dZ''[m] - dZ''[m] . Z[m] - delta''[n])
    dK = s G Q,  dV = e dZ'',  dQ = s G^T K;
* with M = 256 the last three run once per half of the latents, adding.

These tests rebuild the gradient from exactly those pieces (latents split
in two halves, as the M = 256 path does) and require the oracle's result,
so a wrong sign, a dropped term or a mixed-up reference in the
factorisation fails here without a GPU.  The exact form (f = 1, P_e
computed directly) is checked the same way.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from flare_inputs import make_inputs

LOG2E = 1.0 / math.log(2.0)


def _inputs(B, H, N, M, D, seed, per_batch_q):
    x = make_inputs(B, H, N, M, D, dtype=torch.float64, seed=seed, per_batch_q=per_batch_q,
                    with_dy=True)
    return {k: v.numpy() for k, v in x.items()}


def _factored_bwd(Q, K, V, dY, s, halves=2, exact=False):
    B, H, N, D = K.shape
    M = Q.shape[-2]
    Qb = Q if Q.ndim == 4 else np.broadcast_to(Q, (B,) + Q.shape)
    c = s * LOG2E
    dQ = np.zeros((B, H, M, D))
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for b in range(B):
        for h in range(H):
            q, k, v, dy = Qb[b, h], K[b, h], V[b, h], dY[b, h]
            S = k @ q.T                                        # [N, M]
            # the forward's encode: lse2 and Z
            lse2 = np.log2(np.exp2(c * S - (c * S).max(0)).sum(0)) + (c * S).max(0)
            Pe = np.exp2(c * S - lse2)                         # softmax over n
            Z = Pe.T @ v
            # statistics pass
            mxp = np.log2(np.exp2(c * S - (c * S).max(1, keepdims=True)).sum(1)) \
                + (c * S).max(1)
            Pd = np.exp2(c * S - mxp[:, None])                 # softmax over m
            Y = Pd @ Z
            # dZ pass (fixed per-token weights)
            dZ = Pd.T @ dy
            # between the passes
            R = lse2.max()
            f = np.ones(M) if exact else np.exp2(R - lse2)
            g = np.exp2(mxp - R)
            dY2 = dy / g[:, None]
            dZ2 = f[:, None] * dZ
            dpp = (dY2 * Y).sum(1)                             # delta'' = delta_d / g
            for lat in np.array_split(np.arange(M), halves):   # pass B per latent half
                e = np.exp2(c * S[:, lat] - R)
                if exact:
                    # both weights with their own exponentials
                    Pd_h, Pe_h = Pd[:, lat], np.exp2(c * S[:, lat] - lse2[lat])
                    dd = (dy * Y).sum(1)
                    de = (dZ[lat] * Z[lat]).sum(1)
                    G = Pd_h * (dy @ Z[lat].T - dd[:, None]) + Pe_h * (v @ dZ[lat].T - de)
                    dV[b, h] += Pe_h @ dZ[lat]
                else:
                    U = dY2 @ Z[lat].T + v @ dZ2[lat].T - (dZ2[lat] * Z[lat]).sum(1) \
                        - dpp[:, None]
                    G = e * U
                    dV[b, h] += e @ dZ2[lat]
                dK[b, h] += s * G @ q[lat]
                dQ[b, h, lat] += s * G.T @ k
    if Q.ndim == 3:
        dQ = dQ.sum(0)
    return dQ, dK, dV


@pytest.mark.parametrize("exact", [False, True], ids=["one_exponential", "exact"])
@pytest.mark.parametrize("per_batch_q", [False, True], ids=["sharedQ", "batchQ"])
@pytest.mark.parametrize("halves", [1, 2])
def test_factored_gradient_equals_oracle(halves, per_batch_q, exact):
    B, H, N, M, D = 2, 2, 37, 8, 4
    s = 1.0 / math.sqrt(D)
    x = _inputs(B, H, N, M, D, seed=61, per_batch_q=per_batch_q)
    got = _factored_bwd(x["Q"], x["K"], x["V"], x["dY"], s, halves=halves, exact=exact)
    ref = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    for a, r, name in zip(got, ref, ("dQ", "dK", "dV")):
        np.testing.assert_allclose(a, r, rtol=1e-9, atol=1e-12, err_msg=name)


def test_factored_gradient_sharp_softmax():
    # scale x4: lse spread over several tens (log2 units); the split
    # e = P_d g = P_e / f stays exact in float64
    B, H, N, M, D = 1, 2, 29, 6, 4
    s = 4.0 / math.sqrt(D)
    x = _inputs(B, H, N, M, D, seed=62, per_batch_q=False)
    got = _factored_bwd(x["Q"], x["K"], x["V"], x["dY"], s, halves=2)
    ref = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    for a, r, name in zip(got, ref, ("dQ", "dK", "dV")):
        np.testing.assert_allclose(a, r, rtol=1e-8, atol=1e-10, err_msg=name)


def test_dropping_a_term_is_detected():
    # the check has teeth: without the -dZ''.Z term of U the result moves
    B, H, N, M, D = 1, 1, 21, 4, 4
    s = 0.5
    x = _inputs(B, H, N, M, D, seed=63, per_batch_q=False)
    ref = oracle.flare_bwd(x["Q"], x["K"], x["V"], x["dY"], s)
    Q, K, V, dY = x["Q"], x["K"], x["V"], x["dY"]
    c = s * LOG2E
    q, k, v, dy = Q[0], K[0, 0], V[0, 0], dY[0, 0]
    S = k @ q.T
    lse2 = np.log2(np.exp2(c * S).sum(0))
    Z = np.exp2(c * S - lse2).T @ v
    mxp = np.log2(np.exp2(c * S).sum(1))
    Pd = np.exp2(c * S - mxp[:, None])
    Y = Pd @ Z
    dZ = Pd.T @ dy
    R = lse2.max()
    f, g = np.exp2(R - lse2), np.exp2(mxp - R)
    dY2, dZ2 = dy / g[:, None], f[:, None] * dZ
    U_wrong = dY2 @ Z.T + v @ dZ2.T - ((dY2 * Y).sum(1))[:, None]
    dK_wrong = s * (np.exp2(c * S - R) * U_wrong) @ q
    assert np.abs(dK_wrong - ref[1][0, 0]).max() > 1e-3
