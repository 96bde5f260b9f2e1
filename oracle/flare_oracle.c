/*
 * FLARE oracle: a plain, slow, double-precision CPU implementation of the
 * FLARE / FLARE++ token-mixing operator and of its gradient.
 *
 * THIS FILE IS TEST INFRASTRUCTURE.  Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header,
 * table or helper with the CUDA library; the two meet only through seeded
 * input buffers produced by a separate generator module.
 *
 * Sources (web pages about the method):
 *   [P1] "Flare Fast Low Rank Attention" skill page (skillmd.com),
 *        section 2 "Implement Encode Stage" and section 4 "Combine
 *        Encode-Decode into Attention Layer" (encode: latents are the queries,
 *        softmax over the sequence, weighted sum of the values, both logits
 *        divided by sqrt(head_dim)).
 *   [P4] "FLARE: Fast Low-rank Attention Routing Engine", arXiv 2508.12594
 *        abstract (mlsanity.com): each layer induces an input-input mixing
 *        matrix of rank at most M built from two standard SDPA calls and
 *        head-specific latent slices.
 *   [P5] "FLARE++: Low-rank attention with dynamic attention routing",
 *        arXiv 2608.11519 abstract (aiqbench.com): FLARE's own encoder maps
 *        the N tokens to M queries that correct the learned queries; the
 *        corrected queries then drive both compression and redistribution.
 *
 * Readings taken where the pages are silent or disagree (each is argued in
 * the design notes of the repository):
 *   - decode is Y = softmax_M(s K Q^T) Z: the tokens' keys query the latents,
 *     which is the only form giving an input-input mixing matrix
 *     W = softmax(s K Q^T) softmax(s Q K^T) of rank <= M [P4];
 *   - one caller-given scale s is used in every softmax (the pages divide by
 *     sqrt(head_dim) everywhere [P1]);
 *   - FLARE++: Q_dyn = Q + encode(Q, K, V) (plain sum, per batch), then
 *     Z = encode(Q_dyn, K, V) and Y = decode(Q_dyn, Z) [P5];
 *   - the pages give no backward pass; the gradient below is the chain rule
 *     of the two softmax-attention stages applied to L = sum(Y * dY);
 *   - FLARE++ gradient: the same chain rule through Q_dyn = Q + encode(Q, K,
 *     V), with Q shared over the batch (its gradient summed over b).
 *
 * Layouts: Q is [H,M,D] when q_bstride == 0 (shared over the batch) or
 * [B,H,M,D] when q_bstride == H*M*D; K, V, Y, dY are [B,H,N,D]; Z is
 * [B,H,M,D]; lse is [B,H,M].  All arrays are contiguous, row-major double.
 *
 * Sequence lengths (key-padding mask; the skill page's module accepts an
 * attention mask): lens, when not NULL, gives each batch element's number of
 * valid tokens L_b (clamped to [0, N]); tokens n >= L_b are padding.  The
 * encode's softmax runs over n < L_b only, the decode produces Y[n] for
 * n < L_b and Y[n] = 0 for padding, and padding gets zero dK and dV and
 * contributes nothing to any other gradient.  A sequence with no tokens
 * encodes to Z = 0 (an empty weighted sum) with lse = -inf.
 *
 * Parity status: every function here is pinned by CPU tests (brute-force
 * mixing matrix, closed forms, hard-max limit, permutation equivariance,
 * float64 SDPA cross-check, central finite differences for the gradient,
 * hand-derived golden values).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double dotd(const double* a, const double* b, int64_t D) {
  double s = 0.0;
  for (int64_t d = 0; d < D; ++d) s += a[d] * b[d];
  return s;
}

static int64_t seq_len(const int32_t* lens, int64_t b, int64_t N) {
  if (!lens) return N;
  int64_t L = lens[b];
  return L < 0 ? 0 : (L > N ? N : L);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Encode [P1 s2, s4; P4]: for every (b, h, m)
 *   l_n   = s * Q[m] . K[n]                     (n = 0..N-1)
 *   mu    = max_n l_n
 *   Z[m]  = sum_n exp(l_n - mu) V[n] / sum_n exp(l_n - mu)
 *   lse[m]= mu + log(sum_n exp(l_n - mu))      (natural log)
 * lse may be NULL.
 */
void oracle_encode(const double* Q, int64_t q_bstride, const double* K,
                   const double* V, const int32_t* lens, int64_t B, int64_t H,
                   int64_t N, int64_t M, int64_t D, double scale, double* Z,
                   double* lse) {
#pragma omp parallel for collapse(3) schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < H; ++h)
      for (int64_t m = 0; m < M; ++m) {
        const int64_t Nb = seq_len(lens, b, N);
        const double* q = Q + b * q_bstride + (h * M + m) * D;
        const double* Kb = K + (b * H + h) * N * D;
        const double* Vb = V + (b * H + h) * N * D;
        double* z = Z + ((b * H + h) * M + m) * D;
        if (Nb == 0) {   /* no tokens: an empty weighted sum */
          for (int64_t d = 0; d < D; ++d) z[d] = 0.0;
          if (lse) lse[(b * H + h) * M + m] = -INFINITY;
          continue;
        }
        double mu = -INFINITY;
        for (int64_t n = 0; n < Nb; ++n) {
          double l = scale * dotd(q, Kb + n * D, D);
          if (l > mu) mu = l;
        }
        double* acc = (double*)calloc((size_t)D, sizeof(double));
        double den = 0.0;
        for (int64_t n = 0; n < Nb; ++n) {
          double w = exp(scale * dotd(q, Kb + n * D, D) - mu);
          den += w;
          for (int64_t d = 0; d < D; ++d) acc[d] += w * Vb[n * D + d];
        }
        for (int64_t d = 0; d < D; ++d) z[d] = acc[d] / den;
        if (lse) lse[(b * H + h) * M + m] = mu + log(den);
        free(acc);
      }
}

/* Decode of one token row: a_m = s * K[n] . Q[m]; p = softmax_M(a); y = p Z. */
static void decode_row(const double* q_bh, const double* k, const double* z_bh,
                       int64_t M, int64_t D, double scale, double* y) {
  double mu = -INFINITY;
  for (int64_t m = 0; m < M; ++m) {
    double a = scale * dotd(k, q_bh + m * D, D);
    if (a > mu) mu = a;
  }
  double den = 0.0;
  for (int64_t d = 0; d < D; ++d) y[d] = 0.0;
  for (int64_t m = 0; m < M; ++m) {
    double w = exp(scale * dotd(k, q_bh + m * D, D) - mu);
    den += w;
    for (int64_t d = 0; d < D; ++d) y[d] += w * z_bh[m * D + d];
  }
  for (int64_t d = 0; d < D; ++d) y[d] /= den;
}

/* Decode [P4]: Y[b,h,n] = softmax_M(s K[b,h,n] Q[h]^T) Z[b,h]. */
void oracle_decode(const double* Q, int64_t q_bstride, const double* K,
                   const double* Z, const int32_t* lens, int64_t B, int64_t H,
                   int64_t N, int64_t M, int64_t D, double scale, double* Y) {
#pragma omp parallel for collapse(3) schedule(static)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < H; ++h)
      for (int64_t n = 0; n < N; ++n) {
        const double* q_bh = Q + b * q_bstride + h * M * D;
        const double* z_bh = Z + (b * H + h) * M * D;
        const double* k = K + ((b * H + h) * N + n) * D;
        double* y = Y + ((b * H + h) * N + n) * D;
        if (n >= seq_len(lens, b, N)) {   /* padding */
          for (int64_t d = 0; d < D; ++d) y[d] = 0.0;
          continue;
        }
        decode_row(q_bh, k, z_bh, M, D, scale, y);
      }
}

/*
 * Decode of selected token rows only.  rows[i] is the flat index
 * (b*H + h)*N + n of a token; Yrows is [nrows, D].
 */
void oracle_decode_rows(const double* Q, int64_t q_bstride, const double* K,
                        const double* Z, int64_t B, int64_t H, int64_t N,
                        int64_t M, int64_t D, double scale,
                        const int64_t* rows, int64_t nrows, double* Yrows) {
  (void)B;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t r = rows[i];
    int64_t bh = r / N;
    int64_t b = bh / H, h = bh % H;
    const double* q_bh = Q + b * q_bstride + h * M * D;
    const double* z_bh = Z + bh * M * D;
    decode_row(q_bh, K + r * D, z_bh, M, D, scale, Yrows + i * D);
  }
}

/* FLARE forward [P1 s4, P4]: Z = encode(Q,K,V); Y = decode(Q,K,Z). */
void oracle_flare_fwd(const double* Q, int64_t q_bstride, const double* K,
                      const double* V, const int32_t* lens, int64_t B,
                      int64_t H, int64_t N, int64_t M, int64_t D, double scale,
                      double* Y, double* Z, double* lse) {
  oracle_encode(Q, q_bstride, K, V, lens, B, H, N, M, D, scale, Z, lse);
  oracle_decode(Q, q_bstride, K, Z, lens, B, H, N, M, D, scale, Y);
}

/*
 * FLARE++ forward [P5]: learned Q [H,M,D] shared over the batch.
 *   Z1    = encode(Q, K, V)                 [B,H,M,D]
 *   Q_dyn = Q + Z1                          [B,H,M,D]
 *   Z     = encode(Q_dyn, K, V), lse
 *   Y     = decode(Q_dyn, K, Z)
 * Qdyn, Z and lse are outputs (lse may be NULL).
 */
void oracle_flare_pp_fwd(const double* Q, const double* K, const double* V,
                         const int32_t* lens, int64_t B, int64_t H, int64_t N,
                         int64_t M, int64_t D, double scale, double* Y,
                         double* Qdyn, double* Z, double* lse) {
  int64_t per_b = H * M * D;
  double* Z1 = (double*)malloc((size_t)(B * per_b) * sizeof(double));
  oracle_encode(Q, 0, K, V, lens, B, H, N, M, D, scale, Z1, NULL);
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = 0; i < per_b; ++i) Qdyn[b * per_b + i] = Q[i] + Z1[b * per_b + i];
  free(Z1);
  oracle_encode(Qdyn, per_b, K, V, lens, B, H, N, M, D, scale, Z, lse);
  oracle_decode(Qdyn, per_b, K, Z, lens, B, H, N, M, D, scale, Y);
}

/*
 * Gradient of L = sum(Y * dY) for FLARE (fixed Q), chain rule through both
 * softmax-attention stages.  For one (b, h) with s = scale:
 *   encode: A_e = s Q K^T [M,N], P_e = softmax over n, Z = P_e V
 *   decode: A_d = s K Q^T [N,M], P_d = softmax over m, Y = P_d Z
 *   dZ   = P_d^T dY                       dP_d = dY Z^T
 *   dA_d = P_d * (dP_d - rowsum(P_d * dP_d))
 *   dK   = s dA_d Q   (+ encode part)     dQ  = s dA_d^T K (+ encode part)
 *   dV   = P_e^T dZ                       dP_e = dZ V^T
 *   dA_e = P_e * (dP_e - rowsum(P_e * dP_e))
 *   dQ  += s dA_e K                       dK += s dA_e^T Q
 * dQ is [H,M,D] summed over b when q_bstride == 0, else [B,H,M,D].
 */
void oracle_flare_bwd(const double* Q, int64_t q_bstride, const double* K,
                      const double* V, const double* dY, const int32_t* lens,
                      int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                      double scale, double* dQ, double* dK, double* dV) {
  int64_t BH = B * H;
  double* dQbh = (double*)calloc((size_t)(BH * M * D), sizeof(double));
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    int64_t b = bh / H, h = bh % H;
    const int64_t Nb = seq_len(lens, b, N);   /* tokens n >= Nb are padding */
    const double* q = Q + b * q_bstride + h * M * D;
    const double* k = K + bh * N * D;
    const double* v = V + bh * N * D;
    const double* dy = dY + bh * N * D;
    double* dk = dK + bh * N * D;
    double* dv = dV + bh * N * D;
    double* dq = dQbh + bh * M * D;
    double* Pe = (double*)malloc((size_t)(M * N) * sizeof(double));
    double* Pd = (double*)malloc((size_t)(N * M) * sizeof(double));
    double* Z = (double*)calloc((size_t)(M * D), sizeof(double));
    double* dZ = (double*)calloc((size_t)(M * D), sizeof(double));
    /* forward recompute: P_e rows (softmax over n) and Z */
    for (int64_t m = 0; m < M; ++m) {
      double mu = -INFINITY;
      for (int64_t n = 0; n < Nb; ++n) {
        double a = scale * dotd(q + m * D, k + n * D, D);
        Pe[m * N + n] = a;
        if (a > mu) mu = a;
      }
      double den = 0.0;
      for (int64_t n = 0; n < Nb; ++n) {
        Pe[m * N + n] = exp(Pe[m * N + n] - mu);
        den += Pe[m * N + n];
      }
      for (int64_t n = 0; n < Nb; ++n) {
        Pe[m * N + n] /= den;
        for (int64_t d = 0; d < D; ++d) Z[m * D + d] += Pe[m * N + n] * v[n * D + d];
      }
    }
    /* forward recompute: P_d rows (softmax over m) */
    for (int64_t n = 0; n < Nb; ++n) {
      double mu = -INFINITY;
      for (int64_t m = 0; m < M; ++m) {
        double a = scale * dotd(k + n * D, q + m * D, D);
        Pd[n * M + m] = a;
        if (a > mu) mu = a;
      }
      double den = 0.0;
      for (int64_t m = 0; m < M; ++m) {
        Pd[n * M + m] = exp(Pd[n * M + m] - mu);
        den += Pd[n * M + m];
      }
      for (int64_t m = 0; m < M; ++m) Pd[n * M + m] /= den;
    }
    /* decode stage */
    for (int64_t n = 0; n < Nb; ++n) {
      double delta = 0.0;
      for (int64_t m = 0; m < M; ++m)
        delta += Pd[n * M + m] * dotd(dy + n * D, Z + m * D, D);
      for (int64_t d = 0; d < D; ++d) dk[d + n * D] = 0.0;
      for (int64_t m = 0; m < M; ++m) {
        double p = Pd[n * M + m];
        double dA = p * (dotd(dy + n * D, Z + m * D, D) - delta);
        for (int64_t d = 0; d < D; ++d) {
          dk[n * D + d] += scale * dA * q[m * D + d];
          dq[m * D + d] += scale * dA * k[n * D + d];
          dZ[m * D + d] += p * dy[n * D + d];
        }
      }
    }
    /* encode stage */
    for (int64_t n = 0; n < Nb; ++n) {
      for (int64_t d = 0; d < D; ++d) dv[n * D + d] = 0.0;
      for (int64_t m = 0; m < M; ++m)
        for (int64_t d = 0; d < D; ++d) dv[n * D + d] += Pe[m * N + n] * dZ[m * D + d];
    }
    for (int64_t m = 0; m < M; ++m) {
      double delta = 0.0;
      for (int64_t n = 0; n < Nb; ++n)
        delta += Pe[m * N + n] * dotd(dZ + m * D, v + n * D, D);
      for (int64_t n = 0; n < Nb; ++n) {
        double dA = Pe[m * N + n] * (dotd(dZ + m * D, v + n * D, D) - delta);
        for (int64_t d = 0; d < D; ++d) {
          dq[m * D + d] += scale * dA * k[n * D + d];
          dk[n * D + d] += scale * dA * q[m * D + d];
        }
      }
    }
    for (int64_t n = Nb; n < N; ++n)   /* padding: zero gradient */
      for (int64_t d = 0; d < D; ++d) dk[n * D + d] = dv[n * D + d] = 0.0;
    free(Pe);
    free(Pd);
    free(Z);
    free(dZ);
  }
  /* dQ: per-batch copy, or a sum over b in fixed order when Q is shared */
  if (q_bstride == 0) {
    memset(dQ, 0, (size_t)(H * M * D) * sizeof(double));
    for (int64_t b = 0; b < B; ++b)
      for (int64_t i = 0; i < H * M * D; ++i) dQ[i] += dQbh[b * H * M * D + i];
  } else {
    memcpy(dQ, dQbh, (size_t)(BH * M * D) * sizeof(double));
  }
  free(dQbh);
}

/*
 * Adds the gradient of L = sum(Z1 * dZ1) for the encode Z1 = softmax_n(s Q K^T) V
 * with Q [H,M,D] shared over the batch: for one (b, h),
 *   P = softmax over n of s Q K^T [M,N],   dP = dZ1 V^T,
 *   dA = P * (dP - rowsum(P * dP)),
 *   dV += P^T dZ1,   dK += s dA^T Q,   dQ += s dA K (summed over b).
 */
static void encode_bwd_add(const double* Q, const double* K, const double* V,
                           const double* dZ1, const int32_t* lens, int64_t B,
                           int64_t H, int64_t N, int64_t M, int64_t D,
                           double scale, double* dQ, double* dK, double* dV) {
  int64_t BH = B * H;
  double* dQbh = (double*)calloc((size_t)(BH * M * D), sizeof(double));
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    int64_t h = bh % H;
    const int64_t Nb = seq_len(lens, bh / H, N);   /* tokens n >= Nb are padding */
    const double* q = Q + h * M * D;
    const double* k = K + bh * N * D;
    const double* v = V + bh * N * D;
    const double* dz = dZ1 + bh * M * D;
    double* dk = dK + bh * N * D;
    double* dv = dV + bh * N * D;
    double* dq = dQbh + bh * M * D;
    double* P = (double*)malloc((size_t)N * sizeof(double));
    for (int64_t m = 0; m < M; ++m) {
      double mu = -INFINITY;
      for (int64_t n = 0; n < Nb; ++n) {
        P[n] = scale * dotd(q + m * D, k + n * D, D);
        if (P[n] > mu) mu = P[n];
      }
      double den = 0.0;
      for (int64_t n = 0; n < Nb; ++n) {
        P[n] = exp(P[n] - mu);
        den += P[n];
      }
      double delta = 0.0;
      for (int64_t n = 0; n < Nb; ++n) {
        P[n] /= den;
        delta += P[n] * dotd(dz + m * D, v + n * D, D);
      }
      for (int64_t n = 0; n < Nb; ++n) {
        double dA = P[n] * (dotd(dz + m * D, v + n * D, D) - delta);
        for (int64_t d = 0; d < D; ++d) {
          dv[n * D + d] += P[n] * dz[m * D + d];
          dk[n * D + d] += scale * dA * q[m * D + d];
          dq[m * D + d] += scale * dA * k[n * D + d];
        }
      }
    }
    free(P);
  }
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = 0; i < H * M * D; ++i) dQ[i] += dQbh[b * H * M * D + i];
  free(dQbh);
}

/* The encode's gradient alone (outputs overwritten): dQ [H,M,D] summed over
 * the batch, dK, dV [B,H,N,D]. */
void oracle_encode_bwd(const double* Q, const double* K, const double* V,
                       const double* dZ1, const int32_t* lens, int64_t B,
                       int64_t H, int64_t N, int64_t M, int64_t D,
                       double scale, double* dQ, double* dK, double* dV) {
  memset(dQ, 0, (size_t)(H * M * D) * sizeof(double));
  memset(dK, 0, (size_t)(B * H * N * D) * sizeof(double));
  memset(dV, 0, (size_t)(B * H * N * D) * sizeof(double));
  encode_bwd_add(Q, K, V, dZ1, lens, B, H, N, M, D, scale, dQ, dK, dV);
}

/*
 * Gradient of L = sum(Y * dY) for FLARE++ with learned Q [H,M,D]:
 *   Q_dyn = Q + Z1, Z1 = encode(Q, K, V)      (per batch)
 *   Y = FLARE(Q_dyn, K, V)                     (per-batch latents)
 * FLARE's gradient with per-batch latents gives dQ_dyn, dK, dV; Q_dyn's
 * gradient then reaches Q directly (summed over b) and through Z1 (the
 * encode's gradient with upstream dZ1 = dQ_dyn), which also adds to dK, dV.
 */
void oracle_flare_pp_bwd(const double* Q, const double* K, const double* V,
                         const double* dY, const int32_t* lens, int64_t B,
                         int64_t H, int64_t N, int64_t M, int64_t D,
                         double scale, double* dQ, double* dK, double* dV) {
  int64_t per_b = H * M * D;
  double* Z1 = (double*)malloc((size_t)(B * per_b) * sizeof(double));
  double* Qdyn = (double*)malloc((size_t)(B * per_b) * sizeof(double));
  double* dQd = (double*)malloc((size_t)(B * per_b) * sizeof(double));
  oracle_encode(Q, 0, K, V, lens, B, H, N, M, D, scale, Z1, NULL);
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = 0; i < per_b; ++i) Qdyn[b * per_b + i] = Q[i] + Z1[b * per_b + i];
  oracle_flare_bwd(Qdyn, per_b, K, V, dY, lens, B, H, N, M, D, scale, dQd, dK, dV);
  memset(dQ, 0, (size_t)per_b * sizeof(double));
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = 0; i < per_b; ++i) dQ[i] += dQd[b * per_b + i];
  encode_bwd_add(Q, K, V, dQd, lens, B, H, N, M, D, scale, dQ, dK, dV);
  free(Z1);
  free(Qdyn);
  free(dQd);
}
