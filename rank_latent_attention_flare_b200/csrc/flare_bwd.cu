// FLARE backward on CUDA cores: gradients of sum(Y * dY) with respect to Q,
// K and V, logits recomputed from Q, K and the forward's Z and lse.
//
// The pages give no backward; this is the chain rule through the two
// softmax-attention stages (encode: skill page section 2; decode: FLARE arXiv
// abstract).  Per (b, h), with s = scale:
//   decode stage (pass A, over tokens):
//     P_d = softmax_m(s K Q^T), dP_d = dY Z^T, delta_d = rowsum(P_d * dP_d),
//     dA_d = P_d * (dP_d - delta_d), dK = s dA_d Q, dQ += s dA_d^T K,
//     dZ = P_d^T dY
//   encode stage (pass B, over tokens):
//     P_e = exp(s Q K^T - lse), delta_e = rowsum(dZ * Z), dP_e = dZ V^T,
//     dA_e = P_e * (dP_e - delta_e), dV = P_e^T dZ, dK += s dA_e^T Q,
//     dQ += s dA_e K
// Every cross-token sum goes through per-chunk partial records that are then
// added in a fixed order, so the results are bitwise reproducible.
#include "flare_plan.cuh"

namespace flare {
namespace {

constexpr int kT = kBwdTile;  // tokens per tile (= threads per CTA)

template <typename T, int D>
__global__ void __launch_bounds__(kT)
    bwd_decode_kernel(const T* __restrict__ Q, int64_t q_bstride, const T* __restrict__ K,
                      const T* __restrict__ dY, Tok tk, Tok tdy, const int32_t* __restrict__ lens,
                      const float* __restrict__ Z, int H, int64_t N, int M, float c, float s,
                      int64_t chunk_tokens, float* __restrict__ dkf,
                      float* __restrict__ dq_part, float* __restrict__ dz_part) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [M][D] raw latents
  float* zs = qs + M * D;         // [M][D]
  float* ks = zs + M * D;         // [kT][D]
  float* dys = ks + kT * D;       // [kT][D]
  float* tmax = dys + kT * D;     // [kT] row max of the decode logits (log2 units)
  float* tinv = tmax + kT;        // [kT] 1 / softmax denominator
  float* tdel = tinv + kT;        // [kT] delta_d
  const int chunk = blockIdx.x, chunks = gridDim.x;
  const int64_t bh = blockIdx.y, b = bh / H, h = bh % H;
  const int64_t n0 = (int64_t)chunk * chunk_tokens;
  const int64_t n1 = min(seq_len(lens, bh / H, N), n0 + chunk_tokens);   // padding: none
  const int64_t kh = tk.head(bh, H), dyh = tdy.head(bh, H);
  for (int i = threadIdx.x; i < M * D; i += blockDim.x) {
    qs[i] = to_f(Q[b * q_bstride + h * (int64_t)M * D + i]);
    zs[i] = Z[bh * M * D + i];
  }
  const int tid = threadIdx.x;
  const bool active_m = tid < M;
  float dq[D], dz[D];
#pragma unroll
  for (int d = 0; d < D; ++d) dq[d] = dz[d] = 0.f;

  for (int64_t t0 = n0; t0 < n1; t0 += kT) {
    const int nt = (int)imin64(kT, n1 - t0);
    __syncthreads();
    for (int i = tid; i < kT * D; i += blockDim.x) {
      const int j = i / D, d = i % D;
      ks[i] = (j < nt) ? to_f(K[kh + (t0 + j) * tk.sn + d]) : 0.f;
      dys[i] = (j < nt) ? to_f(dY[dyh + (t0 + j) * tdy.sn + d]) : 0.f;
    }
    __syncthreads();
    // phase 1: one thread per token -> softmax statistics, delta_d and dK
    if (tid < nt) {
      float k[D], dy[D];
#pragma unroll
      for (int d = 0; d < D; ++d) {
        k[d] = ks[tid * D + d];
        dy[d] = dys[tid * D + d];
      }
      float mx = -INFINITY;
      for (int m = 0; m < M; ++m) {
        float a = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) a = fmaf(k[d], qs[m * D + d], a);
        mx = fmaxf(mx, a * c);
      }
      float sum = 0.f, dn = 0.f;
      for (int m = 0; m < M; ++m) {
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          a = fmaf(k[d], qs[m * D + d], a);
          dp = fmaf(dy[d], zs[m * D + d], dp);
        }
        const float p = exp2f(a * c - mx);
        sum += p;
        dn = fmaf(p, dp, dn);
      }
      const float inv = 1.f / sum;
      const float delta = dn * inv;
      float dk[D];
#pragma unroll
      for (int d = 0; d < D; ++d) dk[d] = 0.f;
      for (int m = 0; m < M; ++m) {
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          a = fmaf(k[d], qs[m * D + d], a);
          dp = fmaf(dy[d], zs[m * D + d], dp);
        }
        const float p = exp2f(a * c - mx) * inv;
        const float dA = s * p * (dp - delta);
#pragma unroll
        for (int d = 0; d < D; ++d) dk[d] = fmaf(dA, qs[m * D + d], dk[d]);
      }
      float* o = dkf + (bh * N + t0 + tid) * D;
#pragma unroll
      for (int d = 0; d < D; ++d) o[d] = dk[d];
      tmax[tid] = mx;
      tinv[tid] = inv;
      tdel[tid] = delta;
    }
    __syncthreads();
    // phase 2: one thread per latent -> partial dQ (decode part) and dZ
    if (active_m) {
      float q[D], z[D];
#pragma unroll
      for (int d = 0; d < D; ++d) {
        q[d] = qs[tid * D + d];
        z[d] = zs[tid * D + d];
      }
      for (int j = 0; j < nt; ++j) {
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          a = fmaf(ks[j * D + d], q[d], a);
          dp = fmaf(dys[j * D + d], z[d], dp);
        }
        const float p = exp2f(a * c - tmax[j]) * tinv[j];
        const float dA = s * p * (dp - tdel[j]);
#pragma unroll
        for (int d = 0; d < D; ++d) {
          dq[d] = fmaf(dA, ks[j * D + d], dq[d]);
          dz[d] = fmaf(p, dys[j * D + d], dz[d]);
        }
      }
    }
  }
  if (active_m) {
    const int64_t row = (bh * chunks + chunk) * M + tid;
#pragma unroll
    for (int d = 0; d < D; ++d) {
      dq_part[row * D + d] = dq[d];
      dz_part[row * D + d] = dz[d];
    }
  }
}

// dZ = sum over chunks of the partials (fixed order); delta_e = rowsum(dZ * Z).
__global__ void reduce_dz_kernel(const float* __restrict__ dz_part, const float* __restrict__ Z,
                                 int64_t BH, int M, int D, int chunks, float* __restrict__ dz,
                                 float* __restrict__ delta) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= BH * M) return;
  const int64_t bh = w / M, m = w % M;
  float acc = 0.f;
  if (lane < D)
    for (int c = 0; c < chunks; ++c) acc += dz_part[((bh * chunks + c) * M + m) * D + lane];
  float prod = (lane < D) ? acc * Z[w * D + lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) prod += __shfl_xor_sync(0xffffffffu, prod, o);
  if (lane < D) dz[w * D + lane] = acc;
  if (lane == 0) delta[w] = prod;
}

template <typename T, int D>
__global__ void __launch_bounds__(kT)
    bwd_encode_kernel(const T* __restrict__ Q, int64_t q_bstride, const T* __restrict__ K,
                      const T* __restrict__ V, const float* __restrict__ dkf,
                      const float* __restrict__ lse, const float* __restrict__ dzg,
                      const float* __restrict__ delta, Tok tk, Tok tv, Tok tdk, Tok tdv,
                      const int32_t* __restrict__ lens, int H, int64_t N, int M, float c, float s,
                      int64_t chunk_tokens,
                      T* __restrict__ dK, T* __restrict__ dV, float* __restrict__ dq_part) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [M][D]
  float* dzs = qs + M * D;        // [M][D]
  float* ls = dzs + M * D;        // [M] lse in log2 units
  float* des = ls + M;            // [M] delta_e
  float* ks = des + M;            // [kT][D]
  float* vs = ks + kT * D;        // [kT][D]
  const int chunk = blockIdx.x, chunks = gridDim.x;
  const int64_t bh = blockIdx.y, b = bh / H, h = bh % H;
  const int64_t n0 = (int64_t)chunk * chunk_tokens;
  const int64_t n1 = min(seq_len(lens, bh / H, N), n0 + chunk_tokens);   // padding: none
  const int64_t kh = tk.head(bh, H), vh = tv.head(bh, H);
  const int64_t dkh = tdk.head(bh, H), dvh = tdv.head(bh, H);
  for (int i = threadIdx.x; i < M * D; i += blockDim.x) {
    qs[i] = to_f(Q[b * q_bstride + h * (int64_t)M * D + i]);
    dzs[i] = dzg[bh * M * D + i];
  }
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    ls[i] = lse[bh * M + i] * kLog2e;
    des[i] = delta[bh * M + i];
  }
  const int tid = threadIdx.x;
  const bool active_m = tid < M;
  float dq[D];
#pragma unroll
  for (int d = 0; d < D; ++d) dq[d] = 0.f;

  for (int64_t t0 = n0; t0 < n1; t0 += kT) {
    const int nt = (int)imin64(kT, n1 - t0);
    __syncthreads();
    for (int i = tid; i < kT * D; i += blockDim.x) {
      const int j = i / D, d = i % D;
      ks[i] = (j < nt) ? to_f(K[kh + (t0 + j) * tk.sn + d]) : 0.f;
      vs[i] = (j < nt) ? to_f(V[vh + (t0 + j) * tv.sn + d]) : 0.f;
    }
    __syncthreads();
    // phase 1: one thread per token -> dV and the encode part of dK
    if (tid < nt) {
      const int64_t n = t0 + tid;
      float k[D], v[D], dk[D], dv[D];
#pragma unroll
      for (int d = 0; d < D; ++d) {
        k[d] = ks[tid * D + d];
        v[d] = vs[tid * D + d];
        dk[d] = dkf[(bh * N + n) * D + d];
        dv[d] = 0.f;
      }
      for (int m = 0; m < M; ++m) {
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          a = fmaf(k[d], qs[m * D + d], a);
          dp = fmaf(dzs[m * D + d], v[d], dp);
        }
        const float p = exp2f(a * c - ls[m]);
        const float dA = s * p * (dp - des[m]);
#pragma unroll
        for (int d = 0; d < D; ++d) {
          dv[d] = fmaf(p, dzs[m * D + d], dv[d]);
          dk[d] = fmaf(dA, qs[m * D + d], dk[d]);
        }
      }
#pragma unroll
      for (int d = 0; d < D; ++d) {
        dK[dkh + n * tdk.sn + d] = from_f<T>(dk[d]);
        dV[dvh + n * tdv.sn + d] = from_f<T>(dv[d]);
      }
    }
    // phase 2: one thread per latent -> partial dQ (encode part)
    if (active_m) {
      float q[D], dzr[D];
#pragma unroll
      for (int d = 0; d < D; ++d) {
        q[d] = qs[tid * D + d];
        dzr[d] = dzs[tid * D + d];
      }
      const float lm = ls[tid], dm = des[tid];
      for (int j = 0; j < nt; ++j) {
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          a = fmaf(ks[j * D + d], q[d], a);
          dp = fmaf(dzr[d], vs[j * D + d], dp);
        }
        const float p = exp2f(a * c - lm);
        const float dA = s * p * (dp - dm);
#pragma unroll
        for (int d = 0; d < D; ++d) dq[d] = fmaf(dA, ks[j * D + d], dq[d]);
      }
    }
  }
  if (active_m) {
    const int64_t row = (bh * chunks + chunk) * M + tid;
#pragma unroll
    for (int d = 0; d < D; ++d) dq_part[row * D + d] = dq[d];
  }
}

// dQ = sum over (batch when Q is shared) x chunks x {decode, encode}
// partials, in a fixed order.  One thread per output element.
template <typename T>
__global__ void reduce_dq_kernel(const float* __restrict__ dq_dec, const float* __restrict__ dq_enc,
                                 int B, int H, int M, int D, int chunks, bool shared_q,
                                 T* __restrict__ dQ) {
  const int64_t per = (int64_t)H * M * D;
  const int64_t total = shared_q ? per : (int64_t)B * per;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int64_t b0 = shared_q ? 0 : i / per;
  const int64_t b1 = shared_q ? B : b0 + 1;
  const int64_t r = i % per;             // (h, m, d)
  const int64_t h = r / ((int64_t)M * D);
  const int64_t md = r % ((int64_t)M * D);
  float acc = 0.f;
  for (int64_t b = b0; b < b1; ++b) {
    const int64_t bh = b * H + h;
    for (int c = 0; c < chunks; ++c) {
      const int64_t o = (bh * chunks + c) * (int64_t)M * D + md;
      acc += dq_dec[o];
      acc += dq_enc[o];
    }
  }
  dQ[i] = from_f<T>(acc);
}

template <typename T, int D>
cudaError_t bwd_t(const void* Q, int64_t qbs, const void* K, const void* V, const void* dY,
                  const float* Z, const float* lse, void* dQ, void* dK, void* dV, const Dims& d,
                  float scale, const WsLayout& L, char* ws, cudaStream_t st, BwdPhase phase,
                  float* dz_io, float* dq32) {
  const ChunkPlan& p = L.bwd;
  const int M = (int)d.M;
  const float c = scale * kLog2e;
  const int64_t bslots = d.BH() * p.chunks;
  float* dkf = (float*)(ws + L.dkf);
  float* dq_dec = (float*)(ws + L.dqp);
  float* dq_enc = dq_dec + bslots * M * D;
  float* dzp = (float*)(ws + L.dzp);
  float* dz = (float*)(ws + L.dz);
  float* delta = (float*)(ws + L.delta);
  dim3 grid(p.chunks, (unsigned)d.BH());
  cudaError_t e;
  const int64_t warps = d.BH() * M;

  if (phase != BwdPhase::FINISH) {
    const size_t smemA = (size_t)(2 * M * D + 2 * kT * D + 3 * kT) * sizeof(float);
    e = cudaFuncSetAttribute(bwd_decode_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smemA);
    if (e != cudaSuccess) return e;
    bwd_decode_kernel<T, D><<<grid, kT, smemA, st>>>((const T*)Q, qbs, (const T*)K, (const T*)dY,
                                                     d.k, d.dy, d.lens, Z, (int)d.H, d.N, M, c,
                                                     scale, p.chunk_tokens(), dkf, dq_dec, dzp);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    // dZ (this device's tokens) and delta_e = rowsum(dZ * Z)
    reduce_dz_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(
        dzp, Z, d.BH(), M, D, p.chunks, phase == BwdPhase::DZ ? dz_io : dz, delta);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    if (phase == BwdPhase::DZ) return cudaSuccess;
  } else {
    // dZ summed over the shards: delta_e from it
    reduce_dz_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(
        dz_io, Z, d.BH(), M, D, 1, dz, delta);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  }

  const size_t smemB = (size_t)(2 * M * D + 2 * M + 2 * kT * D) * sizeof(float);
  e = cudaFuncSetAttribute(bwd_encode_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smemB);
  if (e != cudaSuccess) return e;
  bwd_encode_kernel<T, D><<<grid, kT, smemB, st>>>((const T*)Q, qbs, (const T*)K, (const T*)V, dkf,
                                                   lse, dz, delta, d.k, d.v, d.dk, d.dv, d.lens,
                                                   (int)d.H, d.N, M, c, scale, p.chunk_tokens(),
                                                   (T*)dK, (T*)dV, dq_enc);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;

  const bool shared_q = (qbs == 0);
  const int64_t total = shared_q ? d.H * M * D : d.BH() * M * D;
  if (dq32)
    reduce_dq_kernel<float><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
        dq_dec, dq_enc, (int)d.B, (int)d.H, M, D, p.chunks, shared_q, dq32);
  else
    reduce_dq_kernel<T><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
        dq_dec, dq_enc, (int)d.B, (int)d.H, M, D, p.chunks, shared_q, (T*)dQ);
  return cudaPeekAtLastError();
}

}  // namespace

cudaError_t launch_bwd(const void* Q, int64_t qbs, const void* K, const void* V, const void* dY,
                       const float* Z, const float* lse, void* dQ, void* dK, void* dV,
                       const Dims& d, flare_dtype_t dt, float scale, const WsLayout& L,
                       char* ws, cudaStream_t st, BwdPhase phase, float* dz, float* dq32,
                       const PadZero* pz, const PlanArgs* plan) {
  // the tensor-core backward zeroes the padding and computes a deferred work
  // plan in its preparation kernel; the CUDA-core one uses the standalone
  // kernels
  if (choose_path(d.N, d.M, d.D, dt).tc_bwd)
    return launch_tc_bwd(Q, qbs, K, V, dY, Z, lse, dQ, dK, dV, d, scale, L, ws, st, phase, dz,
                         dq32, pz, plan);
  if (plan) {
    const cudaError_t e = launch_plan(*plan, st);
    if (e != cudaSuccess) return e;
  }
#define FLARE_BWD_T(T, DD) \
  bwd_t<T, DD>(Q, qbs, K, V, dY, Z, lse, dQ, dK, dV, d, scale, L, ws, st, phase, dz, dq32)
  cudaError_t e = (dt == FLARE_F32) ? (d.D == 16 ? FLARE_BWD_T(float, 16) : FLARE_BWD_T(float, 32))
                                    : (d.D == 16 ? FLARE_BWD_T(__nv_bfloat16, 16)
                                                 : FLARE_BWD_T(__nv_bfloat16, 32));
#undef FLARE_BWD_T
  if (e == cudaSuccess && pz) e = launch_pad_zero(*pz, d.BH(), st);
  return e;
}

}  // namespace flare

// ============================================================ FLARE++ backward
//
// Q_dyn = Q + Z1, Z1 = encode(Q, K, V) with learned Q [H,M,D] shared over the
// batch (FLARE++ abstract), and Y = FLARE(Q_dyn, K, V).  After FLARE's
// backward with per-batch latents Q_dyn has produced dQ_dyn, dK and dV, the
// first encode's gradient with upstream dZ1 = dQ_dyn is added here:
//   P1 = exp(s Q K^T - lse1), dP1 = dZ1 V^T, delta1 = rowsum(dZ1 * Z1),
//   dA1 = P1 * (dP1 - delta1), dV += P1^T dZ1, dK += s dA1^T Q,
//   dQ = sum over b of (dQ_dyn + s dA1 K).

namespace flare {
namespace {

// dZ1 = dQ_dyn (widened to float) and delta1 = rowsum(dZ1 * Z1); one warp per
// latent row.
template <typename T>
__global__ void pp_dz1_kernel(const T* __restrict__ dqd, const float* __restrict__ z1,
                              int64_t rows, int D, float* __restrict__ dz1,
                              float* __restrict__ delta1) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  float v = 0.f, prod = 0.f;
  if (lane < D) {
    v = to_f(dqd[w * D + lane]);
    prod = v * z1[w * D + lane];
    dz1[w * D + lane] = v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) prod += __shfl_xor_sync(0xffffffffu, prod, o);
  if (lane == 0) delta1[w] = prod;
}

// The first encode's gradient, added into dK and dV (read-modify-write of
// each thread's own token rows), with per-chunk partials of its dQ part.
template <typename T, int D>
__global__ void __launch_bounds__(kT)
    pp_encode_bwd_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                         const T* __restrict__ V, const float* __restrict__ lse1,
                         const float* __restrict__ dz1, const float* __restrict__ delta1, Tok tk,
                         Tok tv, Tok tdk, Tok tdv, const int32_t* __restrict__ lens, int H,
                         int64_t N, int M, float c, float s, int64_t chunk_tokens,
                         T* __restrict__ dK, T* __restrict__ dV, float* __restrict__ dq_part) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [M][D]
  float* dzs = qs + M * D;        // [M][D]
  float* ls = dzs + M * D;        // [M] lse1 in log2 units
  float* des = ls + M;            // [M] delta1
  float* ks = des + M;            // [kT][D]
  float* vs = ks + kT * D;        // [kT][D]
  const int chunk = blockIdx.x, chunks = gridDim.x;
  const int64_t bh = blockIdx.y, h = bh % H;
  const int64_t n0 = (int64_t)chunk * chunk_tokens;
  const int64_t n1 = min(seq_len(lens, bh / H, N), n0 + chunk_tokens);   // padding: none
  const int64_t kh = tk.head(bh, H), vh = tv.head(bh, H);
  const int64_t dkh = tdk.head(bh, H), dvh = tdv.head(bh, H);
  for (int i = threadIdx.x; i < M * D; i += blockDim.x) {
    qs[i] = to_f(Q[h * (int64_t)M * D + i]);
    dzs[i] = dz1[bh * M * D + i];
  }
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    ls[i] = lse1[bh * M + i] * kLog2e;
    des[i] = delta1[bh * M + i];
  }
  const int tid = threadIdx.x;
  const bool active_m = tid < M;
  float dq[D];
#pragma unroll
  for (int d = 0; d < D; ++d) dq[d] = 0.f;

  for (int64_t t0 = n0; t0 < n1; t0 += kT) {
    const int nt = (int)imin64(kT, n1 - t0);
    __syncthreads();
    for (int i = tid; i < kT * D; i += blockDim.x) {
      const int j = i / D, d = i % D;
      ks[i] = (j < nt) ? to_f(K[kh + (t0 + j) * tk.sn + d]) : 0.f;
      vs[i] = (j < nt) ? to_f(V[vh + (t0 + j) * tv.sn + d]) : 0.f;
    }
    __syncthreads();
    // one thread per token: the encode's dV and dK parts, added to the rows
    if (tid < nt) {
      const int64_t n = t0 + tid;
      float k[D], v[D], dk[D], dv[D];
#pragma unroll
      for (int d = 0; d < D; ++d) {
        k[d] = ks[tid * D + d];
        v[d] = vs[tid * D + d];
        dk[d] = 0.f;
        dv[d] = 0.f;
      }
      for (int m = 0; m < M; ++m) {
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          a = fmaf(k[d], qs[m * D + d], a);
          dp = fmaf(dzs[m * D + d], v[d], dp);
        }
        const float p = exp2f(a * c - ls[m]);
        const float dA = s * p * (dp - des[m]);
#pragma unroll
        for (int d = 0; d < D; ++d) {
          dv[d] = fmaf(p, dzs[m * D + d], dv[d]);
          dk[d] = fmaf(dA, qs[m * D + d], dk[d]);
        }
      }
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int64_t ok = dkh + n * tdk.sn + d, ov = dvh + n * tdv.sn + d;
        dK[ok] = from_f<T>(to_f(dK[ok]) + dk[d]);
        dV[ov] = from_f<T>(to_f(dV[ov]) + dv[d]);
      }
    }
    // one thread per latent: the encode's part of dQ over this tile
    if (active_m) {
      float q[D], dzr[D];
#pragma unroll
      for (int d = 0; d < D; ++d) {
        q[d] = qs[tid * D + d];
        dzr[d] = dzs[tid * D + d];
      }
      const float lm = ls[tid], dm = des[tid];
      for (int j = 0; j < nt; ++j) {
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          a = fmaf(ks[j * D + d], q[d], a);
          dp = fmaf(dzr[d], vs[j * D + d], dp);
        }
        const float dA = s * exp2f(a * c - lm) * (dp - dm);
#pragma unroll
        for (int d = 0; d < D; ++d) dq[d] = fmaf(dA, ks[j * D + d], dq[d]);
      }
    }
  }
  if (active_m) {
    const int64_t row = (bh * chunks + chunk) * M + tid;
#pragma unroll
    for (int d = 0; d < D; ++d) dq_part[row * D + d] = dq[d];
  }
}

// dQ[h] = sum over b of (dQ_dyn[b, h] + sum over chunks of the encode
// partials), in a fixed order.  One thread per output element.  With dq32
// (a shard of a context-parallel backward) the sum goes to float32 and
// includes dQ_dyn only when add_dqd.
template <typename T>
__global__ void pp_dq_kernel(const T* __restrict__ dqd, const float* __restrict__ dq_part, int B,
                             int H, int M, int D, int chunks, T* __restrict__ dQ,
                             float* __restrict__ dq32, bool add_dqd) {
  const int64_t per = (int64_t)H * M * D;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= per) return;
  const int64_t h = i / ((int64_t)M * D);
  const int64_t md = i % ((int64_t)M * D);
  float acc = 0.f;
  for (int b = 0; b < B; ++b) {
    const int64_t bh = (int64_t)b * H + h;
    if (add_dqd) acc += to_f(dqd[(int64_t)b * per + i]);
    for (int k = 0; k < chunks; ++k) acc += dq_part[(bh * chunks + k) * (int64_t)M * D + md];
  }
  if (dq32)
    dq32[i] = acc;
  else
    dQ[i] = from_f<T>(acc);
}

template <typename T, int D>
cudaError_t pp_tail_t(const void* Q, const void* K, const void* V, const float* z1,
                      const float* lse1, const void* dqd, void* dQ, void* dK, void* dV,
                      const Dims& d, float scale, const WsLayout& L, char* ws, cudaStream_t st,
                      float* dq32, bool add_dqd) {
  const ChunkPlan& p = L.ppe;
  const int M = (int)d.M;
  const int64_t BH = d.BH();
  float* dz1 = (float*)(ws + L.dz1);
  float* delta1 = (float*)(ws + L.delta1);
  float* dqe = (float*)(ws + L.dqe);
  cudaError_t e;
  const int64_t rows = BH * M;
  pp_dz1_kernel<T><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>((const T*)dqd, z1, rows,
                                                                        D, dz1, delta1);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  const size_t smem = (size_t)(2 * M * D + 2 * M + 2 * kT * D) * sizeof(float);
  e = cudaFuncSetAttribute(pp_encode_bwd_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.chunks, (unsigned)BH);
  pp_encode_bwd_kernel<T, D><<<grid, kT, smem, st>>>(
      (const T*)Q, (const T*)K, (const T*)V, lse1, dz1, delta1, d.k, d.v, d.dk, d.dv, d.lens,
      (int)d.H, d.N, M, scale * kLog2e, scale, p.chunk_tokens(), (T*)dK, (T*)dV, dqe);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  const int64_t per = d.H * M * D;
  pp_dq_kernel<T><<<(unsigned)((per + 255) / 256), 256, 0, st>>>((const T*)dqd, dqe, (int)d.B,
                                                                 (int)d.H, M, D, p.chunks,
                                                                 (T*)dQ, dq32,
                                                                 dq32 == nullptr || add_dqd);
  return cudaPeekAtLastError();
}

}  // namespace

cudaError_t launch_pp_bwd_tail(const void* Q, const void* K, const void* V, const float* z1,
                               const float* lse1, const void* dqd, void* dQ, void* dK, void* dV,
                               const Dims& d, flare_dtype_t dt, float scale, const WsLayout& L,
                               char* ws, cudaStream_t st, float* dq32, bool add_dqd) {
  if (choose_path(d.N, d.M, d.D, dt).tc_bwd)
    return launch_tc_enc_bwd(Q, K, V, z1, lse1, dqd, dQ, dK, dV, d, scale, L, ws, st, dq32,
                             add_dqd);
#define FLARE_PP_TAIL_T(T, DD) \
  pp_tail_t<T, DD>(Q, K, V, z1, lse1, dqd, dQ, dK, dV, d, scale, L, ws, st, dq32, add_dqd)
  if (dt == FLARE_F32) return d.D == 16 ? FLARE_PP_TAIL_T(float, 16) : FLARE_PP_TAIL_T(float, 32);
  return d.D == 16 ? FLARE_PP_TAIL_T(__nv_bfloat16, 16) : FLARE_PP_TAIL_T(__nv_bfloat16, 32);
#undef FLARE_PP_TAIL_T
}

}  // namespace flare
