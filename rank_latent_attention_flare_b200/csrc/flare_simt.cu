// CUDA-core (FFMA + exp2f) kernels of the FLARE forward: encode partials,
// partial combine and decode.  They serve float32 inputs (where the
// tensor-core path's bf16 operand rounding would break a 1e-5 tolerance)
// and bf16 shapes the tensor-core kernels do not cover.
//
// Encode, per (b, h) and latent m ("Flare Fast Low Rank Attention" skill
// page, section 2): Z[m] = sum_n softmax_n(s Q[m].K[n]) V[n], evaluated as an
// online softmax over token tiles.  Logits are kept in log2 units
// (s * log2(e) folded into Q) so every exponential is one exp2.
// Decode (FLARE arXiv abstract, second SDPA call): Y[n] = softmax_m(s K[n].Q[m]) Z.
#include "flare_plan.cuh"

namespace flare {
namespace {

// One CTA = one chunk of tokens of one (b, h); thread m owns latent row m.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtEncThreads)
    simt_encode_kernel(const T* __restrict__ Q, int64_t q_bstride, const T* __restrict__ K,
                       const T* __restrict__ V, Tok tk, Tok tv, const int32_t* __restrict__ lens,
                       int H, int64_t N, int M, float c, int64_t chunk_tokens,
                       float* __restrict__ part_ml,
                       float* __restrict__ part_acc) {
  __shared__ float ks[kSimtEncTile][D];
  __shared__ float vs[kSimtEncTile][D];
  const int chunk = blockIdx.x;
  const int chunks = gridDim.x;
  const int64_t bh = blockIdx.y;
  const int64_t b = bh / H, h = bh % H;
  const int64_t n0 = (int64_t)chunk * chunk_tokens;
  const int64_t n1 = min(seq_len(lens, b, N), n0 + chunk_tokens);   // empty past the length
  const T* Kb = K + tk.head(bh, H);
  const T* Vb = V + tv.head(bh, H);
  const int m = threadIdx.x;
  const bool active = m < M;

  float q[D];
#pragma unroll
  for (int d = 0; d < D; ++d)
    q[d] = active ? to_f(Q[b * q_bstride + ((int64_t)h * M + m) * D + d]) * c : 0.f;
  float mref = -INFINITY, l = 0.f;
  float acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) acc[d] = 0.f;

  for (int64_t t0 = n0; t0 < n1; t0 += kSimtEncTile) {
    const int nt = (int)imin64(kSimtEncTile, n1 - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < kSimtEncTile * D; i += blockDim.x) {
      const int j = i / D, d = i % D;
      float kv = 0.f, vv = 0.f;
      if (j < nt) {
        kv = to_f(Kb[(t0 + j) * tk.sn + d]);
        vv = to_f(Vb[(t0 + j) * tv.sn + d]);
      }
      ks[j][d] = kv;
      vs[j][d] = vv;
    }
    __syncthreads();
    if (active) {
      float s[kSimtEncTile];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < kSimtEncTile; ++j) {
        float a = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) a = fmaf(q[d], ks[j][d], a);
        s[j] = (j < nt) ? a : -INFINITY;
        mx = fmaxf(mx, s[j]);
      }
      if (mx > mref) {  // rescale the running sums to the new maximum
        const float f = exp2f(mref - mx);
        l *= f;
#pragma unroll
        for (int d = 0; d < D; ++d) acc[d] *= f;
        mref = mx;
      }
#pragma unroll
      for (int j = 0; j < kSimtEncTile; ++j) {
        const float p = exp2f(s[j] - mref);
        l += p;
#pragma unroll
        for (int d = 0; d < D; ++d) acc[d] = fmaf(p, vs[j][d], acc[d]);
      }
    }
  }
  if (active) {
    const int64_t row = (bh * chunks + chunk) * M + m;
    part_ml[row * 2 + 0] = mref;
    part_ml[row * 2 + 1] = l;
#pragma unroll
    for (int d = 0; d < D; ++d) part_acc[row * D + d] = acc[d];
  }
}

// One thread per token; Q (pre-scaled to log2 units) and Z staged in smem.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtDecThreads)
    simt_decode_kernel(const T* __restrict__ Q, int64_t q_bstride, const T* __restrict__ K,
                       const float* __restrict__ Zf, T* __restrict__ Y, Tok tk, Tok ty,
                       const int32_t* __restrict__ lens, int H, int64_t N, int M, float c) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* zs = sm + M * D;
  const int64_t bh = blockIdx.y;
  const int64_t b = bh / H, h = bh % H;
  for (int i = threadIdx.x; i < M * D; i += blockDim.x) {
    qs[i] = to_f(Q[b * q_bstride + h * (int64_t)M * D + i]) * c;
    zs[i] = Zf[bh * M * D + i];
  }
  __syncthreads();
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= seq_len(lens, b, N)) return;   // padding rows are zeroed separately
  const T* kr = K + tk.head(bh, H) + n * tk.sn;
  float k[D];
#pragma unroll
  for (int d = 0; d < D; ++d) k[d] = to_f(kr[d]);
  float mx = -INFINITY;
  for (int m = 0; m < M; ++m) {
    float a = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) a = fmaf(k[d], qs[m * D + d], a);
    mx = fmaxf(mx, a);
  }
  float sum = 0.f, y[D];
#pragma unroll
  for (int d = 0; d < D; ++d) y[d] = 0.f;
  for (int m = 0; m < M; ++m) {
    float a = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) a = fmaf(k[d], qs[m * D + d], a);
    const float p = exp2f(a - mx);
    sum += p;
#pragma unroll
    for (int d = 0; d < D; ++d) y[d] = fmaf(p, zs[m * D + d], y[d]);
  }
  const float inv = 1.f / sum;
  T* yr = Y + ty.head(bh, H) + n * ty.sn;
#pragma unroll
  for (int d = 0; d < D; ++d) yr[d] = from_f<T>(y[d] * inv);
}

// One warp per (b, h, m); lane d < D owns Z[m][d].  Merges the per-chunk
// (max, sum, acc) records with the log-sum-exp rule and, for FLARE++,
// writes Q_dyn = Q + Z in the input dtype.  The records are `groups` blocks
// of [BH][slots] (one block per token shard when the tokens were encoded in
// shards), merged in a fixed order: block by block, slot by slot.
template <typename T>
__global__ void combine_kernel(const float* __restrict__ part_ml,
                               const float* __restrict__ part_acc, int64_t BH, int H, int M,
                               int D, int slots, int groups, const int2* __restrict__ heads,
                               int sub, const PadZero z, int64_t own_blocks, float* __restrict__ Zf,
                               __nv_bfloat16* __restrict__ Zb, float* __restrict__ Z_save,
                               float* __restrict__ lse_save, const T* __restrict__ Qpp,
                               T* __restrict__ Qdyn) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  if (blockIdx.x >= own_blocks) {   // the padding rows of Y
    const int64_t x = blockIdx.x - own_blocks;
    zero_padding_part(z, x % z.nxb, x / z.nxb);
    return;
  }
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= BH * M) return;
  const int64_t bh = w / M;
  const int m = (int)(w % M);
  // this head's records: `cnt` slots from `r0` in each group (the work
  // plan's units of `sub` records when a head table is given)
  int64_t r0 = bh * slots;
  int cnt = slots;
  if (heads) {
    const int2 hs = heads[bh];
    r0 = (int64_t)hs.x * sub;
    cnt = hs.y * sub;
  }
  const int64_t gstride = BH * slots;
  // lane s reads record s of each run of 32: the loads of a run are in
  // flight together
  float mstar = -INFINITY;
  for (int g = 0; g < groups; ++g)
    for (int s0 = 0; s0 < cnt; s0 += 32)
      if (s0 + lane < cnt)
        mstar = fmaxf(mstar, part_ml[((g * gstride + r0 + s0 + lane) * M + m) * 2]);
  for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));
  // then, record by record in order, l += f l_s and (lane d) acc += f acc_s[d]
  float l = 0.f, acc = 0.f;
  for (int g = 0; g < groups; ++g)
    for (int s0 = 0; s0 < cnt; s0 += 32) {
      const int n = min(32, cnt - s0);   // warp-uniform
      float ms = -INFINITY, ls = 0.f;
      if (lane < n) {
        const int64_t row = (g * gstride + r0 + s0 + lane) * M + m;
        ms = part_ml[row * 2];
        ls = part_ml[row * 2 + 1];
      }
      const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - mstar);   // an empty record: none
      for (int u0 = 0; u0 < n; u0 += 8) {
        float a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          a[u] = (u0 + u < n && lane < D)
                     ? part_acc[((g * gstride + r0 + s0 + u0 + u) * M + m) * D + lane]
                     : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (u0 + u >= n) break;
          const float mu = __shfl_sync(0xffffffffu, ms, u0 + u);
          const float fu = __shfl_sync(0xffffffffu, f, u0 + u);
          const float lu = __shfl_sync(0xffffffffu, ls, u0 + u);
          if (mu == -INFINITY) continue;
          l = fmaf(fu, lu, l);
          acc = fmaf(fu, a[u], acc);
        }
      }
    }
  if (lane < D) {
    const float z = (l > 0.f) ? acc / l : 0.f;   // no tokens: an empty weighted sum
    const int64_t o = w * D + lane;
    Zf[o] = z;
    Zb[o] = __float2bfloat16_rn(z);
    if (Z_save) Z_save[o] = z;
    if (Qdyn) {
      const int64_t h = bh % H;
      Qdyn[o] = from_f<T>(to_f(Qpp[(h * M + m) * D + lane]) + z);
    }
  }
  if (lane == 0 && lse_save) lse_save[w] = (l > 0.f) ? (mstar + log2f(l)) * kLn2 : -INFINITY;
}

__global__ void check_lens_kernel(const int32_t* __restrict__ lens, int64_t B, int64_t N,
                                  uint32_t* __restrict__ err) {
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && (lens[b] < 0 || (int64_t)lens[b] > N)) record_error(err, kErrSeqLen);
}

// ------------------------------------------------ work plans with lengths

// The forward's plan: one block (the backward runs the same body in an extra
// block of its preparation kernel).
constexpr int kPlanThreads = 256;

__global__ void __launch_bounds__(kPlanThreads) var_plan_kernel(const PlanArgs a) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  var_plan_body<kPlanThreads>(a);
}

// Zeroes the padding rows of up to two token tensors: blockIdx.y = b H + h,
// blockIdx.x one of z.nxb blocks per head.
__global__ void zero_padding_kernel(const PadZero z) { zero_padding_part(z, blockIdx.x, blockIdx.y); }

template <typename T, int D>
cudaError_t simt_encode_t(const void* Q, int64_t qbs, const void* K, const void* V,
                          const Dims& d, float scale, const ChunkPlan& plan, float* part_ml,
                          float* part_acc, cudaStream_t st) {
  dim3 grid(plan.chunks, (unsigned)d.BH());
  simt_encode_kernel<T, D><<<grid, kSimtEncThreads, 0, st>>>(
      (const T*)Q, qbs, (const T*)K, (const T*)V, d.k, d.v, d.lens, (int)d.H, d.N, (int)d.M,
      scale * kLog2e, plan.chunk_tokens(), part_ml, part_acc);
  return cudaPeekAtLastError();
}

template <typename T, int D>
cudaError_t simt_decode_t(const void* Q, int64_t qbs, const void* K, const float* Zf, void* Y,
                          const Dims& d, float scale, cudaStream_t st) {
  const size_t smem = (size_t)2 * d.M * D * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(simt_decode_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((d.N + kSimtDecThreads - 1) / kSimtDecThreads), (unsigned)d.BH());
  simt_decode_kernel<T, D><<<grid, kSimtDecThreads, smem, st>>>(
      (const T*)Q, qbs, (const T*)K, Zf, (T*)Y, d.k, d.y, d.lens, (int)d.H, d.N, (int)d.M,
      scale * kLog2e);
  return cudaPeekAtLastError();
}

}  // namespace

cudaError_t launch_simt_encode(const void* Q, int64_t qbs, const void* K, const void* V,
                               const Dims& d, flare_dtype_t dt, float scale,
                               const ChunkPlan& plan, float* part_ml, float* part_acc,
                               cudaStream_t st) {
  if (dt == FLARE_F32)
    return d.D == 16 ? simt_encode_t<float, 16>(Q, qbs, K, V, d, scale, plan, part_ml, part_acc, st)
                     : simt_encode_t<float, 32>(Q, qbs, K, V, d, scale, plan, part_ml, part_acc, st);
  return d.D == 16
             ? simt_encode_t<__nv_bfloat16, 16>(Q, qbs, K, V, d, scale, plan, part_ml, part_acc, st)
             : simt_encode_t<__nv_bfloat16, 32>(Q, qbs, K, V, d, scale, plan, part_ml, part_acc, st);
}

cudaError_t launch_simt_decode(const void* Q, int64_t qbs, const void* K, const float* Zf,
                               void* Y, const Dims& d, flare_dtype_t dt, float scale,
                               cudaStream_t st) {
  if (dt == FLARE_F32)
    return d.D == 16 ? simt_decode_t<float, 16>(Q, qbs, K, Zf, Y, d, scale, st)
                     : simt_decode_t<float, 32>(Q, qbs, K, Zf, Y, d, scale, st);
  return d.D == 16 ? simt_decode_t<__nv_bfloat16, 16>(Q, qbs, K, Zf, Y, d, scale, st)
                   : simt_decode_t<__nv_bfloat16, 32>(Q, qbs, K, Zf, Y, d, scale, st);
}

cudaError_t launch_check_lens(const Dims& d, uint32_t* err, cudaStream_t st) {
  if (d.lens == nullptr) return cudaSuccess;
  check_lens_kernel<<<(unsigned)((d.B + 255) / 256), 256, 0, st>>>(d.lens, d.B, d.N, err);
  return cudaPeekAtLastError();
}

cudaError_t launch_plan(const PlanArgs& a, cudaStream_t st) {
  if (!a.on()) return cudaSuccess;
  var_plan_kernel<<<1, kPlanThreads, 0, st>>>(a);
  return cudaPeekAtLastError();
}

cudaError_t launch_var_plan(Dims& d, const WsLayout& L, char* ws, cudaStream_t st, int sms,
                            PlanArgs* defer) {
  if (d.lens == nullptr) return cudaSuccess;
  uint32_t* err = (uint32_t*)(ws + L.hdr);
  if (L.n_enc == 0) return launch_check_lens(d, err, st);   // CUDA-core path: the chunk plan
  PlanArgs a;
  a.lens = d.lens;
  a.B = d.B;
  a.H = d.H;
  a.N = d.N;
  a.k0 = PlanKind{kTcEncTile, 2 * sms, 12.f, (int)L.n_enc, (int4*)(ws + L.vu_enc), (int2*)(ws + L.vh_enc)};
  a.k1 = PlanKind{kTcTile, sms, 6.f, (int)L.n_tok, (int4*)(ws + L.vu_tok), (int2*)(ws + L.vh_tok)};
  a.err = err;
  d.venc = VarPlan{a.k0.units, a.k0.heads, L.n_enc};
  d.vtok = VarPlan{a.k1.units, a.k1.heads, L.n_tok};
  if (defer) {   // computed by a block of a kernel the caller launches first
    *defer = a;
    return cudaSuccess;
  }
  return launch_plan(a, st);
}

PadZero pad_zero(void* X0, const Tok& t0, void* X1, const Tok& t1, const Dims& d, flare_dtype_t dt,
                 int threads) {
  PadZero z;
  if (d.lens == nullptr) return z;
  z.x0 = (uint8_t*)X0;
  z.t0 = t0;
  z.x1 = (uint8_t*)X1;
  z.t1 = X1 ? t1 : t0;
  z.lens = d.lens;
  z.N = d.N;
  z.H = (int)d.H;
  z.esz = (dt == FLARE_F32) ? 4 : 2;
  const int per_row = (int)d.D * z.esz / 16;   // 16-byte pieces per row: 2, 4 or 8
  z.lg_row = per_row == 2 ? 1 : (per_row == 4 ? 2 : 3);
  // about sixteen pieces per thread for a head that is all padding, at most 32 blocks
  z.nxb = (int)imax64(1, imin64((d.N * per_row + 16 * threads - 1) / (16 * threads), 32));
  return z;
}

cudaError_t launch_pad_zero(const PadZero& z, int64_t BH, cudaStream_t st) {
  if (z.x0 == nullptr) return cudaSuccess;
  zero_padding_kernel<<<dim3((unsigned)z.nxb, (unsigned)BH), 256, 0, st>>>(z);
  return cudaPeekAtLastError();
}

cudaError_t launch_combine(const Dims& d, flare_dtype_t dt, int slots_per_bh, int sub, int groups,
                           const float* part_ml, const float* part_acc, float* Zf,
                           __nv_bfloat16* Zb, float* Z_save, float* lse_save, const void* Qpp,
                           void* Qdyn, cudaStream_t st, const PadZero* pz) {
  const int64_t warps = d.BH() * d.M;
  const int threads = 256;
  const int64_t own = (warps * 32 + threads - 1) / threads;
  const PadZero z = pz ? *pz : PadZero{};
  const unsigned blocks = (unsigned)(own + z.blocks(d.BH()));
  if (dt == FLARE_F32)
    launch_pdl(combine_kernel<float>, blocks, threads, 0, st,
        part_ml, part_acc, d.BH(), (int)d.H, (int)d.M, (int)d.D, slots_per_bh, groups,
        d.venc.heads, sub, z, own, Zf, Zb, Z_save, lse_save, (const float*)Qpp, (float*)Qdyn);
  else
    launch_pdl(combine_kernel<__nv_bfloat16>, blocks, threads, 0, st,
        part_ml, part_acc, d.BH(), (int)d.H, (int)d.M, (int)d.D, slots_per_bh, groups,
        d.venc.heads, sub, z, own, Zf, Zb, Z_save, lse_save, (const __nv_bfloat16*)Qpp,
        (__nv_bfloat16*)Qdyn);
  return cudaPeekAtLastError();
}

}  // namespace flare
