// Tensor-core FLARE backward for sm_100a: bf16 inputs, M in {128, 256}
// latents, D in {16, 32}.  Gradients of sum(Y * dY) with respect to Q, K and V with
// the logits of both stages recomputed on the tensor cores (tcgen05.mma,
// TMEM accumulators, TMA-fed operands).  The pages give no backward; this is
// the chain rule through the encode (skill page section 2: softmax over the
// tokens of every latent row) and the decode (FLARE abstract: softmax over
// the latents of every token), as in flare_bwd.cu.
//
// Token-major notation per (b, h), c = scale * log2(e), all exponentials in
// base 2 ("log2 units"):
//   S[n,m]   = K[n] . Q[m]                        (both stages' logits / scale)
//   P_d[n,m] = 2^(c S - mx'[n])                   decode softmax over m;
//              mx'[n] = c max_m S + log2(row sum) (its log-sum-exp)
//   P_e[n,m] = 2^(c S - lse2[m])                  encode softmax over n;
//              lse2 = forward lse * log2(e)
//   dPd = dY Z^T, delta_d[n] = sum_m P_d dPd = dY[n] . Y[n]
//   dPe = V dZ^T, delta_e[m] = dZ[m] . Z[m],  dZ = P_d^T dY
//   G   = P_d (dPd - delta_d) + P_e (dPe - delta_e)   (the logit gradient / scale)
//   dK = s G Q,  dQ = s G^T K,  dV = P_e^T... = sum_m P_e[n,m] dZ[m]
//
// Pass A (tc_bwd_a_kernel, per 128-token tile, one thread per token row):
// S = K Q^T into TMEM; row max and P = 2^(c S - c max) as in the forward's
// decode; P (bf16) into TMEM for Y = P Z and into shared memory for
// dZ += P^T dY' with dY' = dY / rowsum written over the dY tile; the row's
// mx' and delta_d = dY . Y go to the workspace.
//
// Between the passes (bwd_mid_kernel): dZ = sum of the chunk partials,
// delta_e, and the split of the encode weights
//   P_e[n,m] = P_d[n,m] * g[n] * f[m],  g[n] = 2^(mx'[n] - R), f[m] = 2^(R - lse2[m])
// with R = max_m lse2[m].  f goes into the operand dZ'' = f dZ (bf16) and into
// an extra K-step of the dPe'' = V dZ''^T - f delta_e product (three bf16
// terms of -f delta_e against a tile of ones), so
//   G = P_d (dPd - delta_d + g dPe''),   dV[n] = g[n] sum_m P_d[n,m] dZ''[m]
// and pass B needs ONE exponential per token-latent pair.  When the lse2 of
// a head spread over more than 64 (f or g could leave the float range) the
// head takes the exact form instead: f = 1, P_e = 2^(c S - lse2[m]) per
// element.
//
// Pass B (tc_bwd_b_kernel, per 128-token tile, latents in quarters of 32):
// S, dPd and dPe'' of a quarter into TMEM; G and the dV weights (bf16) back
// into TMEM for dK += G Q and dV += P dZ'' (tensor cores, token rows), and G
// into shared memory for dQ += G^T K (latent rows, accumulated over the
// chunk's tiles).  dK and dV are final per tile; dQ partials per chunk are
// summed in a fixed order afterwards, so results are reproducible bitwise.
//
// With M = 256 the decode stage runs as two passes of the forward's
// pipelines instead of pass A (tc_bwd_t), and pass B once per latent half.
//
// Roles per CTA (384 threads): warps 0-3 and 4-7 are the row warpgroups,
// warp 8 issues TMA loads, warp 9 issues the MMAs, warps 10-11 only lend
// registers (as in the forward's decode kernel).
#include <cudaTypedefs.h>

#include "flare_plan.cuh"
#include "tc_primitives.cuh"

namespace flare {
namespace {

using namespace tc;

constexpr int kT = 128;          // tokens per tile
constexpr int kM = 128;          // latents of one pass-A / pass-B launch (M, or half of it)
constexpr int kThr = 384;
constexpr int kRegsRow = 200;
constexpr int kRegsPro = 104;
constexpr int kWTma = 8;
constexpr int kWMma = 9;
constexpr int kBStages = 3;
constexpr uint32_t kSw128 = 2u;  // UMMA descriptor code of the 128-byte swizzle
constexpr uint32_t kSw32 = 6u;   // ... and of the 32-byte swizzle
constexpr float kSpreadMax = 64.f;     // log2 units: lse spread beyond which a head takes the exact form
constexpr float kRowRangeMax = kBwdRowRange;
// mode bits of the pass-B kernels
constexpr int kModeEncOnly = 1;   // the encode's gradient only (no decode term)
constexpr int kModeAccum = 2;     // dK, dV added to the values already in their rows

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// A [128 tokens x 128 latents] bf16 tile stored latent-contiguous, i.e. as
// the MN-major A operand of a [latents x tokens] x [tokens x D] product:
// 128-byte swizzle atoms of 64 latents x 8 tokens, consecutive atoms along
// the tokens 1 KB apart, the second 64 latents 16 KB further.  Offset of the
// 16-byte group of latents [8 grp, 8 grp + 8) in token row n.
constexpr uint32_t kMnLbo = 16384, kMnSbo = 1024, kMnKStep = 2048;  // K step = 16 tokens
__device__ __forceinline__ uint32_t mn_off(int n, int grp) {
  return (uint32_t)((grp >> 3) * 16384 + (n >> 3) * 1024 + (n & 7) * 128 +
                    (((grp & 7) ^ (n & 7)) << 4));
}

// Offset of 16-byte chunk ch of row r in a tile written by TMA with the
// swizzle make_map uses for rows of 2D bytes (64B for D = 32, 32B for 16).
template <int D>
__device__ __forceinline__ uint32_t tma_row_chunk(int r, int ch) {
  if (D == 32) return (uint32_t)(r * 64 + ((ch ^ ((r >> 1) & 3)) << 4));
  return (uint32_t)(r * 32 + ((ch ^ ((r >> 2) & 1)) << 4));
}

// Empty asm that names 16 registers as in/out operands: placed after a
// tcgen05.wait::ld it keeps every use of them behind the wait.
__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}


// ============================================================== pass A

template <int D>
struct ALayout {
  static constexpr int M = kM;
  static constexpr int KST = 4;               // K tiles: held until their S product
  static constexpr int DST = 4;               // dY tiles: held until their dZ product
  static constexpr int RB = 2 * D;
  static constexpr int TILE = kT * RB;        // one K or dY tile
  static constexpr int PBUF = kT * M * 2;     // one P tile (swizzled, latent-contiguous rows)
  static constexpr int P_OFF = 0;             // two P buffers per row warpgroup
  static constexpr int Q_OFF = 4 * PBUF;
  static constexpr int Z_OFF = Q_OFF + M * RB;
  static constexpr int ONE_OFF = Z_OFF + M * RB;  // second N block of Y's B operand
  static constexpr int K_OFF = ONE_OFF + M * RB;  // K ring
  static constexpr int DY_OFF = K_OFF + KST * TILE;   // dY ring
  static constexpr int BAR_OFF = DY_OFF + DST * TILE;
  static constexpr int NBARS = 2 * KST + 2 * DST + 1 + 2 + 2 + 4 + 2 + 4 + 1 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
};

// Per 128-token tile (the two row warpgroups alternate tiles), software
// pipelined: a warpgroup writes P of its tile j, starts the softmax of its
// tile j + 1 while Y = P [Z | e0] of tile j runs on the tensor cores, and
// then finishes tile j (delta_d, dY', dY'', statistics).  Each warpgroup has
// two Y accumulators in TMEM for that overlap.
template <int D, bool FLAT, bool VAR>
__global__ void __launch_bounds__(kThr, 1)
    tc_bwd_a_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmdY, const __grid_constant__ CUtensorMap tmZ,
                    int H, int64_t N, int q_per_batch, float c, int64_t tiles_per_bh,
                    int64_t chunk_tiles, const float* __restrict__ rref,
                    float4* __restrict__ stats, __nv_bfloat16* __restrict__ dy2,
                    uint32_t* __restrict__ flags, float* __restrict__ dz_part,
                    const int32_t* __restrict__ lens, const int4* __restrict__ units,
                    uint32_t* __restrict__ err) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  using L = ALayout<D>;
  constexpr int M = L::M;
  constexpr int RB = L::RB;
  constexpr int KST = L::KST;
  constexpr int DST = L::DST;
  constexpr uint32_t SW = umma_swizzle_code(RB);
  constexpr int R = M;          // TMEM columns of a row warpgroup's S
  constexpr int YC = D + 16;    // one [Y | row sum of bf16 P] accumulator
  constexpr int TY = 2 * M;     // Y accumulators: warpgroup w, buffer b at TY + YC (2 w + b)
  constexpr int TDZ = TY + 4 * YC;   // dZ accumulator (latent lanes)
  constexpr uint32_t NCOLS = 512;
  static_assert(TDZ + D <= 512, "TMEM budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + KST;
  uint64_t* d_full = k_empty + KST;
  uint64_t* d_empty = d_full + DST;
  uint64_t* qz_full = d_empty + DST;
  uint64_t* s_full = qz_full + 1;   // [w] S of the warpgroup's tile in TMEM
  uint64_t* p_full = s_full + 2;    // [w] P in shared memory, S columns read
  uint64_t* y_full = p_full + 2;    // [2 w + b] Y of the warpgroup's tile in buffer b complete
  uint64_t* a_done = y_full + 4;    // [w] Y read, dY' written
  uint64_t* dz_done = a_done + 2;   // [2 w + b] dZ of warpgroup w's tile in P buffer b complete
  uint64_t* dz_final = dz_done + 4;
  uint64_t* drain = dz_final + 1;   // [2]: one per issuing thread
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CtaWork cw = cta_work<VAR>(units, chunk_tiles, tiles_per_bh);
  if (cw.bh < 0) return;   // a unit the work plan leaves empty
  const int64_t bh = cw.bh;
  const int64_t h = bh % H;
  const int64_t tile0 = cw.tile0;
  const int nt = (int)cw.ntiles;
  // with lengths, tokens past the batch element's length are padding: the
  // work plan covers the head's own tiles only
  const HeadTiles<VAR> ht(lens, bh / H, N);

  // Y = P [Z | e0]: the second N block of the B operand holds a one in
  // column 0 of every latent row (same swizzled layout as the Z rows), so
  // the accumulator's column D is the row sum of the bf16 P the MMA uses.
  for (int m = threadIdx.x; m < M; m += blockDim.x) {
#pragma unroll
    for (int ch = 0; ch < D / 8; ++ch)
      *reinterpret_cast<uint4*>(smem + L::ONE_OFF + tma_row_chunk<D>(m, ch)) =
          make_uint4(ch == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < DST; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_empty[s], 1);
    }
    mbar_init(qz_full, 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], 128);
      mbar_init(&a_done[w], 128);
    }
    for (int k = 0; k < 4; ++k) {
      mbar_init(&y_full[k], 1);
      mbar_init(&dz_done[k], 1);
    }
    mbar_init(dz_final, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWMma) tmem_alloc(tmem_slot, NCOLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_release<kRegsPro>();
    if (warp == kWTma || warp == kWMma + 2) {
      // two producers, one per ring, so a dY tile that waits for its slot
      // never holds back the K tile the next S needs
      if (lane == 0) {
        const bool kq = (warp == kWTma);
        uint64_t* full = kq ? k_full : d_full;
        uint64_t* empty = kq ? k_empty : d_empty;
        const int nst = kq ? KST : DST;
        uint8_t* ring = smem + (kq ? L::K_OFF : L::DY_OFF);
        const CUtensorMap* map = kq ? &tmK : &tmdY;
        prefetch_tmap(map);
        if (kq) {
          prefetch_tmap(&tmQ);
          prefetch_tmap(&tmZ);
          mbar_arrive_expect_tx(qz_full, 2 * M * RB);
          tma_load_3d(smem + L::Q_OFF, &tmQ, qz_full, 0, 0, (int32_t)(q_per_batch ? bh : h));
          tma_load_3d(smem + L::Z_OFF, &tmZ, qz_full, 0, 0, (int32_t)bh);
        }
        int issued = 0;
        for (int i = 0; i < nt; ++i) {
          const int s = i % nst;
          if (i >= nst && !mbar_wait_sleep(&empty[s], (uint32_t)(((i / nst) & 1) ^ 1))) {
            record_error(err, kErrBwdATmaWait);
            *abort_flag = 1;
            break;
          }
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&full[s], L::TILE);
          tma_load_tok<FLAT>(ring + s * L::TILE, map, &full[s], (int32_t)ht.row0(tile0 + i, kT),
                             bh, H);
          issued = i + 1;
        }
        // let every load still in flight land before the CTA can exit
        for (int i = (issued > nst ? issued - nst : 0); i < issued; ++i)
          mbar_wait_sleep(&full[i % nst], (uint32_t)((i / nst) & 1));
        if (kq) mbar_wait_sleep(qz_full, 0);
      }
    } else if (warp == kWMma || warp == kWMma + 1) {
      // Two issuing threads: warp 9 issues S (it waits on TMA tiles), warp
      // 10 issues Y and dZ (they wait on the row warps).
      if (lane == 0) {
        constexpr uint32_t idS = idesc_bf16_f32(128, M, 0, 0);
        constexpr uint32_t idY = idesc_bf16_f32(128, D + 16, 0, 1);   // N = [Z | e0]
        constexpr uint32_t idZ = idesc_bf16_f32(128, D, 1, 1);
        const uint32_t q_addr = smem_u32(smem + L::Q_OFF);
        const uint32_t z_addr = smem_u32(smem + L::Z_OFF);
        const uint32_t k0 = smem_u32(smem + L::K_OFF);
        const uint32_t dy0 = smem_u32(smem + L::DY_OFF);
        const uint32_t p0 = smem_u32(smem + L::P_OFF);
        // descriptors built once; per MMA only the address field moves
        const uint64_t dKk = smem_desc(k0, 16, 8 * RB, SW);           // K tile rows, K-major
        const uint64_t dQk = smem_desc(q_addr, 16, 8 * RB, SW);
        const uint64_t dPk = smem_desc(p0, 16, kMnSbo, kSw128);       // P, K-major (Y = P Z)
        const uint64_t dPm = smem_desc(p0, kMnLbo, kMnSbo, kSw128);   // P, MN-major (dZ)
        const uint64_t dZm = smem_desc(z_addr, M * RB, 8 * RB, SW);   // [Z | e0], MN-major
        const uint64_t dDYm = smem_desc(dy0, L::TILE, 8 * RB, SW);    // dY tile, MN-major
        constexpr uint32_t kTile16 = (uint32_t)L::TILE >> 4;
        constexpr uint32_t kRow16 = (uint32_t)RB;                     // 16 rows >> 4
        constexpr uint32_t kP16 = (uint32_t)L::PBUF >> 4;
        bool ok = mbar_wait_sleep(qz_full, 0);
        if (warp == kWMma) {
          // S(i) into warpgroup (i & 1)'s S columns once its tile i - 2 has
          // been read (p_full) and tile i's K is in shared memory
          for (int i = 0; ok && i < nt; ++i) {
            const int w = i & 1;
            const int s = i % KST;
            if (i >= 2 && !mbar_wait_sleep(&p_full[w], (uint32_t)(((i - 2) >> 1) & 1))) {
              ok = false;
              break;
            }
            if (!mbar_wait_sleep(&k_full[s], (uint32_t)((i / KST) & 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ko = (uint32_t)s * kTile16;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + w * R, dKk + ko + 2 * kk, dQk + 2 * kk, idS, kk > 0);
            mma_commit(&s_full[w]);
            mma_commit(&k_empty[s]);
            if (*abort_flag) ok = false;
          }
        } else {
          // Y(i) as soon as P(i) is written; dZ(i) once its warpgroup has
          // finished tile i (after the softmax of its next tile)
          auto issue_dZ = [&](int i) -> bool {
            const int w = i & 1;
            const int j = i >> 1;
            const int s = i % DST;
            if (!mbar_wait_sleep(&a_done[w], (uint32_t)(j & 1))) return false;
            tc_fence_after();
            const uint32_t po = (uint32_t)(2 * w + (j & 1)) * kP16;
            const uint32_t so = (uint32_t)s * kTile16;
#pragma unroll
            for (int kk = 0; kk < kT / 16; ++kk)
              mma_ss(tmem + TDZ, dPm + po + kk * (kMnKStep >> 4), dDYm + so + kk * kRow16, idZ,
                     (i > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&d_empty[s]);
            mma_commit(&dz_done[2 * w + (j & 1)]);
            return true;
          };
          for (int i = 0; ok && i < nt; ++i) {
            const int w = i & 1;
            const int j = i >> 1;
            if (!mbar_wait_sleep(&p_full[w], (uint32_t)(j & 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t po = (uint32_t)(2 * w + (j & 1)) * kP16;
#pragma unroll
            for (int kk = 0; kk < M / 16; ++kk)
              mma_ss(tmem + TY + YC * (2 * w + (j & 1)),
                     dPk + po + (kk >> 2) * (kMnLbo >> 4) + (kk & 3) * 2, dZm + kk * kRow16, idY,
                     kk > 0);
            mma_commit(&y_full[2 * w + (j & 1)]);
            if (i >= 2) ok = issue_dZ(i - 2);
            if (*abort_flag) ok = false;
          }
          for (int i = (nt > 2 ? nt - 2 : 0); ok && i < nt; ++i) ok = issue_dZ(i);
          mma_commit(dz_final);
        }
        if (!ok) {
          record_error(err, kErrBwdAMmaWait);
          *abort_flag = 1;
        }
        mma_commit(drain + (warp - kWMma));
        mbar_wait_sleep(drain + (warp - kWMma), 0);
      }
    }
  } else {
    regs_acquire<kRegsRow>();
    const int w = warp >> 2, qw = warp & 3;
    const int r = qw * 32 + lane;                    // TMEM lane = token row of the tile
    const uint32_t lb = (uint32_t)(qw * 32) << 16;
    const uint32_t tR = tmem + lb + w * R;
    const float Rh = rref[bh];
    const int nW = (nt - w + 1) / 2;
    bool ok = true;
    float mx_prev = 0.f, l_prev = 0.f;   // statistics of the tile whose finish is pending

    // the second half of tile j: Y (with the row sum of the bf16 P),
    // delta_d = dY . Y, dY' = dY / rowsum in place, dY'' = dY / g, statistics
    auto finish = [&](int j, float mx, float l) -> bool {
      const int i = 2 * j + w;
      const int s = i % DST;
      // rows that are not the tile's own tokens add nothing
      const int64_t tok = ht.row0(tile0 + i, kT) + r;
      const bool mine = ht.own(tile0 + i, kT, r);
      if (!warp_all(mbar_wait(&y_full[2 * w + (j & 1)], (uint32_t)((j >> 1) & 1)) &&
                    mbar_wait(&d_full[s], (uint32_t)((i / DST) & 1)) && !*abort_flag))
        return false;
      __syncwarp();
      tc_fence_after();
      float y[D];
      float lsum;   // row sum of the bf16 P (the weights the tensor cores used)
      const uint32_t ty = tmem + lb + TY + YC * (2 * w + (j & 1));
      if (D == 32) {
        uint32_t o[32], o2[16];
        tmem_ld32(ty, o);
        tmem_ld16(ty + 32, o2);
        tmem_wait_ld_dep(o);
        reg_fence16(o2);
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = __uint_as_float(o[d]);
        lsum = __uint_as_float(o2[0]);
      } else {
        uint32_t o[32];
        tmem_ld32(ty, o);
        tmem_wait_ld_dep(o);
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = __uint_as_float(o[d]);
        lsum = __uint_as_float(o[D]);
      }
      const float inv = 1.f / lsum;
      const float mxp = fmaf(mx, c, log2f(l));   // row log-sum-exp, log2 units
      const float lg = mxp - Rh;                  // log2 of g[n]
      const bool bad = lg < -kRowRangeMax;        // g[n] would leave the float range
      const float ginv = bad ? 0.f : ex2(-lg);    // 1 / g[n]
      uint8_t* dyt = smem + L::DY_OFF + s * L::TILE;
      float dot = 0.f, dot2 = 0.f;
      uint4 o2v[D / 8];
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) {
        uint4* p = reinterpret_cast<uint4*>(dyt + tma_row_chunk<D>(r, ch));
        const uint4 u = *p;
        const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
        uint32_t wv[4], w2[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float a0 = bf_lo(uu[jj]), a1 = bf_hi(uu[jj]);
          const float y0 = y[8 * ch + 2 * jj], y1 = y[8 * ch + 2 * jj + 1];
          dot = fmaf(a0, y0, fmaf(a1, y1, dot));
          w2[jj] = pack_bf16(a0 * ginv, a1 * ginv);           // dY'' = dY / g
          dot2 = fmaf(bf_lo(w2[jj]), y0, fmaf(bf_hi(w2[jj]), y1, dot2));
          // dY' = dY / rowsum (rows past N are zero already; with lengths
          // a right-aligned tile's earlier rows hold real dY)
          wv[jj] = (!VAR || mine) ? pack_bf16(a0 * inv, a1 * inv) : 0u;
        }
        *p = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        o2v[ch] = make_uint4(w2[0], w2[1], w2[2], w2[3]);
      }
      if (mine) {
        // delta_d = dY . Y and its counterpart with the rounded dY'' (= delta_d / g)
        stats[bh * N + tok] = make_float4(mxp, dot * inv, dot2 * inv, 0.f);
        uint4* dst = reinterpret_cast<uint4*>(dy2 + (bh * N + tok) * D);
#pragma unroll
        for (int ch = 0; ch < D / 8; ++ch) dst[ch] = o2v[ch];
      }
      if (warp_any(bad && mine) && lane == 0) atomicOr(flags + bh, 1u);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&a_done[w]);
      return true;
    };

    for (int j = 0; j < nW; ++j) {
      uint8_t* pbuf = smem + L::P_OFF + (2 * w + (j & 1)) * L::PBUF;
      // the P buffer of tile j was last read by the dZ of tile j - 2
      if (!warp_all(mbar_wait(&s_full[w], (uint32_t)(j & 1)) &&
                    (j < 2 || mbar_wait(&dz_done[2 * w + (j & 1)], (uint32_t)(((j - 2) >> 1) & 1))) &&
                    !*abort_flag)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      // pass 1: row max over the M logits (32-column chunks, double-buffered loads)
      constexpr int NC = M / 32;
      uint32_t a[2][32];
      float mf[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      tmem_ld32(tR, a[0]);
#pragma unroll
      for (int cc = 0; cc < NC; ++cc) {
        tmem_wait_ld_dep(a[cc & 1]);
        if (cc + 1 < NC) tmem_ld32(tR + 32 * (cc + 1), a[(cc + 1) & 1]);
        max_fold32(a[cc & 1], mf);
      }
      const float mx = fmaxf(fmaxf(mf[0], mf[1]), fmaxf(mf[2], mf[3]));
      const float neg = -mx * c;
      float sf[4] = {0.f, 0.f, 0.f, 0.f};
      // pass 2: P = 2^(c S - c mx) as bf16 pairs into shared memory (the
      // operand of Y = P [Z | e0] and of dZ += P^T dY')
      tmem_ld32(tR, a[0]);
#pragma unroll
      for (int k = 0; k < NC; ++k) {
        tmem_wait_ld_dep(a[k & 1]);
        if (k + 1 < NC) tmem_ld32(tR + 32 * (k + 1), a[(k + 1) & 1]);
        uint32_t pk[16];
        exp_pack32<0>(a[k & 1], c, neg, pk, sf);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<uint4*>(pbuf + mn_off(r, 4 * k + v)) =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[w]);
      // while Y of tile j runs, finish tile j - 1
      if (j > 0 && !(ok = finish(j - 1, mx_prev, l_prev))) break;
      mx_prev = mx;
      l_prev = (sf[0] + sf[1]) + (sf[2] + sf[3]);
    }
    if (ok && nW > 0) ok = finish(nW - 1, mx_prev, l_prev);
    if (!ok) {
      record_error(err, kErrBwdARowWait);
      *abort_flag = 1;
    }
    // dZ partial of this chunk: warpgroup 0, thread r = latent r
    if (w == 0) {
      float acc[D];
#pragma unroll
      for (int d = 0; d < D; ++d) acc[d] = 0.f;
      if (ok && nt > 0) {
        ok = warp_all(mbar_wait_sleep(dz_final, 0));
        __syncwarp();
        tc_fence_after();
        if (ok) {
          if (D == 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lb + TDZ, o);
            tmem_wait_ld_dep(o);
#pragma unroll
            for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(o[d]);
          } else {
            uint32_t o[16];
            tmem_ld16(tmem + lb + TDZ, o);
            tmem_wait_ld_dep16(o);
#pragma unroll
            for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(o[d & 15]);
          }
        } else {
          record_error(err, kErrBwdARowWait);
          *abort_flag = 1;
        }
      }
      float4* dst = reinterpret_cast<float4*>(dz_part + (cta_slot<VAR>() * M + r) * D);
#pragma unroll
      for (int d = 0; d < D / 4; ++d)
        dst[d] = make_float4(acc[4 * d], acc[4 * d + 1], acc[4 * d + 2], acc[4 * d + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWMma) tmem_dealloc(tmem, NCOLS);
}

// ======================================================= between passes

// One block per (b, h), one thread per latent m: the bf16 copy of Z (the
// operand of Y = P Z and of dY'' Z^T) and R = max_m lse2[m], the reference
// of the split of the encode weights; clears the head's range flag.  With
// lengths, blocks past the heads zero the padding rows of dK and dV, and one
// more block (block 0) computes the work plan of the passes that follow.
template <int D, int M>
__global__ void __launch_bounds__(M)
    bwd_prep_kernel(const float* __restrict__ Z, const float* __restrict__ lse,
                    __nv_bfloat16* __restrict__ zb, float* __restrict__ rref,
                    uint32_t* __restrict__ flags, int64_t BH, const PadZero z,
                    const PlanArgs plan) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  __shared__ float red[M / 32];
  // block 0 computes the work plan with lengths (scheduled first, it runs
  // beside all the others)
  if (plan.on() && blockIdx.x == 0) {
    var_plan_body<M>(plan);
    return;
  }
  const int64_t bx = (int64_t)blockIdx.x - (plan.on() ? 1 : 0);
  if (bx >= BH) {   // the padding rows of dK and dV
    const int64_t x = bx - BH;
    zero_padding_part(z, x % z.nxb, x / z.nxb);
    return;
  }
  const int64_t bh = bx;
  const int m = threadIdx.x;
  const int64_t row = bh * M + m;
#pragma unroll
  for (int d = 0; d < D; d += 4) {
    const float4 v = *reinterpret_cast<const float4*>(Z + row * D + d);
    *reinterpret_cast<uint2*>(zb + row * D + d) = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
  }
  float mx = lse[row] * kLog2e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((m & 31) == 0) red[m >> 5] = mx;
  __syncthreads();
  if (m == 0) {
    float R = red[0];
#pragma unroll
    for (int k = 1; k < M / 32; ++k) R = fmaxf(R, red[k]);
    rref[bh] = R;
    flags[bh] = 0u;
  }
}

// One block per (b, h), kMidLanes(M) threads per latent m, each taking D /
// lanes of its columns.  dZ = sum of the chunk partials (fixed order; the
// work plan's head table locates them when given), lse2 = lse log2(e);
// R = max lse2 over the head; f = 2^(R - lse2) when the head's lse2 spread
// is at most kSpreadMax and no token of it lies more than kRowRangeMax below
// R (else f = 1 and the exact form); the bf16 operand dZ'' = f dZ; the extra
// K-step row: -dZ'' . Z (= -f delta_e) as three bf16 terms, then zeros.
constexpr int kMidThreads = 512;
constexpr int mid_lanes(int M) { return kMidThreads / M; }   // 4 (M = 128) or 2 (M = 256)

template <int D, int M>
__global__ void __launch_bounds__(kMidThreads)
    bwd_mid_kernel(const float* __restrict__ dz_part, int chunks, const int2* __restrict__ heads,
                   const __nv_bfloat16* __restrict__ dz_direct, const float* __restrict__ Z,
                   const float* __restrict__ lse, __nv_bfloat16* __restrict__ dzs,
                   uint32_t* __restrict__ aug, const uint32_t* __restrict__ flags,
                   float2* __restrict__ params, float* __restrict__ lse2_out) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  constexpr int LN = mid_lanes(M);
  constexpr int DL = D / LN;                 // columns of this thread: 4, 8 or 16
  constexpr int NF = DL <= 8 ? 4 : 2;        // partials whose loads are in flight at once
  static_assert(DL % 4 == 0 && M * LN == kMidThreads, "float4 columns, whole rows per block");
  __shared__ float red_max[kMidThreads / 32], red_min[kMidThreads / 32];
  const int64_t bh = blockIdx.x;
  const int m = threadIdx.x / LN, q = threadIdx.x % LN;
  const int64_t row = bh * M + m;
  const int d0 = q * DL;
  float dz[DL];
#pragma unroll
  for (int d = 0; d < DL; ++d) dz[d] = 0.f;
  if (dz_direct) {   // FLARE++'s first encode: dZ1 = dQ_dyn
#pragma unroll
    for (int d = 0; d < DL; ++d) dz[d] = __bfloat162float(dz_direct[row * D + d0 + d]);
  }
  const int2 hs = head_slots(heads, bh, chunks);
  // NF partials' loads in flight at a time, added in partial order
  for (int k = 0; k < hs.y; k += NF) {
    float4 v[NF][DL / 4];
#pragma unroll
    for (int j = 0; j < NF; ++j) {
      const float4* p =
          reinterpret_cast<const float4*>(dz_part + (((int64_t)hs.x + k + j) * M + m) * D + d0);
      if (k + j < hs.y) {
#pragma unroll
        for (int d = 0; d < DL / 4; ++d) v[j][d] = p[d];
      }
    }
#pragma unroll
    for (int j = 0; j < NF; ++j) {
      if (k + j < hs.y) {
#pragma unroll
        for (int d = 0; d < DL / 4; ++d) {
          dz[4 * d] += v[j][d].x;
          dz[4 * d + 1] += v[j][d].y;
          dz[4 * d + 2] += v[j][d].z;
          dz[4 * d + 3] += v[j][d].w;
        }
      }
    }
  }
  const float l2 = lse[row] * kLog2e;
  float mx = l2, mn = l2;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if ((threadIdx.x & 31) == 0) {
    red_max[threadIdx.x >> 5] = mx;
    red_min[threadIdx.x >> 5] = mn;
  }
  __syncthreads();
  float R = red_max[0], lo = red_min[0];
#pragma unroll
  for (int k = 1; k < kMidThreads / 32; ++k) {
    R = fmaxf(R, red_max[k]);
    lo = fminf(lo, red_min[k]);
  }
  const bool fast = (R - lo) <= kSpreadMax && flags[bh] == 0u;
  const float f = fast ? exp2f(R - l2) : 1.f;
  // delta_e is taken with the bf16 operand dZ'' that the tensor cores use,
  // so dPe'' = V dZ''^T - dZ'' . Z vanishes exactly where V = Z.
  float zr[DL];
#pragma unroll
  for (int d = 0; d < DL; d += 4) {
    const float4 zv = *reinterpret_cast<const float4*>(Z + row * D + d0 + d);
    zr[d] = zv.x;
    zr[d + 1] = zv.y;
    zr[d + 2] = zv.z;
    zr[d + 3] = zv.w;
  }
  float de = 0.f;
#pragma unroll
  for (int d = 0; d < DL; d += 2) {
    const uint32_t pr = pack_bf16(f * dz[d], f * dz[d + 1]);
    *reinterpret_cast<uint32_t*>(dzs + row * D + d0 + d) = pr;
    de = fmaf(bf_lo(pr), zr[d], de);
    de = fmaf(bf_hi(pr), zr[d + 1], de);
  }
  // the row's lanes (adjacent threads) add their parts pairwise: every lane
  // ends with the same sum
#pragma unroll
  for (int o = 1; o < LN; o <<= 1) de += __shfl_xor_sync(0xffffffffu, de, o);
  if (q == 0) {
    const float x = -de;
    const __nv_bfloat16 b0 = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(b0);
    const __nv_bfloat16 b1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(b1);
    const __nv_bfloat16 b2 = __float2bfloat16_rn(r2);
    uint32_t* a = aug + row * 8;   // 16 bf16
    a[0] = (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
    a[1] = (uint32_t)__bfloat16_as_ushort(b2);
#pragma unroll
    for (int k = 2; k < 8; ++k) a[k] = 0u;
    lse2_out[row] = l2;
    if (m == 0) params[bh] = make_float2(R, fast ? 1.f : 0.f);
  }
}

// ============================================================== pass B

template <int D>
struct BLayout {
  static constexpr int M = kM;
  static constexpr int NQ = M / 32;           // latent quarters per tile
  static constexpr int RB = 2 * D;
  static constexpr int TILE = kT * RB;
  static constexpr int GBUF = kT * M * 2;     // one G tile, MN-major
  static constexpr int G_OFF = 0;             // two G buffers (tile parity)
  static constexpr int Q_OFF = 2 * GBUF;
  static constexpr int Z_OFF = Q_OFF + M * RB;
  static constexpr int DZ_OFF = Z_OFF + M * RB;
  static constexpr int AUG_OFF = DZ_OFF + M * RB;     // [M][16] bf16, 32-byte rows
  static constexpr int ONES_OFF = AUG_OFF + M * 32;   // [128][16] bf16
  static constexpr int ST_OFF = ONES_OFF + kT * 32;   // stages: K, V, dY tiles
  static constexpr int LSE_OFF = ST_OFF + kBStages * 3 * TILE;
  static constexpr int BAR_OFF = LSE_OFF + M * 4;
  static constexpr int NBARS = 2 * kBStages + 1 + 12 + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
};

template <int D, bool FLAT, bool VAR>
__global__ void __launch_bounds__(kThr, 1)
    tc_bwd_b_exact_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdY,
                    const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmDZ,
                    const __grid_constant__ CUtensorMap tmAug, int H, int64_t N, int q_per_batch,
                    float c, float s, int64_t tiles_per_bh, int64_t chunk_tiles,
                    const float4* __restrict__ stats, const float2* __restrict__ params,
                    const float* __restrict__ lse2, int mode, int m0, int Mt,
                    __nv_bfloat16* __restrict__ dK,
                    __nv_bfloat16* __restrict__ dV, Tok tdk, Tok tdv, float* __restrict__ dq_part,
                    const int32_t* __restrict__ lens, const int4* __restrict__ units,
                    uint32_t* __restrict__ err) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  using L = BLayout<D>;
  constexpr int M = L::M;
  constexpr int NQ = L::NQ;
  constexpr int RB = L::RB;
  constexpr uint32_t SW = umma_swizzle_code(RB);
  constexpr int QC = 96;          // TMEM columns of one quarter: S | dPd | dPe''
  constexpr int TDK = 4 * QC;     // dK accumulator (token lanes)
  constexpr int TDV = TDK + D;    // dV accumulator (token lanes)
  constexpr int TDQ = TDV + D;    // dQ accumulator (latent lanes)
  constexpr uint32_t NCOLS = 512;
  static_assert(TDQ + D <= 512, "TMEM budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  uint64_t* st_full = bars;
  uint64_t* st_empty = bars + kBStages;
  uint64_t* c_full = bars + 2 * kBStages;
  uint64_t* q_full = c_full + 1;     // [slot] a quarter's S, dPd, dPe'' in TMEM
  uint64_t* q_done = q_full + 4;     // [slot] G and the dV weights written
  uint64_t* r_free = q_done + 4;     // [slot] dK/dV MMAs of the quarter complete
  uint64_t* tile_done = r_free + 4;  // dK/dV of a tile final, dQ MMA of the tile complete
  uint64_t* acc_empty = tile_done + 1;
  uint64_t* dq_final = acc_empty + 1;
  uint64_t* drain = dq_final + 1;
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CtaWork cw = cta_work<VAR>(units, chunk_tiles, tiles_per_bh);
  if (cw.bh < 0) return;   // a unit the work plan leaves empty
  const int64_t bh = cw.bh;
  const int64_t h = bh % H;
  const int64_t dk_head = tdk.head(bh, H), dv_head = tdv.head(bh, H);   // row 0 of the head
  const int64_t tile0 = cw.tile0, ntiles = cw.ntiles;
  // with lengths, tokens past the batch element's length are padding: the
  // work plan covers the head's own tiles only
  const HeadTiles<VAR> ht(lens, bh / H, N);
  const int64_t KQ = ntiles * NQ;   // quarters of this chunk
  const bool enc_only = (mode & kModeEncOnly) != 0;   // no decode term
  const bool accum = (mode & kModeAccum) != 0;        // dK, dV added to the rows' values
  if (params[bh].y != 0.f) return;  // head served by tc_bwd_b_fast_kernel

  // the constant A operand of the extra K-step: ones in columns 0-2 of
  // every row, 32-byte swizzle (row t at 32 t, 16-byte chunk x at x ^ bit 2 of t)
  {
    uint8_t* ones = smem + L::ONES_OFF;
    for (int t = threadIdx.x; t < kT; t += blockDim.x) {
      const uint4 one3 = make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
      const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
      const int x0 = 0 ^ ((t >> 2) & 1), x1 = 1 ^ ((t >> 2) & 1);
      *reinterpret_cast<uint4*>(ones + t * 32 + x0 * 16) = one3;
      *reinterpret_cast<uint4*>(ones + t * 32 + x1 * 16) = zero;
    }
    float* ls = (float*)(smem + L::LSE_OFF);
    for (int m = threadIdx.x; m < M; m += blockDim.x) ls[m] = lse2[bh * Mt + m0 + m];
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int k = 0; k < kBStages; ++k) {
      mbar_init(&st_full[k], 1);
      mbar_init(&st_empty[k], 1);
    }
    mbar_init(c_full, 1);
    for (int k = 0; k < 4; ++k) {
      mbar_init(&q_full[k], 1);
      mbar_init(&q_done[k], 128);
      mbar_init(&r_free[k], 1);
    }
    mbar_init(tile_done, 1);
    mbar_init(acc_empty, 256);
    mbar_init(dq_final, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWMma) tmem_alloc(tmem_slot, NCOLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // slot of quarter k: warpgroup k & 1, and each warpgroup alternates two slots
  auto slot_of = [](int64_t k) { return (int)(((k & 1) << 1) | ((k >> 1) & 1)); };

  if (warp >= 8) {
    regs_release<kRegsPro>();
    if (warp == kWTma) {
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdY);
        prefetch_tmap(&tmZ);
        prefetch_tmap(&tmDZ);
        prefetch_tmap(&tmAug);
        mbar_arrive_expect_tx(c_full, 3 * M * RB + M * 32);
        tma_load_3d(smem + L::Q_OFF, &tmQ, c_full, 0, m0, (int32_t)(q_per_batch ? bh : h));
        tma_load_3d(smem + L::Z_OFF, &tmZ, c_full, 0, m0, (int32_t)bh);
        tma_load_3d(smem + L::DZ_OFF, &tmDZ, c_full, 0, m0, (int32_t)bh);
        tma_load_3d(smem + L::AUG_OFF, &tmAug, c_full, 0, m0, (int32_t)bh);
        int64_t issued = 0;
        for (int64_t t = 0; t < ntiles; ++t) {
          const int k = (int)(t % kBStages);
          const uint32_t ph = (uint32_t)((t / kBStages) & 1);
          if (t >= kBStages && !mbar_wait_sleep(&st_empty[k], ph ^ 1)) {
            record_error(err, kErrBwdBTmaWait);
            *abort_flag = 1;
            break;
          }
          if (*abort_flag) break;
          uint8_t* dst = smem + L::ST_OFF + k * 3 * L::TILE;
          mbar_arrive_expect_tx(&st_full[k], 3 * L::TILE);
          const int32_t tok = (int32_t)ht.row0(tile0 + t, kT);
          tma_load_tok<FLAT>(dst, &tmK, &st_full[k], tok, bh, H);
          tma_load_tok<FLAT>(dst + L::TILE, &tmV, &st_full[k], tok, bh, H);
          tma_load_tok<FLAT>(dst + 2 * L::TILE, &tmdY, &st_full[k], tok, bh, H);
          issued = t + 1;
        }
        for (int64_t t = (issued > kBStages ? issued - kBStages : 0); t < issued; ++t)
          mbar_wait_sleep(&st_full[t % kBStages], (uint32_t)((t / kBStages) & 1));
        mbar_wait_sleep(c_full, 0);
      }
    } else if (warp == kWMma) {
      if (lane == 0) {
        constexpr uint32_t idL = idesc_bf16_f32(128, 32, 0, 0);   // quarter logits
        constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);    // dK, dV (A in TMEM)
        constexpr uint32_t idQ = idesc_bf16_f32(128, D, 1, 1);    // dQ (A MN-major)
        const uint32_t q_addr = smem_u32(smem + L::Q_OFF);
        const uint32_t z_addr = smem_u32(smem + L::Z_OFF);
        const uint32_t dz_addr = smem_u32(smem + L::DZ_OFF);
        const uint32_t aug_addr = smem_u32(smem + L::AUG_OFF);
        const uint32_t ones_addr = smem_u32(smem + L::ONES_OFF);
        const uint32_t st0 = smem_u32(smem + L::ST_OFF);
        const uint32_t g0 = smem_u32(smem + L::G_OFF);
        bool ok = mbar_wait_sleep(c_full, 0);
        auto issue_L = [&](int64_t k) -> bool {
          const int64_t t = k / NQ;
          const int qq = (int)(k % NQ);
          const int st = (int)(t % kBStages);
          if (qq == 0 && !mbar_wait_sleep(&st_full[st], (uint32_t)((t / kBStages) & 1)))
            return false;
          tc_fence_after();
          const uint32_t base = tmem + QC * slot_of(k);
          const uint32_t k_addr = st0 + st * 3 * L::TILE;
          const uint32_t v_addr = k_addr + L::TILE;
          const uint32_t dy_addr = k_addr + 2 * L::TILE;
          const uint32_t roff = (uint32_t)(32 * qq * RB);   // latent rows [32 qq, 32 qq + 32)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(base, smem_desc(k_addr + 32 * kk, 16, 8 * RB, SW),
                   smem_desc(q_addr + roff + 32 * kk, 16, 8 * RB, SW), idL, kk > 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(base + 32, smem_desc(dy_addr + 32 * kk, 16, 8 * RB, SW),
                   smem_desc(z_addr + roff + 32 * kk, 16, 8 * RB, SW), idL, kk > 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(base + 64, smem_desc(v_addr + 32 * kk, 16, 8 * RB, SW),
                   smem_desc(dz_addr + roff + 32 * kk, 16, 8 * RB, SW), idL, kk > 0);
          mma_ss(base + 64, smem_desc(ones_addr, 16, 256, kSw32),
                 smem_desc(aug_addr + 32 * qq * 32, 16, 256, kSw32), idL, 1u);
          mma_commit(&q_full[slot_of(k)]);
          return true;
        };
        for (int64_t k = 0; ok && k < 4 && k < KQ; ++k) ok = issue_L(k);
        for (int64_t k = 0; ok && k < KQ; ++k) {
          const int slot = slot_of(k);
          const int64_t t = k / NQ;
          const int qq = (int)(k % NQ);
          const uint32_t use = (uint32_t)((k >> 2) & 1);
          if (!mbar_wait_sleep(&q_done[slot], use)) {
            ok = false;
            break;
          }
          if (qq == 0 && t > 0 && !mbar_wait_sleep(acc_empty, (uint32_t)((t - 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = tmem + QC * slot;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t rows = (uint32_t)((32 * qq + 16 * kk) * RB);
            const uint32_t acc = (qq > 0 || kk > 0) ? 1u : 0u;
            mma_ts(tmem + TDK, base + 8 * kk, smem_desc(q_addr + rows, M * RB, 8 * RB, SW), idO,
                   acc);
            mma_ts(tmem + TDV, base + 32 + 8 * kk, smem_desc(dz_addr + rows, M * RB, 8 * RB, SW),
                   idO, acc);
          }
          mma_commit(&r_free[slot]);
          if (qq == NQ - 1) {
            const int st = (int)(t % kBStages);
            const uint32_t gb = g0 + (uint32_t)((t & 1) * L::GBUF);
            const uint32_t k_addr = st0 + st * 3 * L::TILE;
#pragma unroll
            for (int kk = 0; kk < kT / 16; ++kk)
              mma_ss(tmem + TDQ, smem_desc(gb + kk * kMnKStep, kMnLbo, kMnSbo, kSw128),
                     smem_desc(k_addr + kk * 16 * RB, L::TILE, 8 * RB, SW), idQ,
                     (t > 0 || kk > 0) ? 1u : 0u);
            mma_commit(tile_done);
            mma_commit(&st_empty[st]);
          }
          if (k + 4 < KQ) {
            if (!mbar_wait_sleep(&r_free[slot], use)) {
              ok = false;
              break;
            }
            if (!(ok = issue_L(k + 4))) break;
          }
          if (*abort_flag) ok = false;
        }
        if (!ok) {
          record_error(err, kErrBwdBMmaWait);
          *abort_flag = 1;
        }
        mma_commit(dq_final);
        mma_commit(drain);
        mbar_wait_sleep(drain, 0);
      }
    }
  } else {
    regs_acquire<kRegsRow>();
    const int w = warp >> 2, qw = warp & 3;
    const int r = qw * 32 + lane;                    // TMEM lane = token row of the tile
    const uint32_t lb = (uint32_t)(qw * 32) << 16;
    const float* ls = (const float*)(smem + L::LSE_OFF);
    const uint64_t c2 = f32x2(c, c);
    float mxp = 0.f, dd = 0.f, g = 0.f, gprev = 0.f;
    bool valid = false;
    bool ok = true;

    // dK (warpgroup 0) or dV (warpgroup 1) of tile tt: wait for the tile's
    // accumulators, release them, scale and store the rows.
    auto finish = [&](int64_t tt, float gv) -> bool {
      if (!warp_all(mbar_wait_sleep(tile_done, (uint32_t)(tt & 1)) && !*abort_flag)) return false;
      __syncwarp();
      tc_fence_after();
      float o[D];
      if (D == 32) {
        uint32_t u[32];
        tmem_ld32(tmem + lb + (w == 0 ? TDK : TDV), u);
        tmem_wait_ld_dep(u);
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = __uint_as_float(u[d]);
      } else {
        uint32_t u[16];
        tmem_ld16(tmem + lb + (w == 0 ? TDK : TDV), u);
        tmem_wait_ld_dep16(u);
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = __uint_as_float(u[d & 15]);
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
      const int64_t tok = ht.row0(tile0 + tt, kT) + r;
      if (ht.own(tile0 + tt, kT, r)) {
        const float f = (w == 0) ? s : gv;
        uint4* dst = reinterpret_cast<uint4*>(w == 0 ? dK + dk_head + tok * tdk.sn
                                                     : dV + dv_head + tok * tdv.sn);
        if (accum) {   // added to the gradient already in the rows
#pragma unroll
          for (int v = 0; v < D / 8; ++v) {
            const uint4 q4 = dst[v];
            const uint32_t qq[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              o[8 * v + 2 * jj] = fmaf(o[8 * v + 2 * jj], f, bf_lo(qq[jj]));
              o[8 * v + 2 * jj + 1] = fmaf(o[8 * v + 2 * jj + 1], f, bf_hi(qq[jj]));
            }
          }
        } else {
#pragma unroll
          for (int d = 0; d < D; ++d) o[d] *= f;
        }
#pragma unroll
        for (int v = 0; v < D / 8; ++v)
          dst[v] = make_uint4(pack_bf16(o[8 * v], o[8 * v + 1]), pack_bf16(o[8 * v + 2], o[8 * v + 3]),
                              pack_bf16(o[8 * v + 4], o[8 * v + 5]),
                              pack_bf16(o[8 * v + 6], o[8 * v + 7]));
      }
      return true;
    };

    for (int64_t k = w; k < KQ; k += 2) {
      const int64_t t = k / NQ;
      const int qq = (int)(k % NQ);
      const int slot = slot_of(k);
      if (qq == w) {   // this warpgroup's first quarter of tile t: the row's statistics
        gprev = g;
        // rows that are not the tile's own tokens get G = 0
        const int64_t tok = ht.row0(tile0 + t, kT) + r;
        valid = ht.own(tile0 + t, kT, r);
        if (valid) {
          const float4 st = enc_only ? make_float4(0.f, 0.f, 0.f, 0.f) : stats[bh * N + tok];
          mxp = st.x;
          dd = st.y;
          g = 1.f;
        } else {
          mxp = 0.f;
          dd = 0.f;
          g = 0.f;
        }
      }
      if (!warp_all(mbar_wait_sleep(&q_full[slot], (uint32_t)((k >> 2) & 1)) && !*abort_flag)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      const uint32_t tq = tmem + lb + QC * slot;
      uint8_t* gsm = smem + L::G_OFF + (t & 1) * L::GBUF;
      const uint64_t nm2 = f32x2(-mxp, -mxp), nd2 = f32x2(-dd, -dd);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t a[16], b[16], e[16];
        tmem_ld16(tq + 16 * hh, a);
        tmem_ld16(tq + 32 + 16 * hh, b);
        tmem_ld16(tq + 64 + 16 * hh, e);
        tmem_wait_ld_dep16(a);
        reg_fence16(b);
        reg_fence16(e);
        uint32_t gk[8], vk[8];
        const int m0 = 32 * qq + 16 * hh;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const uint64_t S2 = f32x2(__uint_as_float(a[2 * p]), __uint_as_float(a[2 * p + 1]));
          const uint64_t P2 = f32x2(__uint_as_float(b[2 * p]), __uint_as_float(b[2 * p + 1]));
          const uint64_t E2 = f32x2(__uint_as_float(e[2 * p]), __uint_as_float(e[2 * p + 1]));
          float x0, x1;
          split_f32x2(fma_f32x2(S2, c2, nm2), x0, x1);
          // an encode-only gradient has no decode term: P_d = 0
          // (rows past N have zero K and dY; with lengths a right-aligned
          // tile's earlier rows hold real ones)
          const float p0 = (enc_only || (VAR && !valid)) ? 0.f : ex2(x0);
          const float p1 = (enc_only || (VAR && !valid)) ? 0.f : ex2(x1);
          // exact form: P_e = 2^(c S - lse2[m]); G = P_d (dPd - delta_d) + P_e dPe'
          float s0, s1, e0, e1;
          split_f32x2(S2, s0, s1);
          split_f32x2(E2, e0, e1);
          const float w0 = valid ? ex2(fmaf(s0, c, -ls[m0 + 2 * p])) : 0.f;
          const float w1 = valid ? ex2(fmaf(s1, c, -ls[m0 + 2 * p + 1])) : 0.f;
          float d0, d1;
          split_f32x2(add_f32x2(P2, nd2), d0, d1);
          const float g0v = fmaf(w0, e0, p0 * d0);
          const float g1v = fmaf(w1, e1, p1 * d1);
          gk[p] = pack_bf16(g0v, g1v);
          vk[p] = pack_bf16(w0, w1);
        }
        tmem_st8(tq + 8 * hh, gk);        // over S columns already read
        tmem_st8(tq + 32 + 8 * hh, vk);   // over dPd columns already read
        const int grp = m0 >> 3;
        *reinterpret_cast<uint4*>(gsm + mn_off(r, grp)) = make_uint4(gk[0], gk[1], gk[2], gk[3]);
        *reinterpret_cast<uint4*>(gsm + mn_off(r, grp + 1)) = make_uint4(gk[4], gk[5], gk[6], gk[7]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&q_done[slot]);
      if (qq == w && t > 0 && !(ok = finish(t - 1, gprev))) break;
    }
    if (ok && KQ > 0) ok = finish(ntiles - 1, g);
    if (!ok) {
      record_error(err, kErrBwdBRowWait);
      *abort_flag = 1;
    }
    // dQ partial of this chunk (scaled): warpgroup 0, thread r = latent r
    if (w == 0) {
      float acc[D];
#pragma unroll
      for (int d = 0; d < D; ++d) acc[d] = 0.f;
      if (ok && KQ > 0) {
        ok = warp_all(mbar_wait_sleep(dq_final, 0));
        __syncwarp();
        tc_fence_after();
        if (ok) {
          if (D == 32) {
            uint32_t u[32];
            tmem_ld32(tmem + lb + TDQ, u);
            tmem_wait_ld_dep(u);
#pragma unroll
            for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(u[d]) * s;
          } else {
            uint32_t u[16];
            tmem_ld16(tmem + lb + TDQ, u);
            tmem_wait_ld_dep16(u);
#pragma unroll
            for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(u[d & 15]) * s;
          }
        } else {
          record_error(err, kErrBwdBRowWait);
          *abort_flag = 1;
        }
      }
      float4* dst = reinterpret_cast<float4*>(dq_part + (cta_slot<VAR>() * Mt + m0 + r) * D);
#pragma unroll
      for (int d = 0; d < D / 4; ++d)
        dst[d] = make_float4(acc[4 * d], acc[4 * d + 1], acc[4 * d + 2], acc[4 * d + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWMma) tmem_dealloc(tmem, NCOLS);
}

// ------------------------------------------------- pass B, one-exponential form
//
// For heads whose ranges allow it (params.y = 1): with e = 2^(c S - R),
//   P_d = e / g[n],  P_e = e f[m],
//   G   = e U,  U[n,m] = dY''[n] . Z[m] + V[n] . dZ''[m] - dZ''[m] . Z[m] - delta''[n]
// where dY'' = dY / g (written by pass A), delta'' = dY'' . Y, dZ'' = f dZ.
// The first three terms of U are ONE tensor-core product over a K of
// 2 D + 16 (dY'' | V | ones against Z | dZ'' | -dZ''.Z split in three bf16).
//   dK = s G Q,  dV = e dZ'',  dQ = s G^T K.
// Work unit: half a tile (128 tokens x 64 latents; warpgroup w takes latent
// half w of every tile).  S and U of a half go to one of three TMEM slots;
// the row warps write G and e (bf16) back over the slot's S and U columns,
// where dK += G Q and dV += e dZ'' read them, and G also to shared memory
// (128-byte swizzled, token rows, latents contiguous) for dQ += G^T K.  The
// tensor cores' shared-memory operand traffic bounds this kernel, so every
// operand that can come from TMEM does (G and e for dK / dV, the ones of the
// extra K-step).  Warp 9 keeps the slot ring full; warp 10 issues dK / dV of
// each half (then the slot is refilled) and dQ of each tile.

template <int D>
struct BFLayout {
  static constexpr int M = kM;
  static constexpr int NSLOT = 3;
  static constexpr int KST = 6;                       // K tiles: held until the tile's dQ
  static constexpr int VST = 4;                       // V, dY'' tiles: until its U products
  static constexpr int RB = 2 * D;
  static constexpr int TILE = kT * RB;
  static constexpr int GBUF = kT * M * 2;              // 32 KB
  static constexpr int G_OFF = 0;                      // two G buffers (tile parity)
  static constexpr int Q_OFF = 2 * GBUF;
  static constexpr int Z_OFF = Q_OFF + M * RB;
  static constexpr int DZ_OFF = Z_OFF + M * RB;
  static constexpr int AUG_OFF = DZ_OFF + M * RB;      // [M][16] bf16, 32-byte rows
  static constexpr int K_OFF = AUG_OFF + M * 32;       // K ring
  static constexpr int VD_OFF = K_OFF + KST * TILE;    // (V, dY'') ring
  static constexpr int BAR_OFF = VD_OFF + VST * 2 * TILE;
  static constexpr int NBARS = 2 * KST + 2 * VST + 1 + 3 * NSLOT + 1 + 1 + 1 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
};

template <int D, bool FLAT, bool VAR>
__global__ void __launch_bounds__(kThr, 1)
    tc_bwd_b_fast_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdY2,
                         const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmDZ,
                         const __grid_constant__ CUtensorMap tmAug, int H, int64_t N, int q_per_batch,
                         float c, float s, int64_t tiles_per_bh, int64_t chunk_tiles,
                         const float4* __restrict__ stats, const float2* __restrict__ params,
                         int mode, int m0, int Mt, __nv_bfloat16* __restrict__ dK,
                         __nv_bfloat16* __restrict__ dV, Tok tdk, Tok tdv,
                         float* __restrict__ dq_part, const int32_t* __restrict__ lens,
                         const int4* __restrict__ units, uint32_t* __restrict__ err) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  using L = BFLayout<D>;
  constexpr int M = L::M;
  constexpr int NS = L::NSLOT;
  constexpr int KST = L::KST;
  constexpr int VST = L::VST;
  constexpr int RB = L::RB;
  constexpr uint32_t SW = umma_swizzle_code(RB);
  constexpr int HC = 128;              // TMEM columns of one half slot: S (64) | U (64)
  constexpr int TDK = NS * HC;         // dK accumulator (token lanes)
  constexpr int TDV = TDK + D;         // dV accumulator (token lanes)
  constexpr int TDQ = TDV + D;         // dQ accumulator (latent lanes)
  constexpr int TONE = TDQ + D;        // ones of the extra K-step (8 columns of bf16 pairs)
  constexpr uint32_t NCOLS = 512;
  static_assert(TONE + 8 <= 512, "TMEM budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* c_full = v_empty + VST;
  uint64_t* h_full = c_full + 1;        // [slot] S and U of a half in TMEM
  uint64_t* h_done = h_full + NS;       // [slot] the half's rows read; G, e written back
  uint64_t* r_free = h_done + NS;       // [slot] dK / dV of the half complete: slot free
  uint64_t* tile_done = r_free + NS;    // dK, dV of a tile final; its G buffer free
  uint64_t* acc_empty = tile_done + 1;  // dK, dV accumulators read back
  uint64_t* dq_final = acc_empty + 1;
  uint64_t* drain = dq_final + 1;       // [2]: one per issuing thread
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CtaWork cw = cta_work<VAR>(units, chunk_tiles, tiles_per_bh);
  if (cw.bh < 0) return;   // a unit the work plan leaves empty
  const int64_t bh = cw.bh;
  const int64_t h = bh % H;
  const int64_t dk_head = tdk.head(bh, H), dv_head = tdv.head(bh, H);   // row 0 of the head
  const int64_t tile0 = cw.tile0;
  const int nt = (int)cw.ntiles;
  // with lengths, tokens past the batch element's length are padding: the
  // work plan covers the head's own tiles only
  const HeadTiles<VAR> ht(lens, bh / H, N);
  const float2 prm = params[bh];
  if (prm.y == 0.f) return;   // head served by tc_bwd_b_exact_kernel
  const bool enc_only = (mode & kModeEncOnly) != 0;   // no decode term
  const bool accum = (mode & kModeAccum) != 0;        // dK, dV added to the rows' values

  if (threadIdx.x == 0) {
    for (int k = 0; k < KST; ++k) {
      mbar_init(&k_full[k], 1);
      mbar_init(&k_empty[k], 1);
    }
    for (int k = 0; k < VST; ++k) {
      mbar_init(&v_full[k], 1);
      mbar_init(&v_empty[k], 1);
    }
    mbar_init(c_full, 1);
    for (int k = 0; k < NS; ++k) {
      mbar_init(&h_full[k], 1);
      mbar_init(&h_done[k], 128);
      mbar_init(&r_free[k], 1);
    }
    mbar_init(tile_done, 1);
    mbar_init(acc_empty, 256);
    mbar_init(dq_final, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWMma) tmem_alloc(tmem_slot, NCOLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < 4) {
    // the A operand of the extra K-step: ones in columns 0-2 of every row
    uint32_t one[8] = {0x3F803F80u, 0x00003F80u, 0u, 0u, 0u, 0u, 0u, 0u};
    tmem_st8(tmem + ((uint32_t)(warp * 32) << 16) + TONE, one);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp >= 8) {
    regs_release<kRegsPro>();
    if (warp == kWTma) {
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdY2);
        prefetch_tmap(&tmZ);
        prefetch_tmap(&tmDZ);
        prefetch_tmap(&tmAug);
        mbar_arrive_expect_tx(c_full, 3 * M * RB + M * 32);
        tma_load_3d(smem + L::Q_OFF, &tmQ, c_full, 0, m0, (int32_t)(q_per_batch ? bh : h));
        tma_load_3d(smem + L::Z_OFF, &tmZ, c_full, 0, m0, (int32_t)bh);
        tma_load_3d(smem + L::DZ_OFF, &tmDZ, c_full, 0, m0, (int32_t)bh);
        tma_load_3d(smem + L::AUG_OFF, &tmAug, c_full, 0, m0, (int32_t)bh);
        int issued = 0;
        for (int t = 0; t < nt; ++t) {
          const int32_t tok = (int32_t)ht.row0(tile0 + t, kT);
          const int kb = t % KST, vb = t % VST;
          if (t >= KST && !mbar_wait_sleep(&k_empty[kb], (uint32_t)(((t / KST) & 1) ^ 1))) {
            record_error(err, kErrBwdBTmaWait);
            *abort_flag = 1;
            break;
          }
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&k_full[kb], L::TILE);
          tma_load_tok<FLAT>(smem + L::K_OFF + kb * L::TILE, &tmK, &k_full[kb], tok, bh, H);
          if (t >= VST && !mbar_wait_sleep(&v_empty[vb], (uint32_t)(((t / VST) & 1) ^ 1))) {
            record_error(err, kErrBwdBTmaWait);
            *abort_flag = 1;
            mbar_wait_sleep(&k_full[kb], (uint32_t)((t / KST) & 1));
            break;
          }
          uint8_t* dst = smem + L::VD_OFF + vb * 2 * L::TILE;
          mbar_arrive_expect_tx(&v_full[vb], (enc_only ? 1 : 2) * L::TILE);
          tma_load_tok<FLAT>(dst, &tmV, &v_full[vb], tok, bh, H);
          if (!enc_only) tma_load_3d(dst + L::TILE, &tmdY2, &v_full[vb], 0, tok, (int32_t)bh);
          issued = t + 1;
        }
        // let every load still in flight land before the CTA can exit
        for (int t = (issued > KST ? issued - KST : 0); t < issued; ++t)
          mbar_wait_sleep(&k_full[t % KST], (uint32_t)((t / KST) & 1));
        for (int t = (issued > VST ? issued - VST : 0); t < issued; ++t)
          mbar_wait_sleep(&v_full[t % VST], (uint32_t)((t / VST) & 1));
        mbar_wait_sleep(c_full, 0);
      }
    } else if (warp == kWMma || warp == kWMma + 1) {
      // Two issuing threads: warp 9 keeps the slot ring full (S and U of
      // each half; it waits on TMA tiles), warp 10 issues dK / dV of each
      // half and dQ of each tile (they wait on the row warps).
      if (lane == 0) {
        constexpr uint32_t idH = idesc_bf16_f32(128, 64, 0, 0);   // a half's S or U
        constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);    // dK, dV (A in TMEM)
        constexpr uint32_t idQ = idesc_bf16_f32(128, D, 1, 1);    // dQ (A MN-major)
        const uint32_t q_addr = smem_u32(smem + L::Q_OFF);
        const uint32_t z_addr = smem_u32(smem + L::Z_OFF);
        const uint32_t dz_addr = smem_u32(smem + L::DZ_OFF);
        const uint32_t aug_addr = smem_u32(smem + L::AUG_OFF);
        const uint32_t k0 = smem_u32(smem + L::K_OFF);
        const uint32_t v0 = smem_u32(smem + L::VD_OFF);
        const uint32_t g0 = smem_u32(smem + L::G_OFF);
        // descriptors built once; per MMA only the 14-bit address field
        // moves (offsets >> 4 added; shared addresses stay below 256 KB)
        const uint64_t dK0 = smem_desc(k0, 16, 8 * RB, SW);           // K tile rows, K-major
        const uint64_t dV0 = smem_desc(v0, 16, 8 * RB, SW);           // V / dY'' tile rows
        const uint64_t dQk = smem_desc(q_addr, 16, 8 * RB, SW);       // latent rows, K-major
        const uint64_t dZk = smem_desc(z_addr, 16, 8 * RB, SW);
        const uint64_t dDZk = smem_desc(dz_addr, 16, 8 * RB, SW);
        const uint64_t dAug = smem_desc(aug_addr, 16, 256, kSw32);
        const uint64_t dQm = smem_desc(q_addr, M * RB, 8 * RB, SW);   // latent rows, MN-major
        const uint64_t dDZm = smem_desc(dz_addr, M * RB, 8 * RB, SW);
        const uint64_t dKm = smem_desc(k0, L::TILE, 8 * RB, SW);      // K tile, MN-major
        const uint64_t dGm = smem_desc(g0, kMnLbo, kMnSbo, kSw128);   // G, MN-major
        constexpr uint32_t kTile16 = (uint32_t)L::TILE >> 4;
        constexpr uint32_t kRow16 = (uint32_t)RB;                     // 16 rows >> 4
        constexpr uint32_t kBuf16 = (uint32_t)L::GBUF >> 4;
        const int nh = 2 * nt;
        bool ok = mbar_wait_sleep(c_full, 0);
        // S and U of half k (tile k / 2, latents [64 (k & 1), +64)) into slot k % 3
        auto issue_H = [&](int k) -> bool {
          const int t = k >> 1;
          const int hf = k & 1;
          const int kb = t % KST, vb = t % VST;
          if (hf == 0 && !(mbar_wait_sleep(&k_full[kb], (uint32_t)((t / KST) & 1)) &&
                           mbar_wait_sleep(&v_full[vb], (uint32_t)((t / VST) & 1))))
            return false;
          tc_fence_after();
          const uint32_t base = tmem + HC * (uint32_t)(k % NS);
          const uint32_t ko = (uint32_t)kb * kTile16;
          const uint32_t vo = (uint32_t)(2 * vb) * kTile16;     // V at vo, dY'' at vo + kTile16
          const uint32_t ro = (uint32_t)(64 * hf * RB) >> 4;   // latent rows [64 hf, +64)
          // the S and U chains interleaved, so consecutive MMAs are independent
          // (an encode-only gradient has no dY'' Z^T term)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            mma_ss(base, dK0 + ko + 2 * kk, dQk + ro + 2 * kk, idH, kk > 0);
            if (!enc_only)
              mma_ss(base + 64, dV0 + vo + kTile16 + 2 * kk, dZk + ro + 2 * kk, idH, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(base + 64, dV0 + vo + 2 * kk, dDZk + ro + 2 * kk, idH,
                   (!enc_only || kk > 0) ? 1u : 0u);
          mma_ts(base + 64, tmem + TONE, dAug + (uint32_t)(2 * 64 * hf), idH, 1u);
          mma_commit(&h_full[k % NS]);
          if (hf == 1) mma_commit(&v_empty[vb]);   // V and dY'' of tile t read by both halves
          return true;
        };
        if (warp == kWMma) {
          for (int k = 0; ok && k < NS && k < nh; ++k) ok = issue_H(k);
          for (int k = 0; ok && k + NS < nh; ++k) {
            // dK / dV of half k done: its slot takes half k + 3
            if (!mbar_wait_sleep(&r_free[k % NS], (uint32_t)((k / NS) & 1))) {
              ok = false;
              break;
            }
            if (!(ok = issue_H(k + NS))) break;
            if (*abort_flag) ok = false;
          }
        } else {
          for (int k = 0; ok && k < nh; ++k) {
            const int slot = k % NS;
            const int t = k >> 1;
            const int hf = k & 1;
            if (!mbar_wait_sleep(&h_done[slot], (uint32_t)((k / NS) & 1)) ||
                (hf == 0 && t > 0 && !mbar_wait_sleep(acc_empty, (uint32_t)((t - 1) & 1)))) {
              ok = false;
              break;
            }
            tc_fence_after();
            // dK += G Q, dV += e dZ'' over the half's 64 latents (A from TMEM)
            const uint32_t base = tmem + HC * (uint32_t)slot;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t rows = (uint32_t)(4 * hf + kk) * kRow16;   // latents 64 hf + 16 kk
              const uint32_t acc = (hf > 0 || kk > 0) ? 1u : 0u;
              mma_ts(tmem + TDK, base + 8 * kk, dQm + rows, idO, acc);
              mma_ts(tmem + TDV, base + 64 + 8 * kk, dDZm + rows, idO, acc);
            }
            mma_commit(&r_free[slot]);
            if (hf == 1) {
              // dQ += G^T K over the tile's 128 tokens (G of both halves)
              const uint32_t go = (uint32_t)(t & 1) * kBuf16;
              const uint32_t ko = (uint32_t)(t % KST) * kTile16;
#pragma unroll
              for (int kk = 0; kk < kT / 16; ++kk)
                mma_ss(tmem + TDQ, dGm + go + kk * (kMnKStep >> 4), dKm + ko + kk * kRow16, idQ,
                       (t > 0 || kk > 0) ? 1u : 0u);
              mma_commit(tile_done);
              mma_commit(&k_empty[t % KST]);
            }
            if (*abort_flag) ok = false;
          }
          mma_commit(dq_final);
        }
        if (!ok) {
          record_error(err, kErrBwdBMmaWait);
          *abort_flag = 1;
        }
        mma_commit(drain + (warp - kWMma));
        mbar_wait_sleep(drain + (warp - kWMma), 0);
      }
    }
  } else {
    regs_acquire<kRegsRow>();
    const int w = warp >> 2, qw = warp & 3;
    const int r = qw * 32 + lane;                    // TMEM lane = token row of the tile
    const uint32_t lb = (uint32_t)(qw * 32) << 16;
    const float Rh = prm.x;
    const uint64_t c2 = f32x2(c, c);
    bool ok = true;
    // This thread's token in tile tt, and whether it is one of the tile's
    // own tokens (else e = 0, G = 0 and no store).
    auto row_tok = [&](int tt) -> int64_t { return ht.row0(tile0 + tt, kT) + r; };
    auto own_row = [&](int tt) -> bool { return ht.own(tile0 + tt, kT, r); };
    // delta'' of this thread's row in tile tt, loaded one tile ahead of use
    auto load_dpp = [&](int tt) -> float {
      return (!enc_only && tt < nt && own_row(tt)) ? stats[bh * N + row_tok(tt)].z : 0.f;
    };
    float dpp_next = load_dpp(0);

    // dK (warpgroup 0) or dV (warpgroup 1) of tile tt: wait for the tile's
    // products, read and release the accumulator, scale and store the rows.
    auto finish = [&](int tt) -> bool {
      if (!warp_all(mbar_wait_sleep(tile_done, (uint32_t)(tt & 1)) && !*abort_flag)) return false;
      __syncwarp();
      tc_fence_after();
      float o[D];
      const uint32_t col = (w == 0) ? TDK : TDV;
      if (D == 32) {
        uint32_t u[32];
        tmem_ld32(tmem + lb + col, u);
        tmem_wait_ld_dep(u);
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = __uint_as_float(u[d]);
      } else {
        uint32_t u[16];
        tmem_ld16(tmem + lb + col, u);
        tmem_wait_ld_dep16(u);
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = __uint_as_float(u[d & 15]);
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
      const int64_t tok = row_tok(tt);
      if (own_row(tt)) {
        const float f = (w == 0) ? s : 1.f;
        uint4* dst = reinterpret_cast<uint4*>(w == 0 ? dK + dk_head + tok * tdk.sn
                                                     : dV + dv_head + tok * tdv.sn);
        if (accum) {   // added to the gradient already in the rows
#pragma unroll
          for (int v = 0; v < D / 8; ++v) {
            const uint4 q4 = dst[v];
            const uint32_t qq[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              o[8 * v + 2 * jj] = fmaf(o[8 * v + 2 * jj], f, bf_lo(qq[jj]));
              o[8 * v + 2 * jj + 1] = fmaf(o[8 * v + 2 * jj + 1], f, bf_hi(qq[jj]));
            }
          }
        } else {
#pragma unroll
          for (int d = 0; d < D; ++d) o[d] *= f;
        }
#pragma unroll
        for (int v = 0; v < D / 8; ++v)
          dst[v] = make_uint4(pack_bf16(o[8 * v], o[8 * v + 1]), pack_bf16(o[8 * v + 2], o[8 * v + 3]),
                              pack_bf16(o[8 * v + 4], o[8 * v + 5]),
                              pack_bf16(o[8 * v + 6], o[8 * v + 7]));
      }
      return true;
    };

    for (int t = 0; t < nt; ++t) {
      const int k = 2 * t + w;          // this warpgroup's half of tile t
      const int slot = k % NS;
      const float ndd = -dpp_next;
      const float nR = own_row(t) ? -Rh : -INFINITY;   // not this tile's token: e = 0, G = 0
      dpp_next = load_dpp(t + 1);
      // the row finish(t - 1) adds into: start its load now
      if (accum && t > 0 && own_row(t - 1))
        prefetch_l1(w == 0 ? dK + dk_head + row_tok(t - 1) * tdk.sn
                           : dV + dv_head + row_tok(t - 1) * tdv.sn);
      if (!warp_all(mbar_wait_sleep(&h_full[slot], (uint32_t)((k / NS) & 1)) && !*abort_flag)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      // the G buffer of tile t was last read by tile t - 2's dQ, which
      // completed before this warpgroup's finish(t - 2) returned
      const uint32_t tq = tmem + lb + HC * slot;
      uint8_t* gsm = smem + L::G_OFF + (t & 1) * L::GBUF;
      const uint64_t nR2 = f32x2(nR, nR), nd2 = f32x2(ndd, ndd);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t a[32], u[32];
        tmem_ld32(tq + 32 * cc, a);
        tmem_ld32(tq + 64 + 32 * cc, u);
        tmem_wait_ld_dep(a);
        tmem_wait_ld_dep(u);
        uint32_t gk[16], ek[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          float x0, x1, g0v, g1v;
          split_f32x2(fma_f32x2(f32x2(__uint_as_float(a[2 * p]), __uint_as_float(a[2 * p + 1])), c2,
                                nR2), x0, x1);
          const float e0 = ex2(x0), e1 = ex2(x1);
          split_f32x2(mul_f32x2(f32x2(e0, e1),
                                add_f32x2(f32x2(__uint_as_float(u[2 * p]), __uint_as_float(u[2 * p + 1])),
                                          nd2)),
                      g0v, g1v);
          gk[p] = pack_bf16(g0v, g1v);
          ek[p] = pack_bf16(e0, e1);
        }
        // G over S columns [16 cc, +16) and e over U columns [64 + 16 cc,
        // +16), both already read; G also to shared memory for dQ
        tmem_st16(tq + 16 * cc, gk);
        tmem_st16(tq + 64 + 16 * cc, ek);
        const int grp = 8 * w + 4 * cc;   // latents 64 w + 32 cc, in groups of 8
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<uint4*>(gsm + mn_off(r, grp + v)) =
              make_uint4(gk[4 * v], gk[4 * v + 1], gk[4 * v + 2], gk[4 * v + 3]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&h_done[slot]);
      if (t > 0 && !(ok = finish(t - 1))) break;
    }
    if (ok && nt > 0) ok = finish(nt - 1);
    if (!ok) {
      record_error(err, kErrBwdBRowWait);
      *abort_flag = 1;
    }
    // dQ partial of this chunk (scaled): warpgroup 0, thread r = latent r
    if (w == 0) {
      float acc[D];
#pragma unroll
      for (int d = 0; d < D; ++d) acc[d] = 0.f;
      if (ok && nt > 0) {
        ok = warp_all(mbar_wait_sleep(dq_final, 0));
        __syncwarp();
        tc_fence_after();
        if (ok) {
          if (D == 32) {
            uint32_t u[32];
            tmem_ld32(tmem + lb + TDQ, u);
            tmem_wait_ld_dep(u);
#pragma unroll
            for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(u[d]) * s;
          } else {
            uint32_t u[16];
            tmem_ld16(tmem + lb + TDQ, u);
            tmem_wait_ld_dep16(u);
#pragma unroll
            for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(u[d & 15]) * s;
          }
        } else {
          record_error(err, kErrBwdBRowWait);
          *abort_flag = 1;
        }
      }
      float4* dst = reinterpret_cast<float4*>(dq_part + (cta_slot<VAR>() * Mt + m0 + r) * D);
#pragma unroll
      for (int d = 0; d < D / 4; ++d)
        dst[d] = make_float4(acc[4 * d], acc[4 * d + 1], acc[4 * d + 2], acc[4 * d + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWMma) tmem_dealloc(tmem, NCOLS);
}

// dQ = sum over (batch when Q is shared) x chunks of the scaled partials,
// in a fixed order.  Eight lanes per 4 output elements: with Q shared, lane
// s sums the partials of batch elements s, s + 8, ... (batch outer, chunk
// inner), else those of chunks s, s + 8, ...; the eight sums then combine in
// a butterfly (the same on every lane).  With Q shared, `extra` (if given,
// [B][H][M][D] bf16) is summed over the batch first, by lane 0: FLARE++'s
// dQ_dyn.
constexpr int kDqLanes = 8;

__global__ void bwd_dq_sum_kernel(const float4* __restrict__ dq_part, int B, int H, int M, int D,
                                  int chunks, const int2* __restrict__ heads, bool shared_q,
                                  const __nv_bfloat16* __restrict__ extra,
                                  __nv_bfloat16* __restrict__ dQ, float4* __restrict__ dQ32) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  const int64_t md4 = (int64_t)M * D / 4;
  const int64_t per4 = (int64_t)H * md4;
  const int64_t total4 = shared_q ? per4 : (int64_t)B * per4;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t i = gid / kDqLanes;
  const int s = (int)(gid % kDqLanes);
  // whole warps lie inside or outside the output (total4 is a multiple of 4)
  if (i >= total4) return;
  const int64_t b0 = shared_q ? 0 : i / per4;
  const int64_t rr = i % per4;
  const int64_t h = rr / md4;
  const int64_t e = rr % md4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (extra && shared_q && s == 0) {
    for (int b = 0; b < B; ++b) {
      const uint2 x = *reinterpret_cast<const uint2*>(extra + (b * per4 + i) * 4);
      acc.x += bf_lo(x.x);
      acc.y += bf_hi(x.x);
      acc.z += bf_lo(x.y);
      acc.w += bf_hi(x.y);
    }
  }
  auto add = [&](const float4 v) {
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  };
  if (shared_q) {
    for (int64_t b = s; b < B; b += kDqLanes) {
      const int2 hs = head_slots(heads, b * H + h, chunks);
      int k = 0;
      for (; k + 4 <= hs.y; k += 4) {   // four loads in flight
        const float4 v0 = dq_part[((int64_t)hs.x + k) * md4 + e];
        const float4 v1 = dq_part[((int64_t)hs.x + k + 1) * md4 + e];
        const float4 v2 = dq_part[((int64_t)hs.x + k + 2) * md4 + e];
        const float4 v3 = dq_part[((int64_t)hs.x + k + 3) * md4 + e];
        add(v0);
        add(v1);
        add(v2);
        add(v3);
      }
      for (; k < hs.y; ++k) add(dq_part[((int64_t)hs.x + k) * md4 + e]);
    }
  } else {
    const int2 hs = head_slots(heads, b0 * H + h, chunks);
    for (int k = s; k < hs.y; k += kDqLanes) add(dq_part[((int64_t)hs.x + k) * md4 + e]);
  }
#pragma unroll
  for (int o = 1; o < kDqLanes; o <<= 1) {
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
  }
  if (s != 0) return;
  if (dQ32)
    dQ32[i] = acc;
  else
    *reinterpret_cast<uint2*>(dQ + i * 4) = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
}

// This device's dZ: the fixed-order sum over chunks of pass A's partials,
// [BH][chunks][M][D] -> [BH][M][D].  One thread per 4 elements.
__global__ void bwd_dz_sum_kernel(const float4* __restrict__ dz_part, int64_t BH, int M, int D,
                                  int chunks, const int2* __restrict__ heads,
                                  float4* __restrict__ dz) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  const int64_t md4 = (int64_t)M * D / 4;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BH * md4) return;
  const int64_t bh = i / md4, e = i % md4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int2 hs = head_slots(heads, bh, chunks);
  for (int k = 0; k < hs.y; ++k) {
    const float4 v = dz_part[((int64_t)hs.x + k) * md4 + e];
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  dz[i] = acc;
}

// M = 128: pass A (tc_bwd_a_kernel) gives the per-token statistics and the
// dZ partials in one pass.  M = 256: an S row of 256 latents per token does
// not fit pass A's TMEM and shared-memory layout, so the decode stage runs
// as two passes of the forward's pipelines -- the decode kernel with the
// statistics in place of Y, then the encode kernel with dY as V and the
// per-token weights P_d = 2^(c S - mx') -- and pass B runs once per half of
// the latents (the encode weights and G of a latent depend on it and on the
// per-token statistics alone), the second half adding into dK and dV.
template <int D, int M, bool FLAT, bool VAR>
cudaError_t tc_bwd_t(const void* Q, int64_t qbs, const void* K, const void* V, const void* dY,
                     const float* Z, const float* lse, void* dQ, void* dK, void* dV, const Dims& d,
                     float scale, const WsLayout& L, char* ws, cudaStream_t st, BwdPhase phase,
                     float* dz_io, float* dq32, const PadZero* pz, const PlanArgs* plan) {
  const ChunkPlan& p = L.bwd;
  const int64_t BH = d.BH();
  const int q_per_batch = qbs != 0;
  const float c = scale * kLog2e;
  uint32_t* err = (uint32_t*)(ws + L.hdr);
  __nv_bfloat16* zb = (__nv_bfloat16*)(ws + L.zb);
  float4* stats = (float4*)(ws + L.stats);
  __nv_bfloat16* dy2 = (__nv_bfloat16*)(ws + L.dy2);
  float* rref = (float*)(ws + L.rref);
  uint32_t* flags = (uint32_t*)(ws + L.flags);
  float* dzp = (float*)(ws + L.dzp);
  __nv_bfloat16* dzs = (__nv_bfloat16*)(ws + L.dzs);
  __nv_bfloat16* aug = (__nv_bfloat16*)(ws + L.aug);
  float2* params = (float2*)(ws + L.params);
  float* lse2 = (float*)(ws + L.lse2);
  float* dqp = (float*)(ws + L.dqp);
  const int zchunks = (M == kM) ? p.chunks : L.enc.slots_per_bh();   // dZ partials per head
  // with lengths: the work plans' head tables locate the partials
  const int2* zheads = VAR ? ((M == kM) ? d.vtok.heads : d.venc.heads) : nullptr;
  const int2* qheads = VAR ? d.vtok.heads : nullptr;
  cudaError_t e;

  if (phase != BwdPhase::FINISH) {
    // with lengths, the work plan is computed by one more block (M = 128
    // reads the 128-token plan only)
    const PadZero z = pz ? *pz : PadZero{};
    PlanArgs pa = plan ? *plan : PlanArgs{};
    if (M == kM) pa.k0.units = nullptr;
    const int64_t blocks = BH + z.blocks(BH) + (pa.on() ? 1 : 0);
    bwd_prep_kernel<D, M><<<(unsigned)blocks, M, 0, st>>>(Z, lse, zb, rref, flags, BH, z, pa);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  } else if (plan) {
    if ((e = launch_plan(*plan, st)) != cudaSuccess) return e;
  }

  // latent operands: M rows per head, loaded 128 rows at a time
  CUtensorMap mq, mk, mv, mdy, mdy2, mz, mdz, maug;
  if ((e = make_map(&mq, Q, D, M, q_per_batch ? BH : d.H, kM)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mk, K, d, d.k, kT, FLAT)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mv, V, d, d.v, kT, FLAT)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mdy, dY, d, d.dy, kT, FLAT)) != cudaSuccess) return e;
  if ((e = make_map(&mdy2, dy2, D, d.N, BH, kT)) != cudaSuccess) return e;
  if ((e = make_map(&mz, zb, D, M, BH, kM)) != cudaSuccess) return e;
  if ((e = make_map(&mdz, dzs, D, M, BH, kM)) != cudaSuccess) return e;
  if ((e = make_map(&maug, aug, 16, M, BH, kM)) != cudaSuccess) return e;

  // with lengths: one CTA per unit of the 128-token work plan
  const dim3 grid = VAR ? dim3((unsigned)d.vtok.n) : dim3(p.chunks, (unsigned)BH);
  if (phase != BwdPhase::FINISH) {
    if constexpr (M == kM) {
      const int smemA = ALayout<D>::BYTES + 1024;
      e = cudaFuncSetAttribute(tc_bwd_a_kernel<D, FLAT, VAR>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smemA);
      if (e != cudaSuccess) return e;
      tc_bwd_a_kernel<D, FLAT, VAR><<<grid, kThr, smemA, st>>>(
          mq, mk, mdy, mz, (int)d.H, d.N, q_per_batch, c, p.tiles_per_bh, p.chunk_tiles, rref,
          stats, dy2, flags, dzp, d.lens, d.vtok.units, err);
      if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    } else {
      if ((e = launch_tc_bwd_stats(Q, qbs, K, zb, dY, d, scale, L.dec, rref, stats, dy2, flags,
                                   err, st)) != cudaSuccess)
        return e;
      if ((e = launch_tc_dz(Q, qbs, K, dY, d, scale, L.enc, stats, dzp, err, st)) != cudaSuccess)
        return e;
    }
    if (phase == BwdPhase::DZ) {   // this device's part of dZ
      const int64_t n4 = BH * M * D / 4;
      bwd_dz_sum_kernel<<<(unsigned)((n4 + 127) / 128), 128, 0, st>>>(
          (const float4*)dzp, BH, M, D, zchunks, zheads, (float4*)dz_io);
      return cudaPeekAtLastError();
    }
  }

  // dZ: the chunk partials, or (FINISH) the sum over the shards as one partial
  const bool fin = phase == BwdPhase::FINISH;
  bwd_mid_kernel<D, M><<<(unsigned)BH, kMidThreads, 0, st>>>(
      fin ? dz_io : dzp, fin ? 1 : zchunks, fin ? nullptr : zheads, nullptr, Z, lse, dzs,
      (uint32_t*)aug, flags, params, lse2);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;

  // each head runs in exactly one of the two pass-B kernels (params.y)
  const int smemF = BFLayout<D>::BYTES + 1024;
  e = cudaFuncSetAttribute(tc_bwd_b_fast_kernel<D, FLAT, VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smemF);
  if (e != cudaSuccess) return e;
  const int smemB = BLayout<D>::BYTES + 1024;
  e = cudaFuncSetAttribute(tc_bwd_b_exact_kernel<D, FLAT, VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smemB);
  if (e != cudaSuccess) return e;
  for (int m0 = 0; m0 < M; m0 += kM) {
    const int mode = (m0 > 0) ? kModeAccum : 0;
    tc_bwd_b_fast_kernel<D, FLAT, VAR><<<grid, kThr, smemF, st>>>(
        mq, mk, mv, mdy2, mz, mdz, maug, (int)d.H, d.N, q_per_batch, c, scale, p.tiles_per_bh,
        p.chunk_tiles, stats, params, mode, m0, M, (__nv_bfloat16*)dK, (__nv_bfloat16*)dV, d.dk,
        d.dv, dqp, d.lens, d.vtok.units, err);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    tc_bwd_b_exact_kernel<D, FLAT, VAR><<<grid, kThr, smemB, st>>>(
        mq, mk, mv, mdy, mz, mdz, maug, (int)d.H, d.N, q_per_batch, c, scale, p.tiles_per_bh,
        p.chunk_tiles, stats, params, lse2, mode, m0, M, (__nv_bfloat16*)dK, (__nv_bfloat16*)dV,
        d.dk, d.dv, dqp, d.lens, d.vtok.units, err);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  }

  const bool shared_q = (qbs == 0);
  const int64_t total = shared_q ? d.H * M * D : BH * M * D;
  bwd_dq_sum_kernel<<<(unsigned)((total / 4 * kDqLanes + 127) / 128), 128, 0, st>>>(
      (const float4*)dqp, (int)d.B, (int)d.H, M, D, p.chunks, qheads, shared_q, nullptr,
      (__nv_bfloat16*)dQ, (float4*)dq32);
  return cudaPeekAtLastError();
}

// FLARE++'s first encode, Z1 = softmax_N(s Q K^T) V with Q shared over the
// batch, differentiated with upstream dZ1 = dQ_dyn: the pass-B kernels in
// their encode-only form (no decode term; dK, dV added to the rows that
// FLARE's backward wrote), once per half of the latents with M = 256, then
// dQ = sum over b of (dQ_dyn + the encode's partials).  Runs after FLARE's
// backward on the same stream and reuses its workspace.
template <int D, int M, bool FLAT, bool VAR>
cudaError_t tc_enc_bwd_t(const void* Q, const void* K, const void* V, const float* Z1,
                         const float* lse1, const void* dZ1, void* dQ, void* dK, void* dV,
                         const Dims& d, float scale, const WsLayout& L, char* ws, cudaStream_t st,
                         float* dq32, bool add_dz1) {
  const ChunkPlan& p = L.bwd;
  const int64_t BH = d.BH();
  const float c = scale * kLog2e;
  uint32_t* err = (uint32_t*)(ws + L.hdr);
  __nv_bfloat16* zb = (__nv_bfloat16*)(ws + L.zb);
  float4* stats = (float4*)(ws + L.stats);
  float* rref = (float*)(ws + L.rref);
  uint32_t* flags = (uint32_t*)(ws + L.flags);
  __nv_bfloat16* dzs = (__nv_bfloat16*)(ws + L.dzs);
  __nv_bfloat16* aug = (__nv_bfloat16*)(ws + L.aug);
  float2* params = (float2*)(ws + L.params);
  float* lse2 = (float*)(ws + L.lse2);
  float* dqp = (float*)(ws + L.dqp);
  cudaError_t e;

  // bf16 Z1 and a cleared range flag (no decode, so no token can raise it)
  bwd_prep_kernel<D, M><<<(unsigned)BH, M, 0, st>>>(Z1, lse1, zb, rref, flags, BH, PadZero{},
                                                    PlanArgs{});
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  bwd_mid_kernel<D, M><<<(unsigned)BH, kMidThreads, 0, st>>>(
      nullptr, 0, nullptr, (const __nv_bfloat16*)dZ1, Z1, lse1, dzs, (uint32_t*)aug, flags, params,
      lse2);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;

  // the decode operands' maps point at V: valid tiles that are never used
  CUtensorMap mq, mk, mv, mz, mdz, maug;
  if ((e = make_map(&mq, Q, D, M, d.H, kM)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mk, K, d, d.k, kT, FLAT)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mv, V, d, d.v, kT, FLAT)) != cudaSuccess) return e;
  if ((e = make_map(&mz, zb, D, M, BH, kM)) != cudaSuccess) return e;
  if ((e = make_map(&mdz, dzs, D, M, BH, kM)) != cudaSuccess) return e;
  if ((e = make_map(&maug, aug, 16, M, BH, kM)) != cudaSuccess) return e;

  // with lengths: one CTA per unit of the 128-token work plan
  const dim3 grid = VAR ? dim3((unsigned)d.vtok.n) : dim3(p.chunks, (unsigned)BH);
  const int smemF = BFLayout<D>::BYTES + 1024;
  e = cudaFuncSetAttribute(tc_bwd_b_fast_kernel<D, FLAT, VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smemF);
  if (e != cudaSuccess) return e;
  const int smemB = BLayout<D>::BYTES + 1024;
  e = cudaFuncSetAttribute(tc_bwd_b_exact_kernel<D, FLAT, VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smemB);
  if (e != cudaSuccess) return e;
  for (int m0 = 0; m0 < M; m0 += kM) {
    tc_bwd_b_fast_kernel<D, FLAT, VAR><<<grid, kThr, smemF, st>>>(
        mq, mk, mv, mv, mz, mdz, maug, (int)d.H, d.N, 0, c, scale, p.tiles_per_bh, p.chunk_tiles,
        stats, params, kModeEncOnly | kModeAccum, m0, M, (__nv_bfloat16*)dK, (__nv_bfloat16*)dV,
        d.dk, d.dv, dqp, d.lens, d.vtok.units, err);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    tc_bwd_b_exact_kernel<D, FLAT, VAR><<<grid, kThr, smemB, st>>>(
        mq, mk, mv, mv, mz, mdz, maug, (int)d.H, d.N, 0, c, scale, p.tiles_per_bh, p.chunk_tiles,
        stats, params, lse2, kModeEncOnly | kModeAccum, m0, M, (__nv_bfloat16*)dK,
        (__nv_bfloat16*)dV, d.dk, d.dv, dqp, d.lens, d.vtok.units, err);
    if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  }

  const int64_t total = d.H * M * D;
  bwd_dq_sum_kernel<<<(unsigned)((total / 4 * kDqLanes + 127) / 128), 128, 0, st>>>(
      (const float4*)dqp, (int)d.B, (int)d.H, M, D, p.chunks, VAR ? d.vtok.heads : nullptr, true,
      (dq32 && !add_dz1) ? nullptr : (const __nv_bfloat16*)dZ1, (__nv_bfloat16*)dQ,
      (float4*)dq32);
  return cudaPeekAtLastError();
}

template <int D, int M>
cudaError_t tc_bwd_dispatch(const void* Q, int64_t qbs, const void* K, const void* V,
                            const void* dY, const float* Z, const float* lse, void* dQ, void* dK,
                            void* dV, const Dims& d, float scale, const WsLayout& L, char* ws,
                            cudaStream_t st, BwdPhase ph, float* dz, float* dq32,
                            const PadZero* pz, const PlanArgs* plan) {
  const bool flat = tok_flat(d), var = d.lens != nullptr;
#define FLARE_TC_BWD_T(F, V_)                                                                   \
  tc_bwd_t<D, M, F, V_>(Q, qbs, K, V, dY, Z, lse, dQ, dK, dV, d, scale, L, ws, st, ph, dz, dq32, \
                        pz, plan)
  if (flat) return var ? FLARE_TC_BWD_T(true, true) : FLARE_TC_BWD_T(true, false);
  return var ? FLARE_TC_BWD_T(false, true) : FLARE_TC_BWD_T(false, false);
#undef FLARE_TC_BWD_T
}

template <int D, int M>
cudaError_t tc_enc_bwd_dispatch(const void* Q, const void* K, const void* V, const float* Z1,
                                const float* lse1, const void* dZ1, void* dQ, void* dK, void* dV,
                                const Dims& d, float scale, const WsLayout& L, char* ws,
                                cudaStream_t st, float* dq32, bool add_dz1) {
  const bool flat = tok_flat(d), var = d.lens != nullptr;
#define FLARE_TC_ENC_T(F, V_) \
  tc_enc_bwd_t<D, M, F, V_>(Q, K, V, Z1, lse1, dZ1, dQ, dK, dV, d, scale, L, ws, st, dq32, add_dz1)
  if (flat) return var ? FLARE_TC_ENC_T(true, true) : FLARE_TC_ENC_T(true, false);
  return var ? FLARE_TC_ENC_T(false, true) : FLARE_TC_ENC_T(false, false);
#undef FLARE_TC_ENC_T
}

}  // namespace

cudaError_t launch_tc_bwd(const void* Q, int64_t qbs, const void* K, const void* V,
                          const void* dY, const float* Z, const float* lse, void* dQ, void* dK,
                          void* dV, const Dims& d, float scale, const WsLayout& L, char* ws,
                          cudaStream_t st, BwdPhase phase, float* dz, float* dq32,
                          const PadZero* pz, const PlanArgs* plan) {
#define FLARE_TC_BWD(D_, M_)                                                                  \
  tc_bwd_dispatch<D_, M_>(Q, qbs, K, V, dY, Z, lse, dQ, dK, dV, d, scale, L, ws, st, phase, dz, \
                          dq32, pz, plan)
  if (d.D == 32 && d.M == 128) return FLARE_TC_BWD(32, 128);
  if (d.D == 32 && d.M == 256) return FLARE_TC_BWD(32, 256);
  if (d.D == 16 && d.M == 128) return FLARE_TC_BWD(16, 128);
  if (d.D == 16 && d.M == 256) return FLARE_TC_BWD(16, 256);
#undef FLARE_TC_BWD
  return cudaErrorNotSupported;
}

cudaError_t launch_tc_enc_bwd(const void* Q, const void* K, const void* V, const float* Z1,
                              const float* lse1, const void* dZ1, void* dQ, void* dK, void* dV,
                              const Dims& d, float scale, const WsLayout& L, char* ws,
                              cudaStream_t st, float* dq32, bool add_dz1) {
#define FLARE_TC_ENC(D_, M_) \
  tc_enc_bwd_dispatch<D_, M_>(Q, K, V, Z1, lse1, dZ1, dQ, dK, dV, d, scale, L, ws, st, dq32, add_dz1)
  if (d.D == 32 && d.M == 128) return FLARE_TC_ENC(32, 128);
  if (d.D == 32 && d.M == 256) return FLARE_TC_ENC(32, 256);
  if (d.D == 16 && d.M == 128) return FLARE_TC_ENC(16, 128);
  if (d.D == 16 && d.M == 256) return FLARE_TC_ENC(16, 256);
#undef FLARE_TC_ENC
  return cudaErrorNotSupported;
}

}  // namespace flare
