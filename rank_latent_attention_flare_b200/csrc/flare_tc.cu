// Tensor-core FLARE forward for sm_100a: tcgen05.mma with TMEM accumulators,
// operands staged in shared memory by TMA, softmax on the CUDA cores with one
// TMEM lane (one row) per thread.
//
// Encode, per (b, h) and chunk of tokens ("Flare Fast Low Rank Attention"
// skill page, section 2, latents as queries), for every 48-token tile:
//   S = Q K_tile^T            (tcgen05, M=128 latents x N=48 tokens x K=D)
//   P = 2^(c S - m_ref)       (row = latent, running reference with lazy rescale)
//   O += P V_tile             (tcgen05, A = P from TMEM, B = V from smem)
// and at the end of the chunk the record (m_ref, l = row sum of P, O) goes to
// the workspace for the log-sum-exp combine.  Two CTAs share an SM.
// Decode (FLARE arXiv abstract, second SDPA call), for every 128-token tile:
//   S = K_tile Q^T            (M=128 tokens x N=M latents x K=D)
//   P = 2^(c S - ref)         (row = token, whole row in one thread)
//   Y = (P Z) / rowsum(P)     (A = P from TMEM, B = Z from smem)
// so the N x M logits never leave the SM.  One CTA per SM.
//
// The tensor-core backward with M = 256 reuses both pipelines (template
// flags): the decode with the backward's per-token statistics in place of Y
// (ST), and the encode with dY in place of V and fixed per-token weights in
// place of the online softmax (DZ), which gives dZ = P_d^T dY.
//
// Roles per CTA (384 threads, twelve warps):
//   encode -- warps 0-3 and 4-7 are two softmax warpgroups; warp 8 issues the
//     TMA loads; warps 9 and 10 issue the MMAs of softmax warpgroup 0 and 1
//     (one elected lane each; warp 9 also owns TMEM); warp 11 only lends its
//     registers.  Launched at 80 registers per thread, the producer
//     warpgroup moves to 56 and the softmax warpgroups to 88
//     (2 x 128 x 88 + 128 x 56 <= 384 x 80).
//   decode -- the same softmax warpgroups (alternate tiles), warp 8 TMA,
//     warp 9 TMEM and MMAs, warps 10-11 bound each K tile's row maxima
//     (M = 256).  Launched at 168 registers per thread: the producer
//     warpgroup moves to 104 and the softmax warpgroups to 200.
// Exponentials use ex2.approx (MUFU) with c = scale * log2(e) folded in;
// a fixed share of them runs as a polynomial on the FMA pipe instead.
#include <cudaTypedefs.h>

#include "flare_internal.cuh"
#include "tc_primitives.cuh"

namespace flare {
namespace {

using namespace tc;

// The MMA-issuing threads poll their barriers instead of sleeping between
// polls: the decode's tile chain (Y, then the next S) runs through them
// twice per tile, and a suspended poll added about 8% to its time.
#define MMA_WAIT mbar_wait

constexpr int kTile = 128;        // tokens per tile (MMA M or N)
constexpr int kThreads = 384;
constexpr int kRegsSoftmax = 200;
constexpr int kRegsProducer = 104;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpNorm = 10;   // decode: warps 10 and 11 bound the row max of alternate K tiles
// Slots of the decode's bound ring.  The norm warp fills tile i's slot only
// after the TMA load of tile i, which waits for the S product of tile i - 6,
// which waits for the row warps to finish tile i - 8's S; so 16 slots are
// never refilled before the row warps have read them.
constexpr int kDecBoundSlots = 16;
constexpr int kEncStages = 8;
constexpr int kDecStages = 6;
constexpr float kRescaleTau = 8.0f;   // log2 units: rescale only when the max grows by > 2^8
constexpr float kRedoTau = 64.0f;     // log2 units: past 2^64 above m_ref a tile is recomputed
constexpr float kRescaleLimit = 256.0f;                  // 2^kRescaleTau
constexpr float kRedoLimit = 18446744073709551616.0f;   // 2^kRedoTau
// Every k-th pair of exponentials is computed on the FMA pipe (exp2_fma)
// instead of the MUFU, which is the unit that bounds both kernels.  On the
// million-token workload the encode (four softmax warps per SM
// sub-partition) is fastest with every third pair (5 of 16 and 2 of 8 per
// 48-logit row tile: 1.23 -> 1.21 ms against every fourth; every second is
// 1.37 ms), the decode with every eighth pair of each 32-logit chunk (1.19 ->
// 1.16 ms against the last pair only, once its row sums came from Y's
// product and freed FMA-pipe issue slots; every fifth or fourth pair measured
// the same within noise, and fewer polynomials keep more weights at the
// MUFU's accuracy).
// Decode reference of a token row (M = 256): the max of the first 32-logit
// chunk read, used when c |k| max_m |q_m| (Cauchy-Schwarz: at least every
// logit) lies at most this far (log2 units) above it, so no weight exceeds
// 2^kDecRefTau; else the exact row max (a second pass over the row).  With
// M = 128 the second pass is short and the exact max is always taken.
constexpr float kDecRefTau = 64.f;
constexpr int kMinSmemBytes = 120 * 1024;  // keeps one CTA (and its TMEM) per SM

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// Multiplies this thread's row of a D-column fp32 TMEM accumulator by f.
template <int D>
__device__ __forceinline__ void scale_tmem_row(uint32_t taddr, float f) {
  if (D == 32) {
    uint32_t o[32];
    tmem_ld32(taddr, o);
    tmem_wait_ld_dep(o);
    uint32_t lo[16], hi[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      lo[t] = __float_as_uint(__uint_as_float(o[t]) * f);
      hi[t] = __float_as_uint(__uint_as_float(o[16 + t]) * f);
    }
    tmem_st16(taddr, lo);
    tmem_st16(taddr + 16, hi);
  } else {
    uint32_t o[16];
    tmem_ld16(taddr, o);
    tmem_wait_ld();
#pragma unroll
    for (int t = 0; t < 16; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * f);
    tmem_st16(taddr, o);
  }
}

// ============================================================== encode
//
// Tiles of kEncTile = 48 tokens; two CTAs share an SM (256 TMEM columns and
// an 80-register launch each), so four softmax warpgroups per SM hide each
// other's latencies.  Softmax warpgroup w owns TMEM columns
// [128w, 128w + 128): two 48-column S buffers at 128w + 48b (b = 0, 1), whose
// first 24 columns receive the tile's P (bf16 pairs) once S has been read,
// and the O accumulator at 128w + 96.  While the softmax works on one
// buffer, the MMA fills the other with the next tile's logits.  With M = 256
// warpgroup w owns latent rows [128w, 128w + 128) of every tile; with M = 128
// the warpgroups take alternate tiles, each with its own running record.

constexpr int kEncTile = 48;
constexpr int kEncRegsSoftmax = 88, kEncRegsProducer = 56;   // 256 x 88 + 128 x 56 <= 384 x 80

template <int D, int M, bool DZ = false>
struct EncLayout {
  static constexpr int RB = 2 * D;                  // bytes per row (one token or latent)
  static constexpr int TILE = kEncTile * RB;        // one K or V tile
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = M * RB;
  static constexpr int BAR_OFF = KV_OFF + kEncStages * 2 * TILE;
  static constexpr int NBARS = 2 * kEncStages + 1 + 4 + 4 + 4 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  // dZ form: per stage, the tile's column offsets (kEncTile floats)
  static constexpr int NB_OFF = MISC_OFF + 16;
  static constexpr int BYTES = DZ ? NB_OFF + kEncStages * kEncTile * 4 : MISC_OFF + 16;
};

// p = 2^(c a + nb) for NP consecutive pairs of logits, nb per column (a
// float pair from shared memory): bf16 pairs into pk.  With POLY_EVERY = k
// > 0, every k-th pair on the FMA pipe.
template <int NP, int POLY_EVERY>
__device__ __forceinline__ void exp_bias_pairs(const uint32_t* a, float c, const float* nb,
                                               uint32_t* pk) {
  const uint64_t c2 = f32x2(c, c);
#pragma unroll
  for (int t = 0; t < NP; ++t) {
    const uint64_t b2 = *reinterpret_cast<const uint64_t*>(nb + 2 * t);
    float x0, x1;
    split_f32x2(fma_f32x2(f32x2(__uint_as_float(a[2 * t]), __uint_as_float(a[2 * t + 1])), c2, b2),
                x0, x1);
    const bool poly = POLY_EVERY > 0 && (t % (POLY_EVERY > 0 ? POLY_EVERY : 1)) == POLY_EVERY - 1;
    if (poly) {
      float p0, p1;
      exp2_fma_pair(f32x2(x0, x1), p0, p1);
      pk[t] = pack_bf16(p0, p1);
    } else {
      pk[t] = pack_bf16(ex2(x0), ex2(x1));
    }
  }
}

// DZ = true: the same pipeline computes the decode stage's dZ = P_d^T dY of
// the backward (latents as rows, tV := dY): the weights of token n are
// P_d[n,m] = 2^(c S[m,n] - mx'[n]), mx'[n] the decode log-sum-exp (log2
// units) in stats[n].x, so no running max, rescale or row sum is needed
// (P_d <= 1); the record is the accumulator alone.
template <int D, int M, bool FLAT, bool VAR, bool DZ>
__global__ void __launch_bounds__(kThreads, 2)
    tc_encode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, int H, int64_t N, int q_per_batch,
                     int Mv, float c, int64_t tiles_per_bh, int64_t chunk_tiles,
                     float* __restrict__ part_ml, float* __restrict__ part_acc,
                     const int32_t* __restrict__ lens, const int4* __restrict__ units,
                     const float4* __restrict__ stats, uint32_t* __restrict__ err) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  using L = EncLayout<D, M, DZ>;
  constexpr int NH = M / 128;        // latent halves; M=128 -> the two warpgroups split tiles
  constexpr int SUB = (NH == 1) ? 2 : 1;
  constexpr int RB = L::RB;
  constexpr uint32_t SW = umma_swizzle_code(RB);
  constexpr uint32_t TM_COLS = 256;
  constexpr int stride = (NH == 2) ? 1 : 2;   // tile step of one warpgroup

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* Qs = smem + L::Q_OFF;
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kEncStages;
  uint64_t* q_full = bars + 2 * kEncStages;
  uint64_t* s_full = q_full + 1;      // [2w + b]: S written by the MMA
  uint64_t* sp_done = s_full + 4;     // [2w + b]: S read and P written by the softmax
  uint64_t* pv_done = sp_done + 4;    // [2w + b]: P.V of a tile from buffer b complete
  uint64_t* drain = pv_done + 4;      // [w]
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CtaWork cw = cta_work<VAR>(units, chunk_tiles, tiles_per_bh);
  if (cw.bh < 0) return;   // a unit the work plan leaves empty
  const int64_t bh = cw.bh;
  const int64_t h = bh % H;
  const int64_t tile0 = cw.tile0, ntiles = cw.ntiles;
  // with lengths, tokens past the batch element's length are padding: the
  // work plan covers the head's own tiles only
  const HeadTiles<VAR> ht(lens, bh / H, N);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kEncStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], NH == 2 ? 2 : 1);   // one release per warpgroup reading the tile
    }
    mbar_init(q_full, 1);
    for (int k = 0; k < 4; ++k) {
      mbar_init(&s_full[k], 1);
      mbar_init(&sp_done[k], 128);
      mbar_init(&pv_done[k], 1);
    }
    for (int k = 0; k < 2; ++k) mbar_init(&drain[k], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) tmem_alloc(tmem_slot, TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_release<kEncRegsProducer>();
    if (DZ && warp == kWarpTma) {
      // ------------------------------------ TMA producer, dZ form (whole warp)
      // Each stage also carries the tile's column offsets -mx'[n] (-inf for
      // columns that are not the tile's own tokens), stored by the warp's
      // lanes before lane 0 arms the stage's barrier.
      float* nb_ring = (float*)(smem + L::NB_OFF);
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        mbar_arrive_expect_tx(q_full, M * RB);
        const int32_t qz = (int32_t)(q_per_batch ? bh : h);
        for (int half = 0; half < NH; ++half)
          tma_load_3d(Qs + half * 128 * RB, &tmQ, q_full, 0, half * 128, qz);
      }
      // The offsets of tile i are loaded kNbAhead tiles before they are
      // stored (lane l: columns l and l + 32), so the loads' latency is not
      // on the producer's path; the loop is unrolled by kNbAhead so that
      // each tile's values stay in fixed registers.
      constexpr int kNbAhead = 4;
      auto load_nb = [&](int i, float (&v)[2]) {
        if (i >= (int)ntiles) return;
        const int64_t tok = ht.row0(tile0 + i, kEncTile);
        const int lo = ht.lo(tile0 + i, kEncTile), hi = ht.hi(tile0 + i, kEncTile);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int t = lane + 32 * k;
          v[k] = (t < kEncTile && t >= lo && t < hi) ? -stats[bh * N + tok + t].x : -INFINITY;
        }
      };
      float pre[kNbAhead][2];
#pragma unroll
      for (int u = 0; u < kNbAhead; ++u) load_nb(u, pre[u]);
      int issued = 0;
      bool stopped = false;
      for (int i0 = 0; i0 < (int)ntiles && !stopped; i0 += kNbAhead) {
#pragma unroll
        for (int u = 0; u < kNbAhead; ++u) {
          const int i = i0 + u;
          if (i >= (int)ntiles) break;
          const int s = i % kEncStages;
          const uint32_t ph = (uint32_t)((i / kEncStages) & 1);
          int stop = 0;
          if (lane == 0) {
            if (i >= kEncStages && !mbar_wait_sleep(&kv_empty[s], ph ^ 1)) {
              record_error(err, kErrEncTmaWait);
              *abort_flag = 1;
            }
            stop = *abort_flag;
          }
          if (__shfl_sync(0xffffffffu, stop, 0)) {
            stopped = true;
            break;
          }
          float* nb = nb_ring + s * kEncTile;
          nb[lane] = pre[u][0];
          if (lane + 32 < kEncTile) nb[lane + 32] = pre[u][1];
          load_nb(i + kNbAhead, pre[u]);
          __syncwarp();
          if (lane == 0) {
            const int64_t tok = ht.row0(tile0 + i, kEncTile);
            uint8_t* kt = smem + L::KV_OFF + s * 2 * L::TILE;
            mbar_arrive_expect_tx(&kv_full[s], 2 * L::TILE);
            tma_load_tok<FLAT>(kt, &tmK, &kv_full[s], (int32_t)tok, bh, H);
            tma_load_tok<FLAT>(kt + L::TILE, &tmV, &kv_full[s], (int32_t)tok, bh, H);
          }
          issued = i + 1;
        }
      }
      if (lane == 0) {
        for (int i = (issued > kEncStages ? issued - kEncStages : 0); i < issued; ++i)
          mbar_wait_sleep(&kv_full[i % kEncStages], (uint32_t)((i / kEncStages) & 1));
        mbar_wait_sleep(q_full, 0);
      }
    } else if (warp == kWarpTma) {
      // ---------------------------------------------------- TMA producer
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        mbar_arrive_expect_tx(q_full, M * RB);
        const int32_t qz = (int32_t)(q_per_batch ? bh : h);
        for (int half = 0; half < NH; ++half)
          tma_load_3d(Qs + half * 128 * RB, &tmQ, q_full, 0, half * 128, qz);
        int issued = 0;
        for (int i = 0; i < (int)ntiles; ++i) {
          const int s = i % kEncStages;
          const uint32_t ph = (uint32_t)((i / kEncStages) & 1);
          if (i >= kEncStages && !mbar_wait_sleep(&kv_empty[s], ph ^ 1)) {
            record_error(err, kErrEncTmaWait);
            *abort_flag = 1;
            break;
          }
          if (*abort_flag) break;
          uint8_t* kt = smem + L::KV_OFF + s * 2 * L::TILE;
          mbar_arrive_expect_tx(&kv_full[s], 2 * L::TILE);
          const int32_t tok = (int32_t)ht.row0(tile0 + i, kEncTile);
          tma_load_tok<FLAT>(kt, &tmK, &kv_full[s], tok, bh, H);
          tma_load_tok<FLAT>(kt + L::TILE, &tmV, &kv_full[s], tok, bh, H);
          issued = i + 1;
        }
        // let every load still in flight land before the CTA can exit
        for (int i = (issued > kEncStages ? issued - kEncStages : 0); i < issued; ++i)
          mbar_wait_sleep(&kv_full[i % kEncStages], (uint32_t)((i / kEncStages) & 1));
        mbar_wait_sleep(q_full, 0);
      }
    } else if (warp == kWarpMma || warp == kWarpMma + 1) {
      // -------------------------------------- MMA issuers, one per warpgroup
      // Warp 9 serves softmax warpgroup 0 and warp 10 warpgroup 1.  For the
      // warpgroup's j-th tile (buffer b = j % 2): P.V once the softmax has
      // finished it; then, once that P.V has completed (it reads P from
      // buffer b), the S of tile j + 2 into the same buffer.
      if (lane == 0) {
        const int w = warp - kWarpMma;
        constexpr uint32_t idS = idesc_bf16_f32(128, kEncTile, 0, 0);
        constexpr uint32_t idPV = idesc_bf16_f32(128, D, 0, 1);
        const int nw = (NH == 2) ? (int)ntiles : (int)((ntiles - w + 1) / 2);
        const int first = (NH == 2) ? 0 : w;
        // descriptors built once; per stage / k-step only the address field moves
        const uint32_t kv0 = smem_u32(smem + L::KV_OFF);
        const uint64_t dQ = smem_desc(smem_u32(Qs) + (NH == 2 ? w * 128 * RB : 0), 16, 8 * RB, SW);
        const uint64_t dK = smem_desc(kv0, 16, 8 * RB, SW);
        const uint64_t dV = smem_desc(kv0 + L::TILE, L::TILE, 8 * RB, SW);
        const uint32_t tW = tmem + 128 * w;
        bool ok = mbar_wait_sleep(q_full, 0);
        auto issue_S = [&](int j) -> bool {
          const int i = first + stride * j;
          const int s = i % kEncStages;
          if (!mbar_wait_sleep(&kv_full[s], (uint32_t)((i / kEncStages) & 1))) return false;
          tc_fence_after();
          const uint32_t koff = (uint32_t)(s * 2 * L::TILE) >> 4;
          const int b = j & 1;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tW + 48 * b, dQ + 2 * kk, dK + koff + 2 * kk, idS, kk > 0);
          mma_commit(&s_full[2 * w + b]);
          return true;
        };
        for (int j = 0; ok && j < 2 && j < nw; ++j) ok = issue_S(j);
        for (int j = 0; ok && j < nw; ++j) {
          const int b = j & 1;
          if (!MMA_WAIT(&sp_done[2 * w + b], (uint32_t)((j >> 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int i = first + stride * j;
          const uint32_t voff = (uint32_t)((i % kEncStages) * 2 * L::TILE) >> 4;
#pragma unroll
          for (int kk = 0; kk < kEncTile / 16; ++kk)
            mma_ts(tW + 96, tW + 48 * b + 8 * kk, dV + voff + ((uint32_t)(kk * 16 * RB) >> 4),
                   idPV, (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&pv_done[2 * w + b]);
          mma_commit(&kv_empty[i % kEncStages]);
          if (j + 2 < nw) {
            // buffer b still holds the P this P.V reads: wait for it to finish
            if (!MMA_WAIT(&pv_done[2 * w + b], (uint32_t)((j >> 1) & 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (!(ok = issue_S(j + 2))) break;
          }
          if (*abort_flag) ok = false;
        }
        if (!ok) {
          record_error(err, kErrEncMmaWait);
          *abort_flag = 1;
        }
        mma_commit(drain + w);
        mbar_wait_sleep(drain + w, 0);
      }
    }
  } else {
    // ------------------------------------------------------ softmax warpgroups
    regs_acquire<kEncRegsSoftmax>();
    const int w = warp >> 2, q = warp & 3;
    const int r = q * 32 + lane;                     // TMEM lane = latent row in the half
    const uint32_t lb = (uint32_t)(q * 32) << 16;
    const uint32_t tW = tmem + lb + 128 * w;
    const uint32_t tO = tW + 96;
    const int nW = (NH == 2) ? (int)ntiles : (int)((ntiles - w + 1) / 2);
    const int first = (NH == 2) ? 0 : w;
    float mref = -INFINITY, l = 0.f;
    float pend = 1.f;   // factor O still owes to a move of m_ref
    bool ok = true;
    // P.V of this warpgroup's tile jj (and, by issue order, of every earlier
    // one) has completed.  Each S buffer has its own barrier: with one
    // barrier per warpgroup a waiter two phases behind would read the
    // wrong parity as complete.
    auto pv_wait = [&](int jj) -> bool {
      return mbar_wait(&pv_done[2 * w + (jj & 1)], (uint32_t)((jj >> 1) & 1));
    };
    // Waits for the previous tile's P.V (O stable) and multiplies O by g.
    auto scale_O = [&](int j, float g) -> bool {
      if (!warp_any(g != 1.f)) return true;
      if (j > 0) {
        if (!warp_all(pv_wait(j - 1))) return false;
        __syncwarp();
        tc_fence_after();
      }
      scale_tmem_row<D>(tO, g);   // rows without a rescale multiply by 1
      return true;
    };
    if constexpr (DZ) {
      const float* nb_ring = (const float*)(smem + L::NB_OFF);
      for (int j = 0; j < nW; ++j) {
        const int64_t i = first + (int64_t)stride * j;
        const int b = j & 1;
        const int s = (int)(i % kEncStages);
        const uint32_t tS = tW + 48 * b;
        // the tile's S in TMEM, and its stage (with the column offsets) landed
        if (!warp_all(mbar_wait(&s_full[2 * w + b], (uint32_t)((j >> 1) & 1)) &&
                      mbar_wait(&kv_full[s], (uint32_t)((i / kEncStages) & 1)) && !*abort_flag)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const float* nb = nb_ring + s * kEncTile;
        {
          uint32_t a[32], pk[16];
          tmem_ld32(tS, a);
          tmem_wait_ld_dep(a);
          exp_bias_pairs<16, enc_poly_every32(M)>(a, c, nb, pk);
          tmem_st16(tS, pk);
        }
        {
          uint32_t a[16], pk[8];
          tmem_ld16(tS + 32, a);
          tmem_wait_ld_dep16(a);
          exp_bias_pairs<8, enc_poly_every16(M)>(a, c, nb + 32, pk);
          tmem_st8(tS + 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sp_done[2 * w + b]);
      }
    }
    for (int j = 0; !DZ && j < nW; ++j) {
      const int64_t i = first + (int64_t)stride * j;
      const int b = j & 1;
      // the tile's own tokens are its columns [lo, hi); the rest get weight 0
      const int lo = ht.lo(tile0 + i, kEncTile), hi = ht.hi(tile0 + i, kEncTile);
      const bool full = (lo == 0 && hi == kEncTile);   // warp-uniform: only a head's last tile is partial
      const uint32_t tS = tW + 48 * b;
      if (!warp_all(mbar_wait(&s_full[2 * w + b], (uint32_t)((j >> 1) & 1)) && !*abort_flag)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      // Optimistic single pass (every tile after a warpgroup's first): P is
      // taken against the running reference m_ref and stays in registers
      // until the overflow check below passes.
      bool exact = warp_any(mref == -INFINITY);
      if (!exact) {
        const float neg = -mref;
        float sf[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pa[16], pb[8];
        {
          uint32_t a[32];
          tmem_ld32(tS, a);
          tmem_wait_ld_dep(a);
          if (!full) {   // masked columns get weight 0
#pragma unroll
            for (int t = 0; t < 32; ++t)
              if (t < lo || t >= hi) a[t] = __float_as_uint(-INFINITY);
          }
          exp_pack32<enc_poly_every32(M), true>(a, c, neg, pa, sf);
        }
        {
          uint32_t a[16];
          tmem_ld16(tS + 32, a);
          tmem_wait_ld_dep16(a);
          if (!full) {
#pragma unroll
            for (int t = 0; t < 16; ++t)
              if (32 + t < lo || 32 + t >= hi) a[t] = __float_as_uint(-INFINITY);
          }
          exp_pack16<enc_poly_every16(M), true>(a, c, neg, pb, sf);
        }
        const float sum = (sf[0] + sf[1]) + (sf[2] + sf[3]);
        // Every weight of the tile is at most the tile's row sum, so the sum
        // stands in for the max: above 2^kRedoTau (or not finite) a weight
        // may have overflowed and the tile is recomputed with the exact max;
        // above 2^kRescaleTau the reference moves up by log2(sum), which
        // keeps it within log2(tile) of the running max.
        if (warp_any(!(sum <= kRedoLimit))) {
          exact = true;
        } else {
          if (!scale_O(j, pend)) {   // a rescale decided after the previous tile
            ok = false;
            break;
          }
          pend = 1.f;
          tmem_st16(tS, pa);          // P over S columns already read
          tmem_st8(tS + 16, pb);
          if (sum > kRescaleLimit) {
            const float mx2 = mref + lg2(sum);
            pend = ex2(mref - mx2);
            l = (l + sum) * pend;
            mref = mx2;
          } else {
            l += sum;
          }
        }
      }
      if (exact) {
        // pass 1: exact tile max of the raw logits (masked columns excluded)
        float mf[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        {
          uint32_t a[32];
          tmem_ld32(tS, a);
          tmem_wait_ld_dep(a);
#pragma unroll
          for (int t = 0; t < 32; ++t)
            if (t >= lo && t < hi) mf[t & 3] = fmaxf(mf[t & 3], __uint_as_float(a[t]));
        }
        {
          uint32_t a[16];
          tmem_ld16(tS + 32, a);
          tmem_wait_ld_dep16(a);
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (32 + t >= lo && 32 + t < hi) mf[t & 3] = fmaxf(mf[t & 3], __uint_as_float(a[t]));
        }
        const float mx2 = fmaxf(fmaxf(mf[0], mf[1]), fmaxf(mf[2], mf[3])) * c;
        float f = 1.f;   // rescale of this row's earlier tiles (1 when the max did not move)
        if (mx2 > mref) {
          if (mref != -INFINITY) f = ex2(mref - mx2);
          mref = mx2;
        }
        l *= f;
        if (!scale_O(j, pend * f)) {
          ok = false;
          break;
        }
        pend = 1.f;
        // pass 2: P = 2^(c S - m_ref) as bf16 pairs, and its row sum; chunk
        // 0's P lands on S columns [0, 16) and chunk 1's on [16, 24), both
        // already read.
        const float neg = -mref;
        float sf[4] = {0.f, 0.f, 0.f, 0.f};
        {
          uint32_t a[32];
          tmem_ld32(tS, a);
          tmem_wait_ld_dep(a);
          if (!full) {
#pragma unroll
            for (int t = 0; t < 32; ++t)
              if (t < lo || t >= hi) a[t] = __float_as_uint(-INFINITY);
          }
          uint32_t pk[16];
          exp_pack32<enc_poly_every32(M), true>(a, c, neg, pk, sf);
          tmem_st16(tS, pk);
        }
        {
          uint32_t a[16];
          tmem_ld16(tS + 32, a);
          tmem_wait_ld_dep16(a);
          if (!full) {
#pragma unroll
            for (int t = 0; t < 16; ++t)
              if (32 + t < lo || 32 + t >= hi) a[t] = __float_as_uint(-INFINITY);
          }
          uint32_t pk[8];
          exp_pack16<enc_poly_every16(M), true>(a, c, neg, pk, sf);
          tmem_st8(tS + 16, pk);
        }
        l += (sf[0] + sf[1]) + (sf[2] + sf[3]);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sp_done[2 * w + b]);
    }
    float acc[D];
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = 0.f;
    if (ok && nW > 0) {
      ok = warp_all(pv_wait(nW - 1));
      __syncwarp();
      tc_fence_after();
      if (ok) {
        if (D == 32) {
          uint32_t o[32];
          tmem_ld32(tO, o);
          tmem_wait_ld_dep(o);
#pragma unroll
          for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(o[d]) * pend;
        } else {
          uint32_t o[16];
          tmem_ld16(tO, o);
          tmem_wait_ld_dep16(o);
#pragma unroll
          for (int d = 0; d < D; ++d) acc[d] = __uint_as_float(o[d & 15]) * pend;
        }
      }
    }
    if (!ok) {
      record_error(err, kErrEncSoftmaxWait);
      *abort_flag = 1;
    } else {
      // latent rows past Mv are the zero rows that pad the latents to the
      // MMA's 128-row tiles: computed alongside, never stored
      const int lat = (NH == 2 ? w * 128 : 0) + r;
      if (lat < Mv) {
        const int64_t slot = cta_slot<VAR>() * SUB + (NH == 1 ? w : 0);
        const int64_t row = slot * Mv + lat;
        if (!DZ) {
          part_ml[row * 2 + 0] = (nW > 0) ? mref : -INFINITY;
          part_ml[row * 2 + 1] = l;
        }
        float4* dst = reinterpret_cast<float4*>(part_acc + row * D);
#pragma unroll
        for (int d = 0; d < D / 4; ++d)
          dst[d] = make_float4(acc[4 * d], acc[4 * d + 1], acc[4 * d + 2], acc[4 * d + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, TM_COLS);
}

// ============================================================== decode

template <int D, int M>
struct DecLayout {
  static constexpr int RB = 2 * D;
  static constexpr int TILE = kTile * RB;
  static constexpr int Q_OFF = 0;
  static constexpr int Z_OFF = M * RB;
  // bf16 ones in Z's layout, right after Z: the second N-atom of Y's B
  // operand [Z | 1], so Y's product also gives each row's weight sum
  static constexpr int ONES_OFF = 2 * M * RB;
  static constexpr int K_OFF = 3 * M * RB;
  static constexpr int BAR_OFF = K_OFF + kDecStages * TILE;
  static constexpr int NBARS = 2 * kDecStages + 1 + 4 * 2 + 1 + kDecBoundSlots + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int QN_OFF = MISC_OFF + 16;              // [M] float: |q_m|^2
  static constexpr int KN_OFF = QN_OFF + M * 4;             // [slot][kTile] float: bound U
  static constexpr int BYTES = KN_OFF + kDecBoundSlots * kTile * 4;
};

// The backward's decode statistics (ST = true): in place of Y, every token
// row gets its decode log-sum-exp mx' (log2 units), delta_d = dY . Y and
// delta'' = dY'' . Y with dY'' = bf16(dY / g), g = 2^(mx' - R) (R per
// head), and dY'' itself; a row with g below 2^-kBwdRowRange flags its head
// (the head then takes the backward's exact form).
struct DecStats {
  const __nv_bfloat16* dY;
  Tok tdy;
  const float* rref;     // [BH] R
  float4* stats;         // [BH][N] (mx', delta_d, delta'', 0)
  __nv_bfloat16* dy2;    // [BH][N][D] dY''
  uint32_t* flags;       // [BH]
};

// PAD = true: the latent count Mv (a multiple of 16) is below the kernel's
// M (128 or 256); the Q and Z tiles past row Mv are the TMA's zero fill,
// their logit columns are skipped (never exponentiated, no MMA K-step), and
// every row takes the exact max over its Mv logits.
template <int D, int M, bool FLAT, bool VAR, bool ST, bool PAD = false>
__global__ void __launch_bounds__(kThreads, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmZ, int H, int64_t N, int q_per_batch,
                     int Mv, float c, int64_t tiles_per_bh, int64_t chunk_tiles,
                     __nv_bfloat16* __restrict__ Y, Tok ty, const __nv_bfloat16* __restrict__ Qg,
                     const int32_t* __restrict__ lens, const int4* __restrict__ units,
                     const DecStats bs, uint32_t* __restrict__ err) {
  pdl_wait();   // the previous kernel's results (programmatic dependent launch)
  pdl_trigger();
  using L = DecLayout<D, M>;
  constexpr int RB = L::RB;
  constexpr uint32_t SW = umma_swizzle_code(RB);
  // first-chunk reference under the row-max bound (measured no faster with
  // M = 128, whose exact two-pass row is short)
  constexpr bool kBound = (M == 256) && !PAD;
  // TMEM columns per warpgroup: S (M fp32 columns, P written over the ones
  // already read) and the accumulator [Y | l] (D + 16 columns, l = the row's
  // weight sum in its first column): inside S's upper half with M = 256
  // (columns 128-175, below the upper P at 192), past S with M = 128.
  constexpr int R = 256;
  constexpr uint32_t NCOLS = 2 * R;
  constexpr int TY = (M == 256) ? M / 2 : M;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* Qs = smem + L::Q_OFF;
  uint8_t* Zs = smem + L::Z_OFF;
  uint64_t* bars = (uint64_t*)(smem + L::BAR_OFF);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + kDecStages;
  uint64_t* qz_full = bars + 2 * kDecStages;
  uint64_t* s_full = qz_full + 1;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* y_full = p_full + 2;
  uint64_t* drain = y_full + 2;
  uint64_t* kn_full = drain + 1;   // [slot]: the tile's row bounds written
  // [2w + q]: the P of the first chunks of the warpgroup's tile written
  // (q = 0: the upper half of the latents; q = 1, M = 256: then latents 0-63)
  uint64_t* p_part = kn_full + kDecBoundSlots;
  float* kn = (float*)(smem + L::KN_OFF);
  uint32_t* tmem_slot = (uint32_t*)(smem + L::MISC_OFF);
  volatile int* abort_flag = (volatile int*)(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CtaWork cw = cta_work<VAR>(units, chunk_tiles, tiles_per_bh);
  if (cw.bh < 0) return;   // a unit the work plan leaves empty
  const int64_t bh = cw.bh;
  const int64_t h = bh % H;
  const int64_t yhead = ty.head(bh, H);   // row 0 of this head in Y
  const int64_t tile0 = cw.tile0, ntiles = cw.ntiles;
  // with lengths, tokens past the batch element's length are padding: the
  // work plan covers the head's own tiles only
  const HeadTiles<VAR> ht(lens, bh / H, N);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&k_full[s], 1);
      // released by the S product's commit (and the bound warp, done reading)
      mbar_init(&k_empty[s], kBound ? 2 : 1);
    }
    for (int s = 0; s < kDecBoundSlots; ++s) {
      mbar_init(&kn_full[s], 32);
    }
    mbar_init(qz_full, 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&s_empty[w], 128);
      mbar_init(&p_full[w], 128);
      mbar_init(&y_full[w], 1);
      mbar_init(&p_part[2 * w], 128);
      mbar_init(&p_part[2 * w + 1], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (kBound) {
    // |q_m|^2 of this head's latents, for the bound on each token's row max
    const __nv_bfloat16* qh = Qg + (q_per_batch ? bh : h) * (int64_t)M * D;
    float* qn2 = (float*)(smem + L::QN_OFF);
    for (int m = threadIdx.x; m < M; m += blockDim.x) {
      float acc = 0.f;
#pragma unroll
      for (int v = 0; v < D / 8; ++v) {
        const uint4 u = reinterpret_cast<const uint4*>(qh + (int64_t)m * D)[v];
        const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          acc = fmaf(bf_lo(uu[jj]), bf_lo(uu[jj]), fmaf(bf_hi(uu[jj]), bf_hi(uu[jj]), acc));
      }
      qn2[m] = acc;
    }
  }
  {
    // the ones of Y's B operand (bf16 1.0, in Z's layout after Z)
    uint4* ones = reinterpret_cast<uint4*>(smem + L::ONES_OFF);
    for (int i = threadIdx.x; i < M * RB / 16; i += blockDim.x)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) tmem_alloc(tmem_slot, NCOLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_release<kRegsProducer>();
    if (warp == kWarpTma) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmZ);
      mbar_arrive_expect_tx(qz_full, 2 * M * RB);
      tma_load_3d(Qs, &tmQ, qz_full, 0, 0, (int32_t)(q_per_batch ? bh : h));
      tma_load_3d(Zs, &tmZ, qz_full, 0, 0, (int32_t)bh);
      int64_t issued = 0;
      for (int64_t i = 0; i < ntiles; ++i) {
        const int s = (int)(i % kDecStages);
        const uint32_t ph = (uint32_t)((i / kDecStages) & 1);
        if (i >= kDecStages && !mbar_wait_sleep(&k_empty[s], ph ^ 1)) {
          record_error(err, kErrDecTmaWait);
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&k_full[s], L::TILE);
        tma_load_tok<FLAT>(smem + L::K_OFF + s * L::TILE, &tmK, &k_full[s],
                           (int32_t)ht.row0(tile0 + i, kTile), bh, H);
        issued = i + 1;
      }
      for (int64_t i = (issued > kDecStages ? issued - kDecStages : 0); i < issued; ++i)
        mbar_wait_sleep(&k_full[i % kDecStages], (uint32_t)((i / kDecStages) & 1));
      mbar_wait_sleep(qz_full, 0);
    }
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, M, 0, 0);
      constexpr uint32_t idY = idesc_bf16_f32(128, D + 16, 0, 1);   // N = [Z | 1]
      const uint32_t q_addr = smem_u32(Qs);
      const uint32_t z_addr = smem_u32(Zs);
      bool ok = mbar_wait_sleep(qz_full, 0);
      auto issue_S = [&](int64_t i) -> bool {
        const int w = (int)(i & 1);
        const int64_t j = i >> 1;
        const int s = (int)(i % kDecStages);
        if (!mbar_wait_sleep(&k_full[s], (uint32_t)((i / kDecStages) & 1))) return false;
        if (j > 0 && !MMA_WAIT(&s_empty[w], (uint32_t)((j - 1) & 1))) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + L::K_OFF + s * L::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + w * R, smem_desc(k_addr + 32 * kk, 16, 8 * RB, SW),
                 smem_desc(q_addr + 32 * kk, 16, 8 * RB, SW), idS, kk > 0);
        mma_commit(&s_full[w]);
        mma_commit(&k_empty[s]);
        return true;
      };
      // K-steps [k0, k1) of Y = P Z (16 latents each); the first one issued
      // (k0 = kfirst) starts the accumulator
      auto y_steps = [&](int w, int k0, int k1, int kfirst) {
#pragma unroll
        for (int kk = 0; kk < M / 16; ++kk) {
          if (kk < k0 || kk >= k1) continue;
          if (PAD && 16 * kk >= Mv) break;   // latents past Mv: no K-step
          const uint32_t acol = (kk < M / 32) ? 8 * kk : M / 2 + 8 * kk;
          mma_ts(tmem + w * R + TY, tmem + w * R + acol,
                 smem_desc(z_addr + kk * 16 * RB, M * RB, 8 * RB, SW), idY, kk != kfirst);
        }
      };
      // Y of tile i in step with its softmax: the upper half of the latents
      // (whose chunks the row warps process first, and which hold Y's
      // columns) once they are written, then the lower half (in two parts
      // with M = 256), so little of the product is left when the last P lands.
      auto issue_Y = [&](int64_t i) -> bool {
        const int w = (int)(i & 1);
        const uint32_t ph = (uint32_t)((i >> 1) & 1);
        if constexpr (PAD) {
          if (!MMA_WAIT(&p_full[w], ph)) return false;
          tc_fence_after();
          y_steps(w, 0, M / 16, 0);
        } else {
          if (!MMA_WAIT(&p_part[2 * w], ph)) return false;
          tc_fence_after();
          y_steps(w, M / 32, M / 16, M / 32);
          if (M == 256) {
            if (!MMA_WAIT(&p_part[2 * w + 1], ph)) return false;
            tc_fence_after();
            y_steps(w, 0, 4, -1);
          }
          if (!MMA_WAIT(&p_full[w], ph)) return false;
          tc_fence_after();
          y_steps(w, M == 256 ? 4 : 0, M / 32, -1);
        }
        mma_commit(&y_full[w]);
        return true;
      };
      if (ok && ntiles > 0) ok = issue_S(0);
      if (ok && ntiles > 1) ok = issue_S(1);
      for (int64_t i = 0; ok && i < ntiles; ++i) {
        ok = issue_Y(i);
        if (ok && i + 2 < ntiles) ok = issue_S(i + 2);
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        record_error(err, kErrDecMmaWait);
        *abort_flag = 1;
      }
      mma_commit(drain);
      mbar_wait_sleep(drain, 0);
    }
    } else if (kBound && (warp == kWarpNorm || warp == kWarpNorm + 1)) {
      // The bound U = c |k| max_m |q_m| >= c S[m] on every row of each K tile
      // (the swizzle only permutes a row's 16-byte pieces; rows outside the
      // head's tokens were filled with zeros).
      float qmax2 = 0.f;
      {
        const float4* qn2 = (const float4*)(smem + L::QN_OFF);
        for (int m = 0; m < M / 4; ++m) {
          const float4 v = qn2[m];
          qmax2 = fmaxf(qmax2, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
        }
      }
      bool ok = true;
      for (int64_t i = warp - kWarpNorm; i < ntiles; i += 2) {
        const int s = (int)(i % kDecStages);
        const int slot = (int)(i % kDecBoundSlots);
        if (!warp_all(mbar_wait_sleep(&k_full[s], (uint32_t)((i / kDecStages) & 1)) &&
                      !*abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* kt = smem + L::K_OFF + s * L::TILE;
#pragma unroll
        for (int rr = lane; rr < kTile; rr += 32) {
          uint64_t kq[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
          for (int v = 0; v < D / 8; ++v) {
            const uint4 u = reinterpret_cast<const uint4*>(kt + rr * RB)[v];
            const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const uint64_t p = f32x2(bf_lo(uu[jj]), bf_hi(uu[jj]));
              kq[jj & 1] = fma_f32x2(p, p, kq[jj & 1]);
            }
          }
          float q0, q1, q2, q3;
          split_f32x2(kq[0], q0, q1);
          split_f32x2(kq[1], q2, q3);
          kn[slot * kTile + rr] = c * sqrtf(((q0 + q1) + (q2 + q3)) * qmax2);
        }
        mbar_arrive(&kn_full[slot]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&k_empty[s]);
      }
      if (!ok) {
        record_error(err, kErrDecTmaWait);
        *abort_flag = 1;
      }
    }
  } else {
    regs_acquire<kRegsSoftmax>();
    const int w = warp >> 2, q = warp & 3;
    const int r = q * 32 + lane;                     // TMEM lane = token row in the tile
    const uint32_t lb = (uint32_t)(q * 32) << 16;
    const uint32_t tR = tmem + lb + w * R;
    const int64_t nW = (ntiles - w + 1) / 2;
    bool ok = true;
    const float Rh = ST ? bs.rref[bh] : 0.f;
    const int64_t dyhead = ST ? bs.tdy.head(bh, H) : 0;
    for (int64_t j = 0; j < nW; ++j) {
      const int64_t i = 2 * j + w;
      const int64_t tok = ht.row0(tile0 + i, kTile) + r;
      const bool mine = ht.own(tile0 + i, kTile, r);
      // statistics: the row's dY is read after the softmax; start its load now
      if (ST && mine) prefetch_l1(bs.dY + dyhead + tok * bs.tdy.sn);
      const int slot = (int)(i % kDecBoundSlots);
      if (!warp_all(mbar_wait(&s_full[w], (uint32_t)(j & 1)) &&
                    (!kBound || mbar_wait(&kn_full[slot], (uint32_t)((i / kDecBoundSlots) & 1))) &&
                    !*abort_flag)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      // Chunks of 32 columns, double-buffered: the load of the next chunk is
      // in flight while the current one is processed.  Pass 2 below visits
      // them in the order: upper half last chunk first, then lower half
      // first chunk first.  The P of upper chunk u (S columns [M/2 + 32u,
      // +32)) goes to columns [3M/4 + 16u, +16), inside upper chunks already
      // read; the P of lower chunk u goes to [16u, +16), inside lower chunks
      // already read.  No store touches a chunk that is still to be loaded.
      constexpr int NC = M / 32;
      auto chunk_col = [](int k) { return k < NC / 2 ? M / 2 + 32 * (NC / 2 - 1 - k) : 32 * (k - NC / 2); };
      auto p_col = [](int k) { return k < NC / 2 ? 3 * M / 4 + 16 * (NC / 2 - 1 - k) : 16 * (k - NC / 2); };
      float sf[4] = {0.f, 0.f, 0.f, 0.f};
      float rmx;   // the row's reference logit (its max, or the first chunk's)
      if constexpr (PAD) {
        // Columns [0, Mv) only, in whole or half (16-column) chunks: pass 1
        // the exact row max, pass 2 the weights in the placement order above
        // (a skipped chunk's columns are never read, so the P of an upper
        // chunk may land on them).
        float mf[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int cc = 0; cc < NC; ++cc) {
          if (32 * cc >= Mv) break;
          if (32 * cc + 32 <= Mv) {
            uint32_t a[32];
            tmem_ld32(tR + 32 * cc, a);
            tmem_wait_ld_dep(a);
            max_fold32(a, mf);
          } else {
            uint32_t a[16];
            tmem_ld16(tR + 32 * cc, a);
            tmem_wait_ld_dep16(a);
            max_fold16(a, mf);
          }
        }
        rmx = fmaxf(fmaxf(mf[0], mf[1]), fmaxf(mf[2], mf[3]));
        const float neg = -rmx * c;
#pragma unroll
        for (int k = 0; k < NC; ++k) {
          const int col = chunk_col(k);
          if (col >= Mv) continue;
          if (col + 32 <= Mv) {
            uint32_t a[32], pk[16];
            tmem_ld32(tR + col, a);
            tmem_wait_ld_dep(a);
            exp_pack32<dec_poly_every(M), false, false>(a, c, neg, pk, sf);
            tmem_st16(tR + p_col(k), pk);
          } else {
            uint32_t a[16], pk[8];
            tmem_ld16(tR + col, a);
            tmem_wait_ld_dep16(a);
            exp_pack16<0, false, false>(a, c, neg, pk, sf);
            tmem_st8(tR + p_col(k), pk);
          }
        }
      } else {
        uint32_t a[2][32];
        float mf[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if constexpr (kBound) {
          tmem_ld32(tR + chunk_col(0), a[0]);
          const float U = kn[slot * kTile + r];   // >= c S[m] for every latent (bound warps)
          tmem_wait_ld_dep(a[0]);
          max_fold32(a[0], mf);
          // reference: the first chunk's max, unless the bound allows a logit
          // more than 2^kDecRefTau above it somewhere in the warp's rows; then
          // the exact row max (pass 1 over the other chunks)
          if (warp_any(U - c * fmaxf(fmaxf(mf[0], mf[1]), fmaxf(mf[2], mf[3])) > kDecRefTau)) {
            for (int cc = 1; cc < NC; ++cc) {
              tmem_ld32(tR + chunk_col(cc), a[1]);
              tmem_wait_ld_dep(a[1]);
              max_fold32(a[1], mf);
            }
          }
        } else {
          // pass 1: the exact row max over all M logits
          tmem_ld32(tR, a[0]);
#pragma unroll
          for (int cc = 0; cc < NC; ++cc) {
            tmem_wait_ld_dep(a[cc & 1]);
            if (cc + 1 < NC) tmem_ld32(tR + 32 * (cc + 1), a[(cc + 1) & 1]);
            max_fold32(a[cc & 1], mf);
          }
          tmem_ld32(tR + chunk_col(0), a[0]);
        }
        const float mx = fmaxf(fmaxf(mf[0], mf[1]), fmaxf(mf[2], mf[3]));
        const float neg = -mx * c;
        // pass 2 (chunk 0 is in, or on its way to, a[0]); the MMA warp
        // starts Y on the upper half of the latents (and on latents 0-63
        // with M = 256) as soon as their P is written
#pragma unroll
        for (int k = 0; k < NC; ++k) {
          if (k > 0 || !kBound) tmem_wait_ld_dep(a[k & 1]);
          if (k + 1 < NC) tmem_ld32(tR + chunk_col(k + 1), a[(k + 1) & 1]);
          uint32_t pk[16];
          exp_pack32<dec_poly_every(M), false, false>(a[k & 1], c, neg, pk, sf);
          tmem_st16(tR + p_col(k), pk);
          if (k == NC / 2 - 1 || (NC == 8 && k == 5)) {
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_part[2 * w + (k == NC / 2 - 1 ? 0 : 1)]);
          }
        }
        rmx = mx;
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[w]);
      if (!warp_all(mbar_wait(&y_full[w], (uint32_t)(j & 1)))) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      // [Y | l]: l = the row's sum of its bf16 weights (the ones of Z's N-atom)
      float y[D], l;
      if (D == 32) {
        uint32_t o[32], o2[16];
        tmem_ld32(tR + TY, o);
        tmem_ld16(tR + TY + 32, o2);
        tmem_wait_ld();
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = __uint_as_float(o[d]);
        l = __uint_as_float(o2[0]);
      } else {
        uint32_t o[32];
        tmem_ld32(tR + TY, o);
        tmem_wait_ld();
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = __uint_as_float(o[d & 31]);
        l = __uint_as_float(o[16]);
      }
      tc_fence_before();
      mbar_arrive(&s_empty[w]);
      if constexpr (ST) {
        const float inv = 1.f / l;
        const float mxp = fmaf(rmx, c, log2f(l));   // the row's log-sum-exp, log2 units
        const float lg = mxp - Rh;                  // log2 of g
        const bool bad = mine && lg < -kBwdRowRange;
        if (mine) {
          const float ginv = bad ? 0.f : ex2(-lg);
          const uint4* src = reinterpret_cast<const uint4*>(bs.dY + dyhead + tok * bs.tdy.sn);
          uint4* dst = reinterpret_cast<uint4*>(bs.dy2 + (bh * N + tok) * D);
          float dot = 0.f, dot2 = 0.f;
#pragma unroll
          for (int v = 0; v < D / 8; ++v) {
            const uint4 u = src[v];
            const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
            uint32_t w2[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const float a0 = bf_lo(uu[jj]), a1 = bf_hi(uu[jj]);
              const float y0 = y[8 * v + 2 * jj], y1 = y[8 * v + 2 * jj + 1];
              dot = fmaf(a0, y0, fmaf(a1, y1, dot));
              w2[jj] = pack_bf16(a0 * ginv, a1 * ginv);
              dot2 = fmaf(bf_lo(w2[jj]), y0, fmaf(bf_hi(w2[jj]), y1, dot2));
            }
            dst[v] = make_uint4(w2[0], w2[1], w2[2], w2[3]);
          }
          bs.stats[bh * N + tok] = make_float4(mxp, dot * inv, dot2 * inv, 0.f);
        }
        if (warp_any(bad) && lane == 0) atomicOr(bs.flags + bh, 1u);
      } else if (mine) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(Y + yhead + tok * ty.sn);
#pragma unroll
        for (int v = 0; v < D / 8; ++v) {
          uint4 u;
          u.x = pack_bf16(y[8 * v + 0] * inv, y[8 * v + 1] * inv);
          u.y = pack_bf16(y[8 * v + 2] * inv, y[8 * v + 3] * inv);
          u.z = pack_bf16(y[8 * v + 4] * inv, y[8 * v + 5] * inv);
          u.w = pack_bf16(y[8 * v + 6] * inv, y[8 * v + 7] * inv);
          dst[v] = u;
        }
      }
    }
    if (!ok) {
      record_error(err, kErrDecSoftmaxWait);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, NCOLS);
}

// ============================================================== host side

}  // namespace


PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return (PFN_cuTensorMapEncodeTiled_v12000)p;
  }();
  return fn;
}

// 3-D map over a bf16 tensor [depth][rows][D] with boxes of box_rows rows,
// swizzled to match the UMMA descriptors (row = whole head dimension).
cudaError_t make_map(CUtensorMap* m, const void* base, int D, int64_t rows, int64_t depth,
                     int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    note_error("cuTensorMapEncodeTiled entry point unavailable");
    return cudaErrorNotSupported;
  }
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)depth};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = (D == 32) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    note_error("cuTensorMapEncodeTiled failed (CUresult %d): D=%d rows=%lld depth=%lld box=%d",
               (int)r, D, (long long)rows, (long long)depth, box_rows);
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t make_tok_map(CUtensorMap* m, const void* base, const Dims& d, const Tok& t,
                         int box_rows, bool flat) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    note_error("cuTensorMapEncodeTiled entry point unavailable");
    return cudaErrorNotSupported;
  }
  const int64_t fs = flat_stride(t, d);
  if (flat && fs <= 0) return cudaErrorInvalidValue;
  const cuuint32_t rank = flat ? 3 : 4;
  cuuint64_t dims[4] = {(cuuint64_t)d.D, (cuuint64_t)d.N, (cuuint64_t)d.H, (cuuint64_t)d.B};
  cuuint64_t strides[3] = {(cuuint64_t)t.sn * 2, (cuuint64_t)t.sh * 2, (cuuint64_t)t.sb * 2};
  if (flat) {
    dims[2] = (cuuint64_t)(d.B * d.H);
    strides[1] = (cuuint64_t)fs * 2;
  }
  cuuint32_t box[4] = {(cuuint32_t)d.D, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  const CUtensorMapSwizzle sw = (d.D == 32) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    note_error("cuTensorMapEncodeTiled failed (CUresult %d): token map D=%lld N=%lld H=%lld "
               "B=%lld strides %lld/%lld/%lld box=%d",
               (int)r, (long long)d.D, (long long)d.N, (long long)d.H, (long long)d.B,
               (long long)t.sb, (long long)t.sh, (long long)t.sn, box_rows);
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

namespace {

// DZ: V is dY (token strides d.dy), stats the decode statistics, pml unused.
template <int D, int M, bool FLAT, bool VAR, bool DZ>
cudaError_t tc_encode_t(const void* Q, int64_t qbs, const void* K, const void* V, const Dims& d,
                        float scale, const ChunkPlan& plan, float* pml, float* pacc,
                        const float4* stats, uint32_t* err, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const int q_per_batch = qbs != 0;
  cudaError_t e;
  // Q [.., Mv, D]: rows past Mv of the 128-row boxes are the TMA's zero fill
  if ((e = make_map(&mq, Q, D, d.M, q_per_batch ? d.BH() : d.H, 128)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mk, K, d, d.k, kEncTile, FLAT)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mv, V, d, DZ ? d.dy : d.v, kEncTile, FLAT)) != cudaSuccess) return e;
  // two CTAs per SM: their TMEM (2 x 256 columns) fits exactly
  const int smem = EncLayout<D, M, DZ>::BYTES + 1024;
  e = cudaFuncSetAttribute(tc_encode_kernel<D, M, FLAT, VAR, DZ>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // with lengths: one CTA per unit of the encode's work plan
  const dim3 grid = VAR ? dim3((unsigned)d.venc.n) : dim3(plan.chunks, (unsigned)d.BH());
  launch_pdl(tc_encode_kernel<D, M, FLAT, VAR, DZ>, grid, kThreads, smem, st,
      mq, mk, mv, (int)d.H, d.N, q_per_batch, (int)d.M, scale * kLog2e, plan.tiles_per_bh,
      plan.chunk_tiles, pml, pacc, d.lens, d.venc.units, stats, err);
  return cudaPeekAtLastError();
}

template <int D, int M, bool FLAT, bool VAR, bool ST, bool PAD = false>
cudaError_t tc_decode_t(const void* Q, int64_t qbs, const void* K, const __nv_bfloat16* Zb,
                        void* Y, const Dims& d, float scale, const ChunkPlan& plan,
                        const DecStats& bs, uint32_t* err, cudaStream_t st) {
  CUtensorMap mq, mk, mz;
  const int q_per_batch = qbs != 0;
  cudaError_t e;
  // Q and Z [.., Mv, D] in boxes of M rows: rows past Mv are the TMA's zero fill
  if ((e = make_map(&mq, Q, D, d.M, q_per_batch ? d.BH() : d.H, M)) != cudaSuccess) return e;
  if ((e = make_tok_map(&mk, K, d, d.k, kTile, FLAT)) != cudaSuccess) return e;
  if ((e = make_map(&mz, Zb, D, d.M, d.BH(), M)) != cudaSuccess) return e;
  const int smem = (DecLayout<D, M>::BYTES + 1024 > kMinSmemBytes) ? DecLayout<D, M>::BYTES + 1024
                                                                   : kMinSmemBytes;
  e = cudaFuncSetAttribute(tc_decode_kernel<D, M, FLAT, VAR, ST, PAD>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // with lengths: one CTA per unit of the 128-token work plan
  const dim3 grid = VAR ? dim3((unsigned)d.vtok.n) : dim3(plan.chunks, (unsigned)d.BH());
  launch_pdl(tc_decode_kernel<D, M, FLAT, VAR, ST, PAD>, grid, kThreads, smem, st,
      mq, mk, mz, (int)d.H, d.N, q_per_batch, (int)d.M, scale * kLog2e, plan.tiles_per_bh,
      plan.chunk_tiles, (__nv_bfloat16*)Y, d.y, (const __nv_bfloat16*)Q, d.lens, d.vtok.units, bs,
      err);
  return cudaPeekAtLastError();
}

}  // namespace

template <int D, int M, bool DZ>
cudaError_t tc_encode_dispatch(const void* Q, int64_t qbs, const void* K, const void* V,
                               const Dims& d, float scale, const ChunkPlan& plan, float* pml,
                               float* pacc, const float4* stats, uint32_t* err, cudaStream_t st) {
  const bool flat = tok_flat(d), var = d.lens != nullptr;
#define FLARE_TC_ENC(F, V_) \
  tc_encode_t<D, M, F, V_, DZ>(Q, qbs, K, V, d, scale, plan, pml, pacc, stats, err, st)
  if (flat) return var ? FLARE_TC_ENC(true, true) : FLARE_TC_ENC(true, false);
  return var ? FLARE_TC_ENC(false, true) : FLARE_TC_ENC(false, false);
#undef FLARE_TC_ENC
}

cudaError_t launch_tc_encode(const void* Q, int64_t qbs, const void* K, const void* V,
                             const Dims& d, float scale, const ChunkPlan& plan, float* pml,
                             float* pacc, uint32_t* err, cudaStream_t st) {
#define FLARE_ENC_ARGS Q, qbs, K, V, d, scale, plan, pml, pacc, nullptr, err, st
  // latent counts below 128 (or between 128 and 256) run on the 128-row
  // (256-row) kernel with zero latents past d.M that are never stored
  const int Mp = tc_latent_tile(d.M);
  if (d.D == 32 && Mp == 256) return tc_encode_dispatch<32, 256, false>(FLARE_ENC_ARGS);
  if (d.D == 32 && Mp == 128) return tc_encode_dispatch<32, 128, false>(FLARE_ENC_ARGS);
  if (d.D == 16 && Mp == 256) return tc_encode_dispatch<16, 256, false>(FLARE_ENC_ARGS);
  if (d.D == 16 && Mp == 128) return tc_encode_dispatch<16, 128, false>(FLARE_ENC_ARGS);
#undef FLARE_ENC_ARGS
  return cudaErrorNotSupported;
}

cudaError_t launch_tc_dz(const void* Q, int64_t qbs, const void* K, const void* dY, const Dims& d,
                         float scale, const ChunkPlan& plan, const float4* stats, float* dz_part,
                         uint32_t* err, cudaStream_t st) {
  if (d.M != 256) return cudaErrorNotSupported;
  if (d.D == 32)
    return tc_encode_dispatch<32, 256, true>(Q, qbs, K, dY, d, scale, plan, nullptr, dz_part,
                                             stats, err, st);
  if (d.D == 16)
    return tc_encode_dispatch<16, 256, true>(Q, qbs, K, dY, d, scale, plan, nullptr, dz_part,
                                             stats, err, st);
  return cudaErrorNotSupported;
}

template <int D, int M>
cudaError_t tc_decode_dispatch(const void* Q, int64_t qbs, const void* K,
                               const __nv_bfloat16* Zb, void* Y, const Dims& d, float scale,
                               const ChunkPlan& plan, uint32_t* err, cudaStream_t st) {
  // The decode takes 4-D maps for every layout: its 3-D variant measured no
  // faster and needs more registers.
  const DecStats none{};
  if (d.M != M)   // latents padded to the kernel's M
    return d.lens != nullptr
               ? tc_decode_t<D, M, false, true, false, true>(Q, qbs, K, Zb, Y, d, scale, plan, none,
                                                             err, st)
               : tc_decode_t<D, M, false, false, false, true>(Q, qbs, K, Zb, Y, d, scale, plan,
                                                              none, err, st);
  return d.lens != nullptr
             ? tc_decode_t<D, M, false, true, false>(Q, qbs, K, Zb, Y, d, scale, plan, none, err, st)
             : tc_decode_t<D, M, false, false, false>(Q, qbs, K, Zb, Y, d, scale, plan, none, err, st);
}

cudaError_t launch_tc_decode(const void* Q, int64_t qbs, const void* K, const __nv_bfloat16* Zb,
                             void* Y, const Dims& d, float scale, const ChunkPlan& plan,
                             uint32_t* err, cudaStream_t st) {
  const int Mp = tc_latent_tile(d.M);
  if (d.D == 32 && Mp == 256) return tc_decode_dispatch<32, 256>(Q, qbs, K, Zb, Y, d, scale, plan, err, st);
  if (d.D == 32 && Mp == 128) return tc_decode_dispatch<32, 128>(Q, qbs, K, Zb, Y, d, scale, plan, err, st);
  if (d.D == 16 && Mp == 256) return tc_decode_dispatch<16, 256>(Q, qbs, K, Zb, Y, d, scale, plan, err, st);
  if (d.D == 16 && Mp == 128) return tc_decode_dispatch<16, 128>(Q, qbs, K, Zb, Y, d, scale, plan, err, st);
  return cudaErrorNotSupported;
}

cudaError_t launch_tc_bwd_stats(const void* Q, int64_t qbs, const void* K, const __nv_bfloat16* Zb,
                                const void* dY, const Dims& d, float scale, const ChunkPlan& plan,
                                const float* rref, float4* stats, __nv_bfloat16* dy2,
                                uint32_t* flags, uint32_t* err, cudaStream_t st) {
  if (d.M != 256) return cudaErrorNotSupported;
  const DecStats bs{(const __nv_bfloat16*)dY, d.dy, rref, stats, dy2, flags};
#define FLARE_TC_ST(D_, V_) \
  tc_decode_t<D_, 256, false, V_, true>(Q, qbs, K, Zb, nullptr, d, scale, plan, bs, err, st)
  const bool var = d.lens != nullptr;
  if (d.D == 32) return var ? FLARE_TC_ST(32, true) : FLARE_TC_ST(32, false);
  if (d.D == 16) return var ? FLARE_TC_ST(16, true) : FLARE_TC_ST(16, false);
#undef FLARE_TC_ST
  return cudaErrorNotSupported;
}

}  // namespace flare
