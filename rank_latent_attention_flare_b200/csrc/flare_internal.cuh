// Internal declarations shared by the FLARE CUDA sources: workspace layout,
// work partitioning, device helpers and kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include "flare.h"

namespace flare {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Tensor-core backward: a token whose decode log-sum-exp lies more than
// this far (log2 units) below its head's R = max_m lse2[m] flags the head,
// which then takes the exact form of the encode weights.
constexpr float kBwdRowRange = 100.f;

// Error sites recorded in the workspace header when a bounded wait runs out.
enum ErrorSite : uint32_t {
  kErrNone = 0,
  kErrEncTmaWait = 0x101,
  kErrEncMmaWait = 0x102,
  kErrEncSoftmaxWait = 0x103,
  kErrDecTmaWait = 0x201,
  kErrDecMmaWait = 0x202,
  kErrDecSoftmaxWait = 0x203,
  kErrTmemAlloc = 0x301,
  kErrBwdATmaWait = 0x401,
  kErrBwdAMmaWait = 0x402,
  kErrBwdARowWait = 0x403,
  kErrBwdBTmaWait = 0x501,
  kErrBwdBMmaWait = 0x502,
  kErrBwdBRowWait = 0x503,
  kErrSeqLen = 0x601,   // a sequence length outside [0, N] (clamped)
};

// ------------------------------------------------------------------ planning

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t imax64(int64_t a, int64_t b) { return a > b ? a : b; }

// Split of one (b, h) token range into `chunks` contiguous chunks of
// `chunk_tiles` tiles of `tile` tokens (the last chunk may be shorter).
struct ChunkPlan {
  int tile = 0;
  int64_t tiles_per_bh = 0;
  int chunks = 0;
  int64_t chunk_tiles = 0;
  int sub = 1;  // partial records per chunk (tensor-core encode with M=128: 2)
  int64_t chunk_tokens() const { return chunk_tiles * tile; }
  int slots_per_bh() const { return chunks * sub; }
};

// Picks the chunk count that minimises (waves x tiles per chunk), where a
// wave is `cta_slots` concurrently resident CTAs and each CTA pays
// `overhead_tiles` of set-up.  Deterministic for given arguments.
inline ChunkPlan plan_chunks(int64_t BH, int64_t N, int tile, int64_t cta_slots,
                             double overhead_tiles, int64_t max_chunks) {
  ChunkPlan p;
  p.tile = tile;
  p.tiles_per_bh = (N + tile - 1) / tile;
  int64_t hi = p.tiles_per_bh;
  if (hi > max_chunks) hi = max_chunks;
  double best = 1e300;
  int64_t best_c = 1, best_per = p.tiles_per_bh;
  for (int64_t c = 1; c <= hi; ++c) {
    int64_t per = (p.tiles_per_bh + c - 1) / c;
    int64_t ceff = (p.tiles_per_bh + per - 1) / per;
    if (ceff != c) continue;
    int64_t waves = (BH * ceff + cta_slots - 1) / cta_slots;
    double cost = (double)waves * ((double)per + overhead_tiles);
    if (cost < best - 1e-9) {
      best = cost;
      best_c = ceff;
      best_per = per;
    }
  }
  p.chunks = (int)best_c;
  p.chunk_tiles = best_per;
  return p;
}

// Which kernels a call uses.
struct Path {
  bool tc_fwd = false;  // tcgen05 encode + decode
  bool tc_bwd = false;  // tcgen05 backward (two passes over the tokens)
};

// Latent rows the tensor-core forward computes for M latents: one 128-row
// MMA tile (M <= 128) or two (M <= 256); rows past M are zero latents that
// are never stored (encode) or never weighted (decode).
inline int tc_latent_tile(int64_t M) { return M <= 128 ? 128 : 256; }

// The tcgen05 forward covers bf16 with any supported M (a multiple of 16 in
// [16, 256], padded to tc_latent_tile), D in {16, 32} and N addressable by a
// TMA coordinate; the tcgen05 backward covers M in {128, 256}.
inline Path choose_path(int64_t N, int64_t M, int64_t D, flare_dtype_t dt) {
  Path p;
  p.tc_fwd = (dt == FLARE_BF16) && (M % 16 == 0) && M >= 16 && M <= 256 && (D == 16 || D == 32) &&
             (N < (1LL << 31) - 256);
  p.tc_bwd = (dt == FLARE_BF16) && (M == 128 || M == 256) && (D == 16 || D == 32) &&
             (N < (1LL << 31) - 256);
  return p;
}

// Split of the forward's exponentials between the MUFU (ex2.approx) and the
// FMA-pipe polynomial, per latent tile (128 or 256 rows): in the
// tensor-core encode, every enc_poly_every32-th pair of each 48-logit row
// tile's first 32 logits and every enc_poly_every16-th pair of its last 16
// runs as the polynomial (0 = none); in the decode, every dec_poly_every-th
// pair of each 32-logit chunk.  Measured on the 256-row tile at one million
// tokens, and on the 128-row tile at 16K-65K tokens (where the larger shares
// measured slower).
#ifndef FLARE_ENC_POLY32
#define FLARE_ENC_POLY32 3
#endif
#ifndef FLARE_ENC_POLY16
#define FLARE_ENC_POLY16 3
#endif
#ifndef FLARE_DEC_POLY
#define FLARE_DEC_POLY 8
#endif
constexpr int enc_poly_every32(int Mp) { return Mp == 256 ? FLARE_ENC_POLY32 : 4; }
constexpr int enc_poly_every16(int Mp) { return Mp == 256 ? FLARE_ENC_POLY16 : 4; }
constexpr int dec_poly_every(int Mp) { return Mp == 256 ? FLARE_DEC_POLY : 16; }

// Share of a tensor-core kernel's exponentials computed by the polynomial.
constexpr double enc_poly_fraction(int Mp) {
  return ((enc_poly_every32(Mp) > 0 ? 16 / enc_poly_every32(Mp) : 0) +
          (enc_poly_every16(Mp) > 0 ? 8 / enc_poly_every16(Mp) : 0)) / 24.0;
}
constexpr double dec_poly_fraction(int Mp) {
  return (dec_poly_every(Mp) > 0 ? 16 / dec_poly_every(Mp) : 0) / 16.0;
}

constexpr int kSimtEncTile = 64;
constexpr int kSimtEncThreads = 256;
constexpr int kSimtDecThreads = 128;
constexpr int kTcTile = 128;     // decode tile (tokens)
constexpr int kTcEncTile = 48;   // tensor-core encode tile (tokens)
constexpr int kBwdTile = 256;

inline ChunkPlan encode_plan(int64_t BH, int64_t N, int64_t M, int64_t D, flare_dtype_t dt,
                             int sms) {
  Path path = choose_path(N, M, D, dt);
  if (path.tc_fwd) {
    // two encode CTAs are resident per SM
    ChunkPlan p = plan_chunks(BH, N, kTcEncTile, 2LL * sms, 12.0, 32 * (int64_t)sms);
    p.sub = (tc_latent_tile(M) == 128) ? 2 : 1;   // one 128-row tile: the warpgroups split tiles
    return p;
  }
  return plan_chunks(BH, N, kSimtEncTile, 4LL * sms, 2.0, 64 * (int64_t)sms);
}

inline ChunkPlan decode_plan(int64_t BH, int64_t N, int sms) {
  return plan_chunks(BH, N, kTcTile, sms, 6.0, 16 * (int64_t)sms);
}

// Units a length-proportional plan may use (calls with lengths): at least
// the chunk plan's, and up to two waves of `cta_slots` CTAs, but never more
// than the tiles.
inline int64_t var_units(int64_t BH, const ChunkPlan& p, int64_t cta_slots) {
  return imax64(BH * p.chunks, imin64(2 * cta_slots, BH * p.tiles_per_bh));
}

inline ChunkPlan bwd_plan(int64_t BH, int64_t N, int sms) {
  return plan_chunks(BH, N, kBwdTile, 2LL * sms, 1.0, 16 * (int64_t)sms);
}

// Both passes of the tensor-core backward: 128-token tiles, one CTA per SM.
inline ChunkPlan tc_bwd_plan(int64_t BH, int64_t N, int sms) {
  return plan_chunks(BH, N, kTcTile, sms, 6.0, 16 * (int64_t)sms);
}

// ------------------------------------------------------------- workspace

struct WsLayout {
  size_t hdr = 0;       // uint32 error word (256 bytes reserved)
  size_t part_ml = 0;   // [BH*slots][M][2] float: running max (log2 units), sum
  size_t part_acc = 0;  // [BH*slots][M][D] float
  size_t zf = 0;        // [BH][M][D] float  Z
  size_t zb = 0;        // [BH][M][D] bf16   Z operand copy for the decode
  size_t qdyn = 0;      // [BH][M][D] dtype  FLARE++ corrected queries
  size_t dkf = 0;       // [BH][N][D] float  decode-stage part of dK
  size_t dqp = 0;       // [2][BH*chunks][M][D] float dQ partials (decode, encode)
  size_t dzp = 0;       // [BH*chunks][M][D] float  dZ partials
  size_t dz = 0;        // [BH][M][D] float
  size_t delta = 0;     // [BH][M] float  rowsum(dZ * Z)
  // tensor-core backward (the dZ / dQ partials use dzp / dqp, one set each)
  size_t stats = 0;     // [BH][N] float4  decode log-sum-exp (log2 units), delta_d, delta''
  size_t dy2 = 0;       // [BH][N][D] bf16  dY / g
  size_t rref = 0;      // [BH] float  R = max lse2
  size_t flags = 0;     // [BH] uint32  a token out of the range of the one-exponential form
  size_t dzs = 0;       // [BH][M][D] bf16  f * dZ
  size_t aug = 0;       // [BH][M][16] bf16 extra K-step row (-f delta_e in three terms)
  size_t params = 0;    // [BH] float2  R, fast-form flag
  size_t lse2 = 0;      // [BH][M] float  lse in log2 units
  // FLARE++ backward, in addition to the FLARE backward's buffers
  size_t z1 = 0;        // [BH][M][D] float  first encode's Z1 (recomputed)
  size_t lse1 = 0;      // [BH][M] float  its lse
  size_t dqd = 0;       // [BH][M][D] dtype  dQ_dyn
  size_t dz1 = 0;       // [BH][M][D] float  dQ_dyn widened
  size_t delta1 = 0;    // [BH][M] float  rowsum(dZ1 * Z1)
  size_t dqe = 0;       // [BH*chunks][M][D] float  first encode's dQ partials
  // the work plans of calls with lengths (tensor-core path)
  size_t vu_enc = 0;    // [n_enc] int4 units of the encode
  size_t vh_enc = 0;    // [BH] int2 (first unit, units)
  size_t vu_tok = 0;    // [n_tok] int4 units of the 128-token kernels
  size_t vh_tok = 0;    // [BH] int2
  int64_t n_enc = 0, n_tok = 0;
  size_t total = 0;
  ChunkPlan enc, bwd, ppe;
  ChunkPlan dec;        // tensor-core backward, M = 256: its decode-statistics pass
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline WsLayout ws_layout(flare_op_t op, int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                          flare_dtype_t dt, int sms) {
  WsLayout L;
  const int64_t BH = B * H;
  const size_t esz = (dt == FLARE_F32) ? 4 : 2;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.enc = encode_plan(BH, N, M, D, dt, sms);
  const Path path = choose_path(N, M, D, dt);
  if (path.tc_fwd) {
    L.n_enc = var_units(BH, L.enc, 2 * sms);
    L.n_tok = var_units(BH, decode_plan(BH, N, sms), sms);
  }
  const int64_t slots = imax64(BH * L.enc.slots_per_bh(), L.n_enc * L.enc.sub);
  L.hdr = take(256);
  if (path.tc_fwd) {
    L.vu_enc = take((size_t)L.n_enc * 16);
    L.vh_enc = take((size_t)BH * 8);
    L.vu_tok = take((size_t)L.n_tok * 16);
    L.vh_tok = take((size_t)BH * 8);
  }
  L.part_ml = take((size_t)slots * M * 2 * 4);
  L.part_acc = take((size_t)slots * M * D * 4);
  L.zf = take((size_t)BH * M * D * 4);
  L.zb = take((size_t)BH * M * D * 2);
  if (op == FLARE_OP_PP_FWD) L.qdyn = take((size_t)BH * M * D * esz);
  const bool bwd_like = (op == FLARE_OP_BWD || op == FLARE_OP_PP_BWD);
  if (bwd_like && choose_path(N, M, D, dt).tc_bwd) {
    L.bwd = tc_bwd_plan(BH, N, sms);
    const int64_t bslots = imax64(BH * L.bwd.chunks, L.n_tok);
    // with M = 256 the dZ partials come from the encode pipeline (its chunks)
    const int64_t zslots = (M == 256) ? slots : bslots;
    if (M == 256) L.dec = decode_plan(BH, N, sms);
    L.stats = take((size_t)BH * N * 16);
    L.dy2 = take((size_t)BH * N * D * 2);
    L.rref = take((size_t)BH * 4);
    L.flags = take((size_t)BH * 4);
    L.dzp = take((size_t)zslots * M * D * 4);
    L.dqp = take((size_t)bslots * M * D * 4);
    L.dzs = take((size_t)BH * M * D * 2);
    L.aug = take((size_t)BH * M * 16 * 2);
    L.params = take((size_t)BH * 8);
    L.lse2 = take((size_t)BH * M * 4);
  } else if (bwd_like) {
    L.bwd = bwd_plan(BH, N, sms);
    const int64_t bslots = BH * L.bwd.chunks;
    L.dkf = take((size_t)BH * N * D * 4);
    L.dqp = take((size_t)2 * bslots * M * D * 4);
    L.dzp = take((size_t)bslots * M * D * 4);
    L.dz = take((size_t)BH * M * D * 4);
    L.delta = take((size_t)BH * M * 4);
  }
  if (op == FLARE_OP_PP_BWD) {
    L.z1 = take((size_t)BH * M * D * 4);
    L.lse1 = take((size_t)BH * M * 4);
    L.dqd = take((size_t)BH * M * D * esz);
  }
  if (op == FLARE_OP_PP_BWD && !choose_path(N, M, D, dt).tc_bwd) {
    // the first encode's gradient on CUDA cores
    L.ppe = bwd_plan(BH, N, sms);
    L.dz1 = take((size_t)BH * M * D * 4);
    L.delta1 = take((size_t)BH * M * 4);
    L.dqe = take((size_t)BH * L.ppe.chunks * M * D * 4);
  }
  L.total = off;
  return L;
}

// ------------------------------------------------------------ device helpers

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ void record_error(uint32_t* err, uint32_t site) {
  if (err) atomicCAS(err, 0u, site);
}

// Records a description of the last launch-time failure on this host thread
// (read back through flare_last_error_detail).
void note_error(const char* fmt, ...);

// ------------------------------------------------------------ launchers
// Each returns cudaSuccess or the launch error.

// Element strides of a token tensor [B,H,N,D] whose head dimension D is
// contiguous: element (b, h, n, d) sits at b sb + h sh + n sn + d.
struct Tok {
  int64_t sb, sh, sn;
  // offset of row 0 of head bh = b H + h
  __host__ __device__ __forceinline__ int64_t head(int64_t bh, int64_t H) const {
    return (bh / H) * sb + (bh % H) * sh;
  }
};

// A length-proportional work plan.  Unit u of a launch of `n` CTAs is
// units[u] = (bh, first tile, tiles, 0) -- head bh's tiles split into
// max(1, ceil(tiles / per)) near-equal units, heads in order, one CTA each;
// bh < 0 marks a unit the plan leaves empty.  heads[bh] = (first unit, units)
// locates a head's records, which the CTAs write at their unit's slot.
struct VarPlan {
  const int4* units = nullptr;
  const int2* heads = nullptr;
  int64_t n = 0;
  bool on() const { return units != nullptr; }
};

// Problem sizes and the layouts of the token tensors (contiguous [B,H,N,D]
// unless the caller gave strides).
struct Dims {
  int64_t B, H, N, M, D;
  Tok k = contig(), v = contig(), y = contig();     // K, V, the forward's Y
  Tok dy = contig(), dk = contig(), dv = contig();  // dY, dK, dV
  const int32_t* lens = nullptr;   // device [B]: valid tokens per batch element (NULL: N)
  // With lengths on the tensor-core path, the length-proportional work plans
  // that a plan block writes into the workspace (NULL otherwise): one for
  // the 48-token encode, one for the 128-token kernels (decode, backward).
  VarPlan venc, vtok;
  int64_t BH() const { return B * H; }
  Tok contig() const { return Tok{H * N * D, N * D, D}; }
};

// The padding rows (tokens [L_b, N)) of up to two token tensors of the same
// shape, to be zeroed by `nxb` blocks per head: the standalone kernel, or
// extra blocks of a kernel launched anyway (the combine, the backward's
// preparation) beside its own.
struct PadZero {
  uint8_t* x0 = nullptr;   // NULL: nothing to zero
  Tok t0{};
  uint8_t* x1 = nullptr;
  Tok t1{};
  const int32_t* lens = nullptr;
  int64_t N = 0;
  int H = 1, esz = 2;
  int lg_row = 2;          // log2 of the 16-byte pieces per row
  int nxb = 0;             // blocks per head
  int64_t blocks(int64_t BH) const { return x0 ? (int64_t)nxb * BH : 0; }
};

// Valid tokens of batch element b: lens[b] clamped to [0, N] (N when lens is
// NULL).  Tokens n >= that count are padding: never read, outputs zero.
__device__ __forceinline__ int64_t seq_len(const int32_t* __restrict__ lens, int64_t b,
                                           int64_t N) {
  if (lens == nullptr) return N;
  const int64_t L = __ldg(lens + b);
  return L < 0 ? 0 : (L > N ? N : L);
}

__host__ __device__ __forceinline__ int64_t tiles_of(int64_t nb, int T) { return (nb + T - 1) / T; }

// Block xb of a PadZero's nxb blocks for head bh: a stride loop over the
// head's padding in 16-byte stores.
__device__ __forceinline__ void zero_padding_part(const PadZero& z, int64_t xb, int64_t bh) {
  const int64_t L = seq_len(z.lens, bh / z.H, z.N);
  const int64_t total = (z.N - L) << z.lg_row;
  if (total == 0) return;
  const int mask = (1 << z.lg_row) - 1;
  uint8_t* p0 = z.x0 + (z.t0.head(bh, z.H) + L * z.t0.sn) * z.esz;
  uint8_t* p1 = z.x1 ? z.x1 + (z.t1.head(bh, z.H) + L * z.t1.sn) * z.esz : nullptr;
  const int64_t r0 = z.t0.sn * z.esz, r1 = z.t1.sn * z.esz;   // row strides in bytes
  for (int64_t i = xb * blockDim.x + threadIdx.x; i < total; i += (int64_t)z.nxb * blockDim.x) {
    const int64_t n = i >> z.lg_row;
    const int piece = (int)i & mask;
    reinterpret_cast<uint4*>(p0 + n * r0)[piece] = make_uint4(0u, 0u, 0u, 0u);
    if (p1) reinterpret_cast<uint4*>(p1 + n * r1)[piece] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Token tiles of one head, T tokens each.  Without lengths (VAR false) the
// head has all N tokens: tile t covers rows [tT, tT + T) and TMA fills the
// rows past N with zeros.  With lengths it has nb <= N tokens and a partial
// last tile is right-aligned to end at nb, so no padding row is ever read.
// Both are compile-time variants: the N-token code is unchanged by lengths,
// and the length-aware one works in 32 bits (the tensor-core kernels take
// N < 2^31) to keep register pressure down.
template <bool VAR>
struct HeadTiles;

template <>
struct HeadTiles<false> {
  int64_t nb;   // the head's tokens (N)
  __device__ __forceinline__ HeadTiles(const int32_t* __restrict__, int64_t, int64_t N) : nb(N) {}
  __device__ __forceinline__ int64_t count(int T) const { return tiles_of(nb, T); }
  // token of row 0 of tile t
  __device__ __forceinline__ int64_t row0(int64_t t, int T) const { return t * T; }
  // row r of tile t is one of the tile's own tokens
  __device__ __forceinline__ bool own(int64_t t, int T, int r) const { return t * T + r < nb; }
  // the tile's own tokens are its columns [lo, hi)
  __device__ __forceinline__ int lo(int64_t, int) const { return 0; }
  __device__ __forceinline__ int hi(int64_t t, int T) const { return (int)imin64(T, nb - t * T); }
};

template <>
struct HeadTiles<true> {
  int nb;   // the batch element's length, clamped to [0, N]
  __device__ __forceinline__ HeadTiles(const int32_t* __restrict__ lens, int64_t b, int64_t N)
      : nb((int)seq_len(lens, b, N)) {}
  __device__ __forceinline__ int64_t count(int T) const { return (nb + T - 1) / T; }
  // token of row 0 of tile t: a partial last tile ends at nb (rows before
  // token 0 read as zeros)
  __device__ __forceinline__ int64_t row0(int64_t t, int T) const {
    const int s = (int)t * T;
    return s + T > nb ? nb - T : s;
  }
  __device__ __forceinline__ bool own(int64_t t, int T, int r) const {
    const int s = (int)t * T;
    return (s + T > nb ? nb - T : s) + r >= s;
  }
  __device__ __forceinline__ int lo(int64_t t, int T) const {
    const int x = ((int)t + 1) * T - nb;
    return x > 0 ? x : 0;
  }
  __device__ __forceinline__ int hi(int64_t, int T) const { return T; }
};

// Programmatic dependent launch.  A kernel launched by launch_pdl may be
// scheduled while the kernel before it in the stream is still running:
// pdl_wait() returns once that kernel has completed and its writes are
// visible (at once when there is none), so each such kernel calls it before
// touching global memory or tensor memory; pdl_trigger() lets the next
// kernel be scheduled as soon as every CTA of this one has started.  The
// next kernel's CTAs then wait on the SMs this one frees, and the launch gap
// between the two disappears.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The work of one CTA of a tensor-core kernel: head bh, its tiles [tile0,
// tile0 + ntiles), and the slot of the records (partials) it writes.
// Without lengths the grid is (chunks, BH) over the chunk plan; with them it
// is one CTA per unit of the work plan, and bh < 0 leaves the CTA idle.
struct CtaWork {
  int64_t bh, tile0, ntiles, slot;
};

template <bool VAR>
__device__ __forceinline__ CtaWork cta_work(const int4* __restrict__ units, int64_t chunk_tiles,
                                            int64_t tiles_per_bh) {
  CtaWork w;
  if constexpr (VAR) {
    const int4 u = units[blockIdx.x];
    w.bh = u.x;
    w.tile0 = u.y;
    w.ntiles = u.z;
    w.slot = blockIdx.x;
  } else {
    w.bh = blockIdx.y;
    w.tile0 = (int64_t)blockIdx.x * chunk_tiles;
    w.ntiles = imin64(chunk_tiles, tiles_per_bh - w.tile0);
    w.slot = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
  }
  return w;
}

// The slot of this CTA's records (the same as cta_work's).
template <bool VAR>
__device__ __forceinline__ int64_t cta_slot() {
  return VAR ? (int64_t)blockIdx.x : (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
}

// Records (partials) of head bh: `count` slots from `first`, by the work
// plan's head table when there is one, else the chunk plan's `chunks` per head.
__device__ __forceinline__ int2 head_slots(const int2* __restrict__ heads, int64_t bh, int chunks) {
  return heads ? heads[bh] : make_int2((int)(bh * chunks), chunks);
}

cudaError_t launch_simt_encode(const void* Q, int64_t qbs, const void* K, const void* V,
                               const Dims& d, flare_dtype_t dt, float scale,
                               const ChunkPlan& plan, float* part_ml, float* part_acc,
                               cudaStream_t st);
cudaError_t launch_simt_decode(const void* Q, int64_t qbs, const void* K, const float* Zf,
                               void* Y, const Dims& d, flare_dtype_t dt, float scale,
                               cudaStream_t st);
// Records kErrSeqLen when a length lies outside [0, N] (lens non-NULL).
cudaError_t launch_check_lens(const Dims& d, uint32_t* err, cudaStream_t st);
// The arguments of a work-plan block (flare_plan.cuh).
struct PlanArgs;
// Checks the lengths (as launch_check_lens) and writes the work plans of a
// tensor-core call with lengths into the workspace; returns d with them
// attached.  With `defer` the plan kernel is not launched: *defer receives
// its arguments (lens NULL when there is no plan), and the caller has the
// plan computed before any kernel that reads it (launch_bwd does, by a block
// of the backward's preparation kernel).
cudaError_t launch_var_plan(Dims& d, const WsLayout& L, char* ws, cudaStream_t st, int sms,
                            PlanArgs* defer = nullptr);
// Zeroes the padding rows (n >= the batch element's length) of the token
// tensor X0 with strides t0 and, when X1 is not NULL, of X1 (no-op when
// d.lens is NULL).
// The padding of X0 (and X1) for blocks of `threads` threads (x0 NULL
// without lengths).
PadZero pad_zero(void* X0, const Tok& t0, void* X1, const Tok& t1, const Dims& d, flare_dtype_t dt,
                 int threads);
cudaError_t launch_pad_zero(const PadZero& z, int64_t BH, cudaStream_t st);
// Records of head bh: slots_per_bh per head in each of `groups` blocks, or,
// when d carries the encode's work plan, its units of `sub` records.
cudaError_t launch_combine(const Dims& d, flare_dtype_t dt, int slots_per_bh, int sub, int groups,
                           const float* part_ml, const float* part_acc, float* Zf,
                           __nv_bfloat16* Zb, float* Z_save, float* lse_save, const void* Qpp,
                           void* Qdyn, cudaStream_t st, const PadZero* pz = nullptr);
cudaError_t launch_tc_encode(const void* Q, int64_t qbs, const void* K, const void* V,
                             const Dims& d, float scale, const ChunkPlan& plan,
                             float* part_ml, float* part_acc, uint32_t* err, cudaStream_t st);
cudaError_t launch_tc_decode(const void* Q, int64_t qbs, const void* K,
                             const __nv_bfloat16* Zb, void* Y, const Dims& d, float scale,
                             const ChunkPlan& plan, uint32_t* err, cudaStream_t st);
// Tensor-core backward with M = 256, decode stage.  launch_tc_bwd_stats: the
// decode pipeline with the backward's per-token statistics in place of Y
// (stats, dY'' = dY / g, the head's range flag).  launch_tc_dz: the encode
// pipeline with dY as V and the weights P_d = 2^(c S - mx'[n]), giving the
// chunk partials of dZ = P_d^T dY ([BH][slots][M][D], plan = the encode's).
cudaError_t launch_tc_bwd_stats(const void* Q, int64_t qbs, const void* K, const __nv_bfloat16* Zb,
                                const void* dY, const Dims& d, float scale, const ChunkPlan& plan,
                                const float* rref, float4* stats, __nv_bfloat16* dy2,
                                uint32_t* flags, uint32_t* err, cudaStream_t st);
cudaError_t launch_tc_dz(const void* Q, int64_t qbs, const void* K, const void* dY, const Dims& d,
                         float scale, const ChunkPlan& plan, const float4* stats, float* dz_part,
                         uint32_t* err, cudaStream_t st);
// 3-D TMA map over a bf16 tensor [depth][rows][D] (D in {16, 32}) with
// boxes of box_rows whole rows, swizzled to match the UMMA descriptors
// (64-byte swizzle for 64-byte rows, 32-byte for 32-byte rows).
cudaError_t make_map(CUtensorMap* m, const void* base, int D, int64_t rows, int64_t depth,
                     int box_rows);
// Stride of the flattened head index bh = b H + h of a token tensor, or -1
// when its batch and head dimensions do not flatten into one.
inline int64_t flat_stride(const Tok& t, const Dims& d) {
  if (d.B == 1) return t.sh;
  if (d.H == 1) return t.sb;
  return t.sb == d.H * t.sh ? t.sh : -1;
}
// True when K, V and dY all flatten (contiguous tensors do): the tensor-core
// kernels then take 3-D maps {D, N, B*H}, else 4-D maps {D, N, H, B}.
inline bool tok_flat(const Dims& d) {
  return flat_stride(d.k, d) > 0 && flat_stride(d.v, d) > 0 && flat_stride(d.dy, d) > 0;
}
// TMA map over a bf16 token tensor [B,H,N,D] with strides t: 3-D
// {D, N, B*H} when `flat`, else 4-D {D, N, H, B}; boxes of box_rows tokens
// of one head, swizzled as make_map.
cudaError_t make_tok_map(CUtensorMap* m, const void* base, const Dims& d, const Tok& t,
                         int box_rows, bool flat);

// Which part of the backward a call runs.  With the tokens sharded (context
// parallelism) each shard runs DZ (the decode stage over its tokens, then
// its part of dZ, written to `dz`), the shards' parts are summed, and each
// runs FINISH (the encode stage over its tokens given the summed dZ in `dz`:
// its rows of dK, dV and its fp32 part of dQ in `dq32`) on the same
// workspace.  ALL is the whole backward on one device.
enum class BwdPhase { ALL, DZ, FINISH };

cudaError_t launch_tc_bwd(const void* Q, int64_t qbs, const void* K, const void* V,
                          const void* dY, const float* Z, const float* lse, void* dQ, void* dK,
                          void* dV, const Dims& d, float scale, const WsLayout& L, char* ws,
                          cudaStream_t st, BwdPhase phase = BwdPhase::ALL, float* dz = nullptr,
                          float* dq32 = nullptr, const PadZero* pz = nullptr,
                          const PlanArgs* plan = nullptr);
// FLARE++'s first-encode gradient on the tensor cores (bf16, M = 128,
// D in {16, 32}): adds into dK, dV and writes dQ (sum over the batch of dZ1
// and the encode's dQ); reuses the tensor-core backward's workspace.
// With dq32 (a shard of a context-parallel backward) dQ is written in
// float32 and holds the encode's part, plus the sum over the batch of dZ1
// only when add_dz1 (one shard of the context-parallel group adds it).
cudaError_t launch_tc_enc_bwd(const void* Q, const void* K, const void* V, const float* Z1,
                              const float* lse1, const void* dZ1, void* dQ, void* dK, void* dV,
                              const Dims& d, float scale, const WsLayout& L, char* ws,
                              cudaStream_t st, float* dq32 = nullptr, bool add_dz1 = false);
cudaError_t launch_pp_bwd_tail(const void* Q, const void* K, const void* V, const float* z1,
                               const float* lse1, const void* dqd, void* dQ, void* dK, void* dV,
                               const Dims& d, flare_dtype_t dt, float scale, const WsLayout& L,
                               char* ws, cudaStream_t st, float* dq32 = nullptr,
                               bool add_dqd = false);
cudaError_t launch_bwd(const void* Q, int64_t qbs, const void* K, const void* V, const void* dY,
                       const float* Z, const float* lse, void* dQ, void* dK, void* dV,
                       const Dims& d, flare_dtype_t dt, float scale, const WsLayout& L,
                       char* ws, cudaStream_t st, BwdPhase phase = BwdPhase::ALL,
                       float* dz = nullptr, float* dq32 = nullptr, const PadZero* pz = nullptr,
                       const PlanArgs* plan = nullptr);

}  // namespace flare
