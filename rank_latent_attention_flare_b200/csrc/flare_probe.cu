// Measurement and self-test support (not part of the method).
//
// flare_probe_unit_rates: throughput microbenchmarks of the units that bound
// the FLARE kernels -- the MUFU exponential (ex2.approx.ftz.f32, what every
// softmax weight costs), the fp32 FMA pipe (fma.rn.f32 and the packed
// fma.rn.f32x2 that the polynomial exponential uses) and a mix of the two
// at the issue rate -- each timed with CUDA events over enough work to hide
// the launch, with the SM clock read inside the kernels (clock64 against the
// global nanosecond timer) so that every rate is also given per clock.
//
// flare_probe_mma_rate: the time a tcgen05.mma of the kernels' shapes
// (kind::f16, M = 128, K = 16, N tokens or latents) takes an SM, with its
// A operand in shared memory or in TMEM and one to four threads of the SM
// issuing at once, so that the cost of a product can be told apart from the
// issue latency of one thread.
//
// flare_eval_exp2: the kernels' exponentials (the MUFU one and the
// FMA-pipe polynomial, scalar and packed) evaluated element by element, so
// that a test can hold them against their stated error bounds.
//
// flare_selftest_wait_timeout: a kernel that waits, with the same bounded
// wait the FLARE kernels use, on an mbarrier that nothing ever arrives on,
// after allocating TMEM and starting a bulk copy as those kernels do; when the
// wait runs out it records its site in the workspace error word, lets the
// copy land, frees TMEM and returns, so that flare_device_status then
// reports FLARE_ERR_DEVICE_TIMEOUT with the device still usable.
#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

#include "flare_internal.cuh"
#include "tc_primitives.cuh"

namespace flare {
namespace {

using namespace tc;

constexpr int kProbeThreads = 256;
constexpr int kProbeBlocksPerSm = 4;
constexpr int kChains = 8;

// Per block: clock64 and globaltimer at the start and at the end (thread 0).
struct ClockRec {
  unsigned long long c0, c1, t0, t1;
};

__device__ __forceinline__ void rec_start(ClockRec* r, unsigned long long& c0,
                                          unsigned long long& t0) {
  if (threadIdx.x == 0) {
    c0 = clock64();
    t0 = globaltimer();
  }
  (void)r;
}

__device__ __forceinline__ void rec_end(ClockRec* r, unsigned long long c0, unsigned long long t0) {
  __syncthreads();
  if (threadIdx.x == 0) {
    ClockRec v;
    v.c0 = c0;
    v.t0 = t0;
    v.c1 = clock64();
    v.t1 = globaltimer();
    r[blockIdx.x] = v;
  }
}

// kChains independent chains x <- 2^-x per thread (fixed point near 0.64).
__global__ void __launch_bounds__(kProbeThreads) probe_ex2_kernel(int iters, float seed,
                                                                  float* sink, ClockRec* rec) {
  float x[kChains];
#pragma unroll
  for (int k = 0; k < kChains; ++k) x[k] = seed + 1e-3f * k + 1e-6f * threadIdx.x;
  unsigned long long c0 = 0, t0 = 0;
  __syncthreads();
  rec_start(rec, c0, t0);
#pragma unroll 1
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int k = 0; k < kChains; ++k) x[k] = ex2(-x[k]);
  }
  rec_end(rec, c0, t0);
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kChains; ++k) s += x[k];
  if (s == 1234.5f) sink[blockIdx.x] = s;   // never true; keeps the chains live
}

// kChains independent chains x <- x a + b (scalar fma.rn.f32).
__global__ void __launch_bounds__(kProbeThreads) probe_fma_kernel(int iters, float seed,
                                                                  float* sink, ClockRec* rec) {
  float x[kChains];
#pragma unroll
  for (int k = 0; k < kChains; ++k) x[k] = seed + 1e-3f * k + 1e-6f * threadIdx.x;
  const float a = 0.99990f, b = 1e-4f;
  unsigned long long c0 = 0, t0 = 0;
  __syncthreads();
  rec_start(rec, c0, t0);
#pragma unroll 1
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int k = 0; k < kChains; ++k) x[k] = fmaf(x[k], a, b);
  }
  rec_end(rec, c0, t0);
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kChains; ++k) s += x[k];
  if (s == 1234.5f) sink[blockIdx.x] = s;
}

// kChains independent packed chains (two fp32 FMAs per fma.rn.f32x2).
__global__ void __launch_bounds__(kProbeThreads) probe_fma2_kernel(int iters, float seed,
                                                                   float* sink, ClockRec* rec) {
  uint64_t x[kChains];
#pragma unroll
  for (int k = 0; k < kChains; ++k)
    x[k] = f32x2(seed + 1e-3f * k + 1e-6f * threadIdx.x, seed - 1e-3f * k);
  const uint64_t a = f32x2(0.99990f, 0.99991f), b = f32x2(1e-4f, 1e-4f);
  unsigned long long c0 = 0, t0 = 0;
  __syncthreads();
  rec_start(rec, c0, t0);
#pragma unroll 1
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int k = 0; k < kChains; ++k) x[k] = fma_f32x2(x[k], a, b);
  }
  rec_end(rec, c0, t0);
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kChains; ++k) {
    float lo, hi;
    split_f32x2(x[k], lo, hi);
    s += lo + hi;
  }
  if (s == 1234.5f) sink[blockIdx.x] = s;
}

// Mixed: per step, kChains exponentials and 6 x kChains scalar FMAs on
// independent chains -- seven of every eight issue slots of an SM
// sub-partition, with one MUFU instruction in each eight.
__global__ void __launch_bounds__(kProbeThreads) probe_mix_kernel(int iters, float seed,
                                                                  float* sink, ClockRec* rec) {
  float x[kChains], y[kChains];
#pragma unroll
  for (int k = 0; k < kChains; ++k) {
    x[k] = seed + 1e-3f * k + 1e-6f * threadIdx.x;
    y[k] = seed - 1e-3f * k;
  }
  const float a = 0.99990f, b = 1e-4f;
  unsigned long long c0 = 0, t0 = 0;
  __syncthreads();
  rec_start(rec, c0, t0);
#pragma unroll 1
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int k = 0; k < kChains; ++k) {
        x[k] = ex2(-x[k]);
        y[k] = fmaf(y[k], a, b);
        y[k] = fmaf(y[k], a, b);
        y[k] = fmaf(y[k], a, b);
        y[k] = fmaf(y[k], a, b);
        y[k] = fmaf(y[k], a, b);
        y[k] = fmaf(y[k], a, b);
      }
  }
  rec_end(rec, c0, t0);
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kChains; ++k) s += x[k] + y[k];
  if (s == 1234.5f) sink[blockIdx.x] = s;
}

__global__ void eval_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n,
                                 int form) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i >= n) return;
  const float x0 = x[2 * i];
  const float x1 = (2 * i + 1 < n) ? x[2 * i + 1] : 0.f;
  float r0, r1;
  if (form == 0) {
    r0 = ex2(x0);
    r1 = ex2(x1);
  } else if (form == 1) {
    r0 = exp2_fma(x0);
    r1 = exp2_fma(x1);
  } else if (form == 2) {
    exp2_fma_pair(f32x2(x0, x1), r0, r1);
  } else {
    // the form the softmax loops use: 2^(c a + neg) with c = 1, neg = 0
    exp2_fma_pair_logits(x0, x1, 1.0f / 251.0f, 125.0f / 251.0f, r0, r1);
  }
  y[2 * i] = r0;
  if (2 * i + 1 < n) y[2 * i + 1] = r1;
}

constexpr uint32_t kErrSelftestWait = 0x701;

// One CTA of 128 threads.  Warp 0 owns TMEM; thread 32 starts a bulk copy
// of 256 bytes of the workspace into shared memory (completing on `copied`);
// thread 0 waits on `never`, which nothing arrives on, for limit_ns, then
// records the site and raises the CTA's abort flag.  Warps 1-3 watch the
// flag (bounded).  The copy is waited for (bounded by the library's usual
// limit), every thread meets at the CTA barrier, TMEM is freed and the CTA
// exits.
__global__ void __launch_bounds__(128) selftest_wait_kernel(const uint8_t* __restrict__ src,
                                                            uint32_t* __restrict__ err,
                                                            uint64_t limit_ns) {
  __shared__ __align__(128) uint8_t buf[256];
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  uint64_t* never = &bars[0];
  uint64_t* copied = &bars[1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(never, 1);
    mbar_init(copied, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_slot, 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 32) {
    mbar_arrive_expect_tx(copied, 256);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 256, [%2];"
        ::"r"(smem_u32(buf)), "l"(src), "r"(smem_u32(copied))
        : "memory");
  }
  if (threadIdx.x == 0) {
    if (!mbar_wait(never, 0, limit_ns)) {
      record_error(err, kErrSelftestWait);
      abort_flag = 1;
    }
  } else if (warp > 0 && lane == 0) {
    const uint64_t t0 = globaltimer();
    while (!abort_flag && globaltimer() - t0 < kWaitLimitNs) {
    }
  }
  __syncwarp();
  if (threadIdx.x == 32) mbar_wait_sleep(copied, 0);   // the copy lands before exit
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 32);
}

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

// One CTA per SM (its shared memory keeps a second one out); warps 0 ..
// issuers - 1 each issue `reps` products of N columns into their own TMEM
// columns (A from TMEM: its own 8 columns from column 256) on zeroed
// operands, then wait for them to complete (bounded).  Each issuer records
// its clocks from the first issue to the completion.
struct MmaRec {
  unsigned long long clk;
  unsigned ok, pad;
};

template <int N, bool TS>
__global__ void __launch_bounds__(128, 1) probe_mma_kernel(int reps, int issuers, MmaRec* out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t bar[4];
  __shared__ uint32_t slot;
  // A: 128 rows x 64 bytes, B: up to 256 rows x 64 bytes, all zero
  for (int i = threadIdx.x; i < (128 + 256) * 64 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int k = 0; k < 4; ++k) mbar_init(&bar[k], 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) tmem_alloc(&slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = slot;
  const int w = threadIdx.x >> 5;
  if (w < issuers && (threadIdx.x & 31) == 0) {
    const uint64_t da = smem_desc(smem_u32(sm), 16, 8 * 64, umma_swizzle_code(64));
    const uint64_t db = smem_desc(smem_u32(sm + 128 * 64), 16, 8 * 64, umma_swizzle_code(64));
    constexpr uint32_t id = idesc_bf16_f32(128, N, 0, 0);
    const unsigned long long t0 = clock64();
    for (int i = 0; i < reps; ++i) {
      if (TS)
        mma_ts(tmem + N * w, tmem + 256 + 8 * w, db, id, 1u);
      else
        mma_ss(tmem + N * w, da, db, id, i > 0 ? 1u : 0u);
    }
    mma_commit(&bar[w]);
    const bool ok = mbar_wait(&bar[w], 0);
    out[blockIdx.x * 4 + w] = MmaRec{clock64() - t0, ok ? 1u : 0u, 0u};
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tmem, 512);
}

template <int N, bool TS>
cudaError_t launch_probe_mma(int sms, int reps, int issuers, MmaRec* out, cudaStream_t st) {
  const int smem = 120 * 1024;   // one CTA per SM
  cudaError_t e =
      cudaFuncSetAttribute(probe_mma_kernel<N, TS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  probe_mma_kernel<N, TS><<<sms, 128, smem, st>>>(reps, issuers, out);
  return cudaPeekAtLastError();
}

}  // namespace
}  // namespace flare

using flare::ClockRec;

extern "C" flare_status_t flare_probe_mma_rate(int n, int a_in_tmem, int issuers, void* scratch,
                                               size_t scratch_bytes, double* clk_per_mma,
                                               void* stream) {
  using namespace flare;
  if (clk_per_mma == nullptr || scratch == nullptr) return FLARE_ERR_INVALID_ARG;
  if (issuers < 1 || issuers > 4) return FLARE_ERR_INVALID_ARG;
  if (n != 32 && n != 48 && n != 64 && n != 128 && n != 256) return FLARE_ERR_UNSUPPORTED;
  if (n * issuers > 256) return FLARE_ERR_UNSUPPORTED;   // each issuer's TMEM columns
  const int sms = sm_count();
  if (sms <= 0) return FLARE_ERR_CUDA;
  if (scratch_bytes < (size_t)sms * 4 * sizeof(MmaRec) || ((uintptr_t)scratch & 15u))
    return FLARE_ERR_WORKSPACE;
  MmaRec* rec = (MmaRec*)scratch;
  cudaStream_t st = (cudaStream_t)stream;
  const int reps = 1024;
  cudaError_t e = cudaSuccess;
  // one untimed launch (code load, clocks), then the measured one
  for (int rep = 0; rep < 2 && e == cudaSuccess; ++rep) {
#define FLARE_PROBE_MMA(NN)                                                          \
  e = a_in_tmem ? launch_probe_mma<NN, true>(sms, reps, issuers, rec, st)            \
                : launch_probe_mma<NN, false>(sms, reps, issuers, rec, st)
    if (n == 32) FLARE_PROBE_MMA(32);
    else if (n == 48) FLARE_PROBE_MMA(48);
    else if (n == 64) FLARE_PROBE_MMA(64);
    else if (n == 128) FLARE_PROBE_MMA(128);
    else FLARE_PROBE_MMA(256);
#undef FLARE_PROBE_MMA
  }
  std::vector<MmaRec> host((size_t)sms * 4);
  if (e != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess ||
      cudaMemcpy(host.data(), rec, host.size() * sizeof(MmaRec), cudaMemcpyDeviceToHost) !=
          cudaSuccess) {
    note_error("flare_probe_mma_rate: probe kernel failed (%s)", cudaGetErrorName(cudaGetLastError()));
    return FLARE_ERR_CUDA;
  }
  // per SM: the issuers' products share it, so its clocks per product are
  // the slowest issuer's span over all of them; the median over the SMs
  std::vector<double> per_sm;
  for (int b = 0; b < sms; ++b) {
    unsigned long long span = 0;
    for (int w = 0; w < issuers; ++w) {
      const MmaRec& r = host[(size_t)b * 4 + w];
      if (!r.ok) return FLARE_ERR_DEVICE_TIMEOUT;
      span = r.clk > span ? r.clk : span;
    }
    per_sm.push_back((double)span / ((double)reps * issuers));
  }
  std::sort(per_sm.begin(), per_sm.end());
  *clk_per_mma = per_sm[per_sm.size() / 2];
  return FLARE_OK;
}

extern "C" size_t flare_probe_scratch_bytes(void) {
  const int sms = flare::sm_count();
  if (sms <= 0) return 0;
  return (size_t)sms * flare::kProbeBlocksPerSm * (sizeof(ClockRec) + sizeof(float));
}

extern "C" flare_status_t flare_probe_unit_rates(void* scratch, size_t scratch_bytes,
                                                 flare_unit_rates_t* out, void* stream) {
  using namespace flare;
  if (out == nullptr || scratch == nullptr) return FLARE_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return FLARE_ERR_CUDA;
  const int blocks = sms * kProbeBlocksPerSm;
  if (scratch_bytes < flare_probe_scratch_bytes() || ((uintptr_t)scratch & 15u))
    return FLARE_ERR_WORKSPACE;
  ClockRec* rec = (ClockRec*)scratch;
  float* sink = (float*)(rec + blocks);
  cudaStream_t st = (cudaStream_t)stream;
  std::vector<ClockRec> host(blocks);
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
    note_error("flare_probe_unit_rates: cudaEventCreate failed");
    return FLARE_ERR_CUDA;
  }
  // ops per thread per iteration: 4 x kChains of the probed instruction
  struct Probe {
    void (*k)(int, float, float*, ClockRec*);
    int iters;
    double ops_per_iter;   // results (exponentials or fp32 FMAs) per thread per iteration
    double* rate;
    double* ms;
  };
  double mix_fma = 0.0;
  Probe probes[4] = {
      {probe_ex2_kernel, 4096, 4.0 * kChains, &out->ex2_per_clk_sm, &out->ex2_ms},
      {probe_fma_kernel, 16384, 4.0 * kChains, &out->fma_per_clk_sm, &out->fma_ms},
      {probe_fma2_kernel, 8192, 8.0 * kChains, &out->fma2_per_clk_sm, &out->fma2_ms},
      {probe_mix_kernel, 2048, 4.0 * kChains, &out->mix_ex2_per_clk_sm, &out->mix_ms},
  };
  double mhz_sum = 0.0;
  flare_status_t status = FLARE_OK;
  for (int p = 0; p < 4 && status == FLARE_OK; ++p) {
    // one untimed launch (clocks ramp, code loads), then the timed one
    for (int rep = 0; rep < 2; ++rep) {
      if (rep == 1) cudaEventRecord(e0, st);
      probes[p].k<<<blocks, kProbeThreads, 0, st>>>(probes[p].iters, 0.5f, sink, rec);
      if (rep == 1) cudaEventRecord(e1, st);
    }
    if (cudaPeekAtLastError() != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
        cudaMemcpy(host.data(), rec, blocks * sizeof(ClockRec), cudaMemcpyDeviceToHost) !=
            cudaSuccess) {
      note_error("flare_probe_unit_rates: probe kernel %d failed (%s)", p,
                 cudaGetErrorName(cudaGetLastError()));
      status = FLARE_ERR_CUDA;
      break;
    }
    float ms = 0.f;
    cudaEventElapsedTime(&ms, e0, e1);
    double clk = 0.0, ns = 0.0;
    for (const ClockRec& r : host) {
      clk += (double)(r.c1 - r.c0);
      ns += (double)(r.t1 - r.t0);
    }
    const double mhz = ns > 0 ? 1e3 * clk / ns : 0.0;
    mhz_sum += mhz;
    const double ops = (double)blocks * kProbeThreads * probes[p].iters * probes[p].ops_per_iter;
    *probes[p].ms = ms;
    *probes[p].rate = (ms > 0 && mhz > 0) ? ops / (ms * 1e-3) / (mhz * 1e6) / sms : 0.0;
    if (p == 3) mix_fma = 6.0 * *probes[p].rate;
  }
  out->mix_fma_per_clk_sm = mix_fma;
  out->sms = sms;
  out->sm_mhz = mhz_sum / 4.0;
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  return status;
}

extern "C" flare_status_t flare_exp_split(int kernel, int64_t M, int64_t D, flare_dtype_t dtype,
                                          double* poly_fraction) {
  if (poly_fraction == nullptr || (kernel != 0 && kernel != 1)) return FLARE_ERR_INVALID_ARG;
  if ((D != 16 && D != 32) || M < 16 || M > 256 || (M % 16) != 0 ||
      (dtype != FLARE_F32 && dtype != FLARE_BF16))
    return FLARE_ERR_UNSUPPORTED;
  const flare::Path p = flare::choose_path(1, M, D, dtype);
  const int Mp = flare::tc_latent_tile(M);
  *poly_fraction = !p.tc_fwd ? 0.0
                             : (kernel == 0 ? flare::enc_poly_fraction(Mp)
                                            : flare::dec_poly_fraction(Mp));
  return FLARE_OK;
}

extern "C" flare_status_t flare_eval_exp2(const float* x, float* y, int64_t n, int form,
                                          void* stream) {
  if (n < 0 || form < 0 || form > 3) return FLARE_ERR_INVALID_ARG;
  if (n == 0) return FLARE_OK;
  if (x == nullptr || y == nullptr) return FLARE_ERR_INVALID_ARG;
  const int64_t pairs = (n + 1) / 2;
  const int threads = 256;
  const int64_t grid = (pairs + threads - 1) / threads;
  if (grid > 0x7fffffff) return FLARE_ERR_UNSUPPORTED;
  flare::eval_exp2_kernel<<<(unsigned)grid, threads, 0, (cudaStream_t)stream>>>(x, y, n, form);
  if (cudaPeekAtLastError() != cudaSuccess) {
    flare::note_error("flare_eval_exp2: launch failed (%s)", cudaGetErrorName(cudaGetLastError()));
    return FLARE_ERR_CUDA;
  }
  return FLARE_OK;
}

extern "C" flare_status_t flare_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                      uint64_t limit_ns, void* stream) {
  if (workspace == nullptr || workspace_bytes < 512 || ((uintptr_t)workspace & 255u))
    return FLARE_ERR_WORKSPACE;
  if (limit_ns > flare::tc::kWaitLimitNs) return FLARE_ERR_INVALID_ARG;
  uint8_t* ws = (uint8_t*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, 4, st) != cudaSuccess) {
    flare::note_error("flare_selftest_wait_timeout: clearing the error word failed");
    return FLARE_ERR_CUDA;
  }
  flare::selftest_wait_kernel<<<1, 128, 0, st>>>(ws + 256, (uint32_t*)ws, limit_ns);
  if (cudaPeekAtLastError() != cudaSuccess) {
    flare::note_error("flare_selftest_wait_timeout: launch failed (%s)",
                      cudaGetErrorName(cudaGetLastError()));
    return FLARE_ERR_CUDA;
  }
  return FLARE_OK;
}
