// sm_100a building blocks written as inline PTX: mbarriers with bounded
// waits, TMA tile loads, TMEM allocation / loads / stores, tcgen05.mma with
// shared-memory and tensor-memory operands, and the UMMA descriptors.
//
// Every wait is bounded by wall time (the global nanosecond timer): a wait
// that runs out returns false so the caller can record an error and leave,
// instead of spinning forever.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace flare {
namespace tc {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s
constexpr uint32_t kSuspendHintNs = 100000u;       // per poll; far below the bound

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking: true once the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes (or the hint expires) instead of re-issuing the poll.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// As mbar_wait, but suspended between polls: for waits whose spinning would
// take issue slots from the exponential-bound softmax warps on the same SM
// sub-partition.  Same bound; false on timeout.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity,
                                                uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait_sleep(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_sleep(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

// Waits for the phase with the given parity to complete; false once
// limit_ns have passed without it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

// Orders this thread's generic-proxy writes to shared memory before later
// async-proxy accesses of the same bytes (tcgen05.mma operand reads, TMA
// loads into a reused buffer).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA

// 3-D tiled bulk tensor load global -> shared, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];"
      ::"r"(smem_u32(dst)), "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
      : "memory");
}

// One box of a token tensor: tokens [tok, tok + box) of head bh = b H + h,
// through a 3-D map {D, N, B*H} (FLAT) or a 4-D map {D, N, H, B}.
template <bool FLAT>
__device__ __forceinline__ void tma_load_tok(void* dst, const CUtensorMap* map, uint64_t* bar,
                                             int32_t tok, int64_t bh, int H) {
  if constexpr (FLAT)
    tma_load_3d(dst, map, bar, 0, tok, (int32_t)bh);
  else
    tma_load_4d(dst, map, bar, 0, tok, (int32_t)(bh % H), (int32_t)(bh / H));
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// Starts moving the 128-byte line holding p into this SM's L1 (a hint: no
// register waits on it), so a load of it issued later finds it there.
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// ------------------------------------------------------ register split

// Warpgroup-wide: lower / raise this warpgroup's per-thread register limit.
template <int N>
__device__ __forceinline__ void regs_release() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_acquire() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- TMEM

// Whole-warp calls.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Waits for this thread's outstanding TMEM loads.  The registers of the load
// being consumed are passed through the asm as in/out operands, so the
// compiler cannot schedule any use of them before the wait.
__device__ __forceinline__ void tmem_wait_ld_dep(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane
// (warp's lane quarter base + t), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// tcgen05.wait::ld that names 16 loaded registers as in/out operands.
__device__ __forceinline__ void tmem_wait_ld_dep16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// tcgen05.wait::ld that names two loads' registers (32 + 16) as in/out
// operands, for a 48-column row read as two loads in flight together.
__device__ __forceinline__ void tmem_wait_ld_dep48(uint32_t (&r)[32], uint32_t (&q)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31]), "+r"(q[0]), "+r"(q[1]), "+r"(q[2]), "+r"(q[3]),
                 "+r"(q[4]), "+r"(q[5]), "+r"(q[6]), "+r"(q[7]), "+r"(q[8]), "+r"(q[9]),
                 "+r"(q[10]), "+r"(q[11]), "+r"(q[12]), "+r"(q[13]), "+r"(q[14]), "+r"(q[15])
               :
               : "memory");
}

// 32 lanes x 64 consecutive 32-bit columns in one load.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}

// tcgen05.wait::ld that names the 64 loaded registers as in/out operands.
__device__ __forceinline__ void tmem_wait_ld_dep64(uint32_t (&r)[64]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]), "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]), "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]), "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]), "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// ---------------------------------------------------------------- MMA

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor of kind::f16 with bf16 A/B and f32 accumulator.
// Fields: [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B
// format, [15] A major (0 = K), [16] B major (1 = MN), [17,23) N >> 3,
// [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major,
                                                      int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
         ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor (tcgen05 form).  Fields: [0,14) start
// address >> 4, [16,30) leading byte offset >> 4, [32,46) stride byte offset
// >> 4, [46,48) version = 1, [61,64) swizzle mode (4 = 64B, 6 = 32B).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint32_t swizzle_code) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(swizzle_code & 7u) << 61;
  return d;
}

// Swizzle mode that matches a row of `row_bytes` (the whole head dimension):
// 64-byte rows (D = 32 bf16) -> 64B swizzle, 32-byte rows (D = 16) -> 32B.
__host__ __device__ constexpr uint32_t umma_swizzle_code(int row_bytes) {
  return row_bytes == 64 ? 4u : 6u;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Warp votes.  Every branch that guards a warp-collective tcgen05 instruction
// (.sync.aligned loads, stores and waits) must be taken by all 32 lanes, so
// per-lane decisions in front of one go through these.
__device__ __forceinline__ bool warp_all(bool b) { return __all_sync(0xffffffffu, b); }
__device__ __forceinline__ bool warp_any(bool b) { return __any_sync(0xffffffffu, b); }

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Max of 32 values folded into four independent accumulators.
__device__ __forceinline__ void max_fold32(const uint32_t (&a)[32], float (&m)[4]) {
#pragma unroll
  for (int t = 0; t < 32; t += 8) {
    m[0] = max3(m[0], __uint_as_float(a[t + 0]), __uint_as_float(a[t + 1]));
    m[1] = max3(m[1], __uint_as_float(a[t + 2]), __uint_as_float(a[t + 3]));
    m[2] = max3(m[2], __uint_as_float(a[t + 4]), __uint_as_float(a[t + 5]));
    m[3] = max3(m[3], __uint_as_float(a[t + 6]), __uint_as_float(a[t + 7]));
  }
}

// The two bf16 halves of a packed pair, widened exactly to float.
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// 2^x on the FMA pipe, leaving the MUFU free for other exponentials.
// Single-split range reduction x = j + f with j = round(x) (the 1.5 * 2^23
// add puts round(x) in the low mantissa bits), f in [-1/2, 1/2]; 2^f by a
// degree-3 polynomial fitted by Remez exchange for minimum relative error
// (7.5e-5, see fit_exp2_poly.py); j is added to the result's exponent field.
// Exact enough for values that are rounded to bf16 next.  Valid for
// x <= 126; x below -125 is clamped (result 2^-125 instead of smaller).
__device__ __forceinline__ float exp2_fma(float x) {
  constexpr float kE0 = 0.9999280571937561f, kE1 = 0.6932609677314758f;
  constexpr float kE2 = 0.2426111251115799f, kE3 = 0.0551716685295105f;
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
  x = fmaxf(x, -125.0f);
  const float t = x + kRound;
  const float f = x - (t - kRound);
  float p = fmaf(kE3, f, kE2);
  p = fmaf(p, f, kE1);
  p = fmaf(p, f, kE0);
  return __uint_as_float((__float_as_uint(t) << 23) + __float_as_uint(p));
}

// Max of 16 values folded into four independent accumulators.
__device__ __forceinline__ void max_fold16(const uint32_t (&a)[16], float (&m)[4]) {
#pragma unroll
  for (int t = 0; t < 16; t += 8) {
    m[0] = max3(m[0], __uint_as_float(a[t + 0]), __uint_as_float(a[t + 1]));
    m[1] = max3(m[1], __uint_as_float(a[t + 2]), __uint_as_float(a[t + 3]));
    m[2] = max3(m[2], __uint_as_float(a[t + 4]), __uint_as_float(a[t + 5]));
    m[3] = max3(m[3], __uint_as_float(a[t + 6]), __uint_as_float(a[t + 7]));
  }
}

// p = 2^(a*c + neg) for 32 logits: packed into 16 bf16 pairs, sums folded
// into four independent accumulators.  With POLY_EVERY = k > 0, every k-th
// pair is computed on the FMA pipe (exp2_fma) instead of the MUFU.
template <int POLY_EVERY = 0, bool CLAMP_HI = false, bool SUM = true>
__device__ __forceinline__ void exp_pack32(const uint32_t (&a)[32], float c, float neg,
                                           uint32_t (&pk)[16], float (&s)[4]);

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Packed fp32x2 arithmetic (sm_100): one instruction for two lanes of
// float work, halving the issue slots of the scale-shift and the row sums.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void split_f32x2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x for a pair of values (x.lo, x.hi) on the FMA pipe, as exp2_fma but
// with the range reduction and the polynomial in packed fp32x2 arithmetic
// (one instruction for both values): two clamps, three packed adds, three
// packed FMAs and two exponent-field adds per pair.  The same
// coefficients, hence the same error bound (7.5e-5 relative) and domain
// (x <= 126; x below -125 gives 2^-125 times the polynomial).
__device__ __forceinline__ void exp2_fma_pair(uint64_t x, float& r0, float& r1) {
  constexpr float kE0 = 0.9999280571937561f, kE1 = 0.6932609677314758f;
  constexpr float kE2 = 0.2426111251115799f, kE3 = 0.0551716685295105f;
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
  float x0, x1;
  split_f32x2(x, x0, x1);
  const uint64_t xc = f32x2(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t rr = f32x2(kRound, kRound);
  const uint64_t t = add_f32x2(xc, rr);
  const uint64_t f = sub_f32x2(xc, sub_f32x2(t, rr));
  uint64_t p = fma_f32x2(f32x2(kE3, kE3), f, f32x2(kE2, kE2));
  p = fma_f32x2(p, f, f32x2(kE1, kE1));
  p = fma_f32x2(p, f, f32x2(kE0, kE0));
  float t0, t1, p0, p1;
  split_f32x2(t, t0, t1);
  split_f32x2(p, p0, p1);
  r0 = __uint_as_float((__float_as_uint(t0) << 23) + __float_as_uint(p0));
  r1 = __uint_as_float((__float_as_uint(t1) << 23) + __float_as_uint(p1));
}

// 2^(c a + neg) for a pair of raw logits (a0, a1) on the FMA pipe, with the
// exponent x = c a + neg clamped to [-125, 126] for free: the saturating FMA
// that computes y = (x + 125) / 251 = a cs + ns (cs = c / 251,
// ns = (neg + 125) / 251) clamps y to [0, 1].  Then x = 251 y - 125, its
// integer part j by round-to-nearest (t = 251 y + (1.5 * 2^23 - 125)) and
// f = 251 y - 125 - j in packed FMAs, 2^f by the Horner steps of
// exp2_fma, j added to the exponent field.  Error: the polynomial's
// 7.5e-5 plus the rounding of y (at most 251 * 2^-25 in x, 5.2e-6
// relative).  A clamped exponent keeps a large positive x finite (2^126),
// so a sum of such weights still exposes it.
__device__ __forceinline__ void exp2_fma_pair_logits(float a0, float a1, float cs, float ns,
                                                     float& r0, float& r1) {
  constexpr float kE0 = 0.9999280571937561f, kE1 = 0.6932609677314758f;
  constexpr float kE2 = 0.2426111251115799f, kE3 = 0.0551716685295105f;
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
  float y0, y1;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(y0) : "f"(a0), "f"(cs), "f"(ns));
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(y1) : "f"(a1), "f"(cs), "f"(ns));
  const uint64_t y = f32x2(y0, y1);
  const uint64_t w = f32x2(251.0f, 251.0f), r = f32x2(kRound - 125.0f, kRound - 125.0f);
  const uint64_t t = fma_f32x2(y, w, r);
  const uint64_t f = fma_f32x2(y, w, sub_f32x2(r, t));
  uint64_t p = fma_f32x2(f32x2(kE3, kE3), f, f32x2(kE2, kE2));
  p = fma_f32x2(p, f, f32x2(kE1, kE1));
  p = fma_f32x2(p, f, f32x2(kE0, kE0));
  float t0, t1, p0, p1;
  split_f32x2(t, t0, t1);
  split_f32x2(p, p0, p1);
  r0 = __uint_as_float((__float_as_uint(t0) << 23) + __float_as_uint(p0));
  r1 = __uint_as_float((__float_as_uint(t1) << 23) + __float_as_uint(p1));
}

// 2^(a*c + neg) for NP consecutive pairs of logits: bf16 pairs into pk, the
// values summed into s (s[0], s[2] collect even lanes, s[1], s[3] odd ones).
// CLAMP_HI: the polynomial pairs clamp their exponent to [-125, 126]
// (exp2_fma_pair_logits), for callers whose exponents can be large and
// positive; otherwise they use exp2_fma_pair (exponents known to be at most
// 126).
template <int NP, int POLY_EVERY, bool CLAMP_HI = false, bool SUM = true>
__device__ __forceinline__ void exp_pack_pairs(const uint32_t* a, float c, float neg,
                                               uint32_t* pk, float (&s)[4]) {
  const uint64_t c2 = f32x2(c, c), n2 = f32x2(neg, neg);
  const float cs = c * (1.0f / 251.0f), ns = (neg + 125.0f) * (1.0f / 251.0f);
  uint64_t acc[2] = {f32x2(s[0], s[1]), f32x2(s[2], s[3])};
#pragma unroll
  for (int t = 0; t < NP; ++t) {
    const bool poly = POLY_EVERY > 0 && (t % (POLY_EVERY > 0 ? POLY_EVERY : 1)) == POLY_EVERY - 1;
    float p0, p1;
    if (poly && CLAMP_HI) {
      exp2_fma_pair_logits(__uint_as_float(a[2 * t]), __uint_as_float(a[2 * t + 1]), cs, ns, p0,
                           p1);
    } else if (poly) {
      exp2_fma_pair(
          fma_f32x2(f32x2(__uint_as_float(a[2 * t]), __uint_as_float(a[2 * t + 1])), c2, n2), p0,
          p1);
    } else {
      const uint64_t x =
          fma_f32x2(f32x2(__uint_as_float(a[2 * t]), __uint_as_float(a[2 * t + 1])), c2, n2);
      float x0, x1;
      split_f32x2(x, x0, x1);
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    if (SUM) acc[t & 1] = add_f32x2(acc[t & 1], f32x2(p0, p1));
    pk[t] = pack_bf16(p0, p1);
  }
  split_f32x2(acc[0], s[0], s[1]);
  split_f32x2(acc[1], s[2], s[3]);
}

template <int POLY_EVERY, bool CLAMP_HI, bool SUM>
__device__ __forceinline__ void exp_pack32(const uint32_t (&a)[32], float c, float neg,
                                           uint32_t (&pk)[16], float (&s)[4]) {
  exp_pack_pairs<16, POLY_EVERY, CLAMP_HI, SUM>(a, c, neg, pk, s);
}

// p = 2^(a*c + neg) for 16 logits: 8 bf16 pairs, sums into four accumulators.
template <int POLY_EVERY = 0, bool CLAMP_HI = false, bool SUM = true>
__device__ __forceinline__ void exp_pack16(const uint32_t (&a)[16], float c, float neg,
                                           uint32_t (&pk)[8], float (&s)[4]) {
  exp_pack_pairs<8, POLY_EVERY, CLAMP_HI, SUM>(a, c, neg, pk, s);
}

}  // namespace tc
}  // namespace flare
