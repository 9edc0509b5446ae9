// sm_100a building blocks: shared-memory barriers, TMA tile loads, tcgen05
// MMAs with TMEM accumulators, and bounded waits.
//
// Everything here is inline PTX written from the public PTX ISA description
// of mbarrier, cp.async.bulk.tensor and the tcgen05 family.  Nothing here is
// specific to attention.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

// ---------------------------------------------------------------------------
// Device-side error word.  Kernels never trap: on a problem they record a code
// here and leave.  Defined here because the library is one translation unit.  The host reads and clears it with fa_device_status().
// Layout: bits 0..7 status code, bits 8..15 site, bits 16..31 block index.
// ---------------------------------------------------------------------------
__device__ unsigned int g_error_word = 0;

enum : unsigned {
  kErrDeviceTimeout = 6u,
  kErrDeviceSeqlen = 7u,
  kErrDeviceLayout = 9u,
  kErrDeviceScale = 11u  // an 8-bit descale factor (or a quantised tile's amax) not finite and > 0
};

__device__ __forceinline__ void record_error(unsigned code, unsigned site) {
  unsigned w = (code & 0xffu) | ((site & 0xffu) << 8) | ((blockIdx.x & 0xffffu) << 16);
  atomicCAS(&g_error_word, 0u, w);
}

// Optional device timeline (build with -DFA_TRACE): SM clock stamps of
// pipeline events of CTA 0, slot = iteration * 32 + event.  Compiled out by
// default.
#ifndef FA_TRACE_SM_THREAD
#define FA_TRACE_SM_THREAD 0  // the softmax thread whose events are recorded
#endif
#ifdef FA_TRACE
constexpr int kTraceSlots = 1 << 16;
__device__ unsigned long long g_trace[kTraceSlots];
#define FA_TRACE_AT(it, ev)                                                        \
  do {                                                                            \
    if (blockIdx.x == 0 && (it) < (kTraceSlots / 32))                             \
      g_trace[(it) * 32 + (ev)] = static_cast<unsigned long long>(clock64());     \
  } while (0)
#else
#define FA_TRACE_AT(it, ev) \
  do {                      \
  } while (0)
#endif

// Default bound of a pipeline wait: it gives up after this long and reports
// kErrDeviceTimeout.  No wait in a correct pipeline lasts more than
// microseconds.  The host may set another bound per launch (WaitCtl).
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// What a pipeline wait needs besides its barrier: the CTA-wide abort flag
// (in shared memory) and the bound of one wait in nanoseconds.
struct WaitCtl {
  volatile int* abort;
  unsigned long long limit_ns;
};

// Wait until the phase with the given parity has completed.  Returns false if
// the CTA-wide abort flag is raised or the wait runs past wc.limit_ns (in
// which case it records the error and raises the flag itself).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                          unsigned site) {
  const uint32_t a = smem_addr(bar);
  if (mbar_try_wait(a, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (*wc.abort) return false;
    if (globaltimer_ns() - t0 > wc.limit_ns) {
      record_error(kErrDeviceTimeout, site);
      *wc.abort = 1;
      return false;
    }
  }
}

// Warp-uniform wait: every lane polls, and the warp proceeds only if all
// lanes saw the phase complete, so .sync.aligned tcgen05 ops that follow are
// reached by the whole warp or by none of it.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, const WaitCtl& wc,
                                               unsigned site) {
  const bool ok = mbar_wait(bar, parity, wc, site);
  return __all_sync(0xffffffffu, ok);
}

// Agreement of `threads` threads (whole warps) that meet at named barrier
// `id`: true only if every one of them passes true.  Warps that share a
// named barrier later on decide together whether to go on, so that none of
// them waits there for a warp that has left.
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(ok ? 1u : 0u), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// Same, with an explicit (short) limit and no error report: used only while
// draining after an abort.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity,
                                                unsigned long long limit_ns) {
  const uint32_t a = smem_addr(bar);
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// TMA: 3-D tiled load global -> shared, completion counted on an mbarrier.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// TMA: 3-D tiled reduce-add shared -> global (fp32 add in L2), bulk group.
// Out-of-range elements of the box are skipped; x, y, z must be >= 0.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int x,
                                                  int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_addr(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Same, allowing the most recent group to still be reading.
__device__ __forceinline__ void bulk_wait_read_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Named barrier over a subset of the block's warps.
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation (warp-wide), MMA issue (one thread), commit, fences
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Move registers between warpgroups (all warps of a warpgroup execute it).
// The shares of all warpgroups must add up to at most the block's launch
// allocation (threads x registers per thread), or the increase never returns;
// launchers check the compiled register count before launching.
template <int N>
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on the mbarrier when every tcgen05 async op issued so far by
// this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Instruction descriptor, kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int M, int N, bool a_mn_major,
                                                 bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | ((bf16 ? 1u : 0u) << 7)                   // A format: f16 / bf16
         | ((bf16 ? 1u : 0u) << 10)                  // B format
         | ((a_mn_major ? 1u : 0u) << 15)            // A major-ness
         | ((b_mn_major ? 1u : 0u) << 16)            // B major-ness
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Instruction descriptor, kind::f8f6f4 with fp32 accumulation and both
// operands e4m3 (format code 0 for A and B; the same bit positions as
// kind::f16).  8-bit operands may be MN-major (e4m3 and e5m2 allow it).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7) | (0u << 10)                    // A, B format: e4m3
         | ((a_mn_major ? 1u : 0u) << 15)
         | ((b_mn_major ? 1u : 0u) << 16)
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Grouped MMAs: a whole K = 64 or K = 128 contraction (4 or 8 tcgen05.mma of
// K = 16) into one accumulator from one asm statement.  Every descriptor of
// the group is the 128-byte-swizzled descriptor of its first step plus an
// immediate offset on the start-address field, so a step costs one 32-bit add
// per shared operand; the accumulate predicate is set once.  Operands are
// given by the low descriptor word (start address >> 4 | leading byte offset
// >> 4 << 16, see sdesc_lo); the high word (stride byte offset 1024, sm_100
// version bit, 128-byte swizzle) is the same for every operand here.  The
// start-address field never carries into the next field: shared addresses
// stay below 256 KB.
// ---------------------------------------------------------------------------
constexpr uint32_t kSdescHi = (1024u >> 4) | (1u << 14) | (2u << 29);

// K-major operand (rows of 128 bytes, 64-element panels 16 KB apart): LBO 16.
// MN-major operand (64-element MN panels 16 KB apart): LBO 16384.
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t saddr, bool mn_major) {
  return ((saddr >> 4) & 0x3FFFu) | ((mn_major ? (16384u >> 4) : 1u) << 16);
}

// Start-address step (16-byte units) of K-step kk (16 elements of 16 bits):
// K-major walks 32 bytes inside a 64-element panel, then the next panel;
// MN-major walks 16 rows of 128 bytes.
__host__ __device__ constexpr uint32_t sw128_step(bool mn_major, int kk) {
  return mn_major ? static_cast<uint32_t>(kk) * 128u
                  : static_cast<uint32_t>(kk >> 2) * 1024u + static_cast<uint32_t>(kk & 3) * 2u;
}

#define FA_MMA_PROLOGUE                                                        \
  "{\n\t.reg .pred p, t;\n\t.reg .b32 h, a, b;\n\t.reg .b64 da, db;\n\t"       \
  "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\tmov.b32 h, %5;\n\t"
#define FA_MMA_SS_FIRST                                                        \
  "mov.b64 da, {%1, h};\n\tmov.b64 db, {%2, h};\n\t"                           \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n\t"
#define FA_MMA_SS_STEP(ao, bo)                                                 \
  "add.u32 a, %1, %" #ao ";\n\tadd.u32 b, %2, %" #bo ";\n\t"                   \
  "mov.b64 da, {a, h};\n\tmov.b64 db, {b, h};\n\t"                             \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t"
#define FA_MMA_TS_FIRST                                                        \
  "mov.b64 db, {%2, h};\n\t"                                                   \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %3, p;\n\t"
#define FA_MMA_TS_STEP(ao, bo)                                                 \
  "add.u32 a, %1, %" #ao ";\n\tadd.u32 b, %2, %" #bo ";\n\t"                   \
  "mov.b64 db, {b, h};\n\t"                                                    \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], db, %3, t;\n\t"

// D (+)= A B over K = 16 * NK (NK = 4 or 8), A and B in shared memory.
// accumulate = 0 overwrites D with the first step.
template <int NK, bool A_MN, bool B_MN>
__device__ __forceinline__ void umma_ss_group(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                              uint32_t idesc, uint32_t accumulate) {
  static_assert(NK == 4 || NK == 8, "group of 4 or 8 steps");
  if constexpr (NK == 8) {
    asm volatile(FA_MMA_PROLOGUE FA_MMA_SS_FIRST FA_MMA_SS_STEP(6, 13) FA_MMA_SS_STEP(7, 14)
                     FA_MMA_SS_STEP(8, 15) FA_MMA_SS_STEP(9, 16) FA_MMA_SS_STEP(10, 17)
                         FA_MMA_SS_STEP(11, 18) FA_MMA_SS_STEP(12, 19) "}" ::"r"(d_tmem),
                 "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kSdescHi),
                 "n"(sw128_step(A_MN, 1)), "n"(sw128_step(A_MN, 2)), "n"(sw128_step(A_MN, 3)),
                 "n"(sw128_step(A_MN, 4)), "n"(sw128_step(A_MN, 5)), "n"(sw128_step(A_MN, 6)),
                 "n"(sw128_step(A_MN, 7)), "n"(sw128_step(B_MN, 1)), "n"(sw128_step(B_MN, 2)),
                 "n"(sw128_step(B_MN, 3)), "n"(sw128_step(B_MN, 4)), "n"(sw128_step(B_MN, 5)),
                 "n"(sw128_step(B_MN, 6)), "n"(sw128_step(B_MN, 7))
                 : "memory");
  } else {
    asm volatile(FA_MMA_PROLOGUE FA_MMA_SS_FIRST FA_MMA_SS_STEP(6, 9) FA_MMA_SS_STEP(7, 10)
                     FA_MMA_SS_STEP(8, 11) "}" ::"r"(d_tmem),
                 "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kSdescHi),
                 "n"(sw128_step(A_MN, 1)), "n"(sw128_step(A_MN, 2)), "n"(sw128_step(A_MN, 3)),
                 "n"(sw128_step(B_MN, 1)), "n"(sw128_step(B_MN, 2)), "n"(sw128_step(B_MN, 3))
                 : "memory");
  }
}

// TMEM column step of K-step kk (16 elements of 16 bits = 8 columns): either
// contiguous, or split so that steps 4..7 sit 64 columns after steps 0..3.
__host__ __device__ constexpr uint32_t tmem_step(bool split, int kk) {
  return split ? static_cast<uint32_t>(kk >> 2) * 64u + static_cast<uint32_t>(kk & 3) * 8u
               : static_cast<uint32_t>(kk) * 8u;
}

// D (+)= A B over K = 128, A in TMEM (16-bit elements packed in pairs, laid
// out as tmem_step says), B in shared memory.
template <bool B_MN, bool A_SPLIT>
__device__ __forceinline__ void umma_ts_group8(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(FA_MMA_PROLOGUE FA_MMA_TS_FIRST FA_MMA_TS_STEP(6, 13) FA_MMA_TS_STEP(7, 14)
                   FA_MMA_TS_STEP(8, 15) FA_MMA_TS_STEP(9, 16) FA_MMA_TS_STEP(10, 17)
                       FA_MMA_TS_STEP(11, 18) FA_MMA_TS_STEP(12, 19) "}" ::"r"(d_tmem),
               "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kSdescHi),
               "n"(tmem_step(A_SPLIT, 1)), "n"(tmem_step(A_SPLIT, 2)), "n"(tmem_step(A_SPLIT, 3)),
               "n"(tmem_step(A_SPLIT, 4)), "n"(tmem_step(A_SPLIT, 5)), "n"(tmem_step(A_SPLIT, 6)),
               "n"(tmem_step(A_SPLIT, 7)), "n"(sw128_step(B_MN, 1)), "n"(sw128_step(B_MN, 2)),
               "n"(sw128_step(B_MN, 3)), "n"(sw128_step(B_MN, 4)), "n"(sw128_step(B_MN, 5)),
               "n"(sw128_step(B_MN, 6)), "n"(sw128_step(B_MN, 7))
               : "memory");
}
// 8-bit (e4m3) groups: K = 128 as 4 tcgen05.mma of K = 32 (32 bytes), kind
// f8f6f4.  In bytes the operands are laid out like a 16-bit operand with 64
// elements per row: K-major steps walk 32 bytes inside the 128-byte swizzled
// row, MN-major steps walk 32 rows (4096 bytes), and an A operand in TMEM
// holds four elements per 32-bit column (8 columns per step).
#define FA_MMA8_SS_FIRST                                                       \
  "mov.b64 da, {%1, h};\n\tmov.b64 db, {%2, h};\n\t"                           \
  "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %3, p;\n\t"
#define FA_MMA8_SS_STEP(ao, bo)                                                \
  "add.u32 a, %1, %" #ao ";\n\tadd.u32 b, %2, %" #bo ";\n\t"                   \
  "mov.b64 da, {a, h};\n\tmov.b64 db, {b, h};\n\t"                             \
  "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %3, t;\n\t"
#define FA_MMA8_TS_FIRST                                                       \
  "mov.b64 db, {%2, h};\n\t"                                                   \
  "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], db, %3, p;\n\t"
#define FA_MMA8_TS_STEP(ao, bo)                                                \
  "add.u32 a, %1, %" #ao ";\n\tadd.u32 b, %2, %" #bo ";\n\t"                   \
  "mov.b64 db, {b, h};\n\t"                                                    \
  "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [a], db, %3, t;\n\t"

// Start-address step (16-byte units) of 8-bit K-step kk (32 elements).
__host__ __device__ constexpr uint32_t sw128_step8(bool mn_major, int kk) {
  return mn_major ? static_cast<uint32_t>(kk) * 256u : static_cast<uint32_t>(kk) * 2u;
}

// D (+)= A B over K = 128 e4m3 elements, A and B in shared memory (K-major).
__device__ __forceinline__ void umma_ss_group4_e4m3(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(FA_MMA_PROLOGUE FA_MMA8_SS_FIRST FA_MMA8_SS_STEP(6, 9) FA_MMA8_SS_STEP(7, 10)
                   FA_MMA8_SS_STEP(8, 11) "}" ::"r"(d_tmem),
               "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kSdescHi),
               "n"(sw128_step8(false, 1)), "n"(sw128_step8(false, 2)), "n"(sw128_step8(false, 3)),
               "n"(sw128_step8(false, 1)), "n"(sw128_step8(false, 2)), "n"(sw128_step8(false, 3))
               : "memory");
}

// D (+)= A B over K = 128 e4m3 elements, A in TMEM (32 columns, 4 elements
// per column, ascending K in ascending bytes), B in shared memory MN-major.
__device__ __forceinline__ void umma_ts_group4_e4m3(uint32_t d_tmem, uint32_t a_tmem,
                                                    uint32_t b_lo, uint32_t idesc,
                                                    uint32_t accumulate) {
  asm volatile(FA_MMA_PROLOGUE FA_MMA8_TS_FIRST FA_MMA8_TS_STEP(6, 9) FA_MMA8_TS_STEP(7, 10)
                   FA_MMA8_TS_STEP(8, 11) "}" ::"r"(d_tmem),
               "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kSdescHi),
               "n"(8u), "n"(16u), "n"(24u),
               "n"(sw128_step8(true, 1)), "n"(sw128_step8(true, 2)), "n"(sw128_step8(true, 3))
               : "memory");
}
#undef FA_MMA8_SS_FIRST
#undef FA_MMA8_SS_STEP
#undef FA_MMA8_TS_FIRST
#undef FA_MMA8_TS_STEP
#undef FA_MMA_PROLOGUE
#undef FA_MMA_SS_FIRST
#undef FA_MMA_SS_STEP
#undef FA_MMA_TS_FIRST
#undef FA_MMA_TS_STEP

// ---------------------------------------------------------------------------
// TMEM <-> registers, 32 data-path lanes x 32 bit, 32 consecutive columns.
// The warp's lane quarter is fixed by (warp id % 4); taddr carries it.
// tmem_ld32 waits for its own load inside the same asm statement, so the
// compiler cannot move a use of the outputs above the wait.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
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

// N (8, 16 or 32) consecutive columns from a register array, by pointer
// (the caller's indices are compile-time after unrolling).
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t* r) {
  static_assert(N == 8 || N == 16 || N == 32, "8, 16 or 32 columns");
  if constexpr (N == 8) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
  } else if constexpr (N == 16) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
  } else {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
  }
}

// Wide TMEM moves (generated): 64 or 128 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64};"
               :
               : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
               : "memory");
}

// 128 consecutive columns as two 64-column loads (each instruction stays
// within a 128-register kernel limit), one wait.
__device__ __forceinline__ void tmem_ld64x2(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%129];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr), "r"(taddr + 64)
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Dropout masks: the counter-based generator Philox4x32-10 (Salmon, Moraes,
// Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011), from
// its published definition, and the quad-level data movement that hands each
// thread the bytes of its own scores.
// ---------------------------------------------------------------------------
// One call: 128-bit counter c, 64-bit key (k0, k1), 10 rounds.  A round forms
// the 64-bit products M0 c0 and M1 c2 and sets c = (hi1 ^ c1 ^ k0, lo1,
// hi0 ^ c3 ^ k1, lo0); the key is bumped by (W0, W1) between rounds.
__device__ __forceinline__ void philox_round(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
  const uint32_t hi0 = __umulhi(0xD2511F53u, c[0]), lo0 = 0xD2511F53u * c[0];
  const uint32_t hi1 = __umulhi(0xCD9E8D57u, c[2]), lo1 = 0xCD9E8D57u * c[2];
  const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
  c[0] = n0;
  c[1] = lo1;
  c[2] = n2;
  c[3] = lo0;
}

__device__ __forceinline__ void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    philox_round(c, k0, k1);
  }
}

// G independent calls with the same key, interleaved round by round.  A
// round is a chain of dependent multiplies (one call alone leaves the
// multiplier idle most of the time), so G calls in one stream keep it busy.
template <int G>
__device__ __forceinline__ void philox4x32_10_n(uint32_t (&c)[G][4], uint32_t k0, uint32_t k1) {
  // the round keys are rebuilt at each use (two adds a round, shared by the G
  // calls) rather than held in registers across the caller's loops
  asm volatile("" : "+r"(k0), "+r"(k1));
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) philox_round(c[g], k0, k1);
  }
}

// 4 x 4 transpose of words across the 4 lanes of a quad (w = lane & 3): on
// return a[s] holds what lane s held in a[w].  Two butterfly stages (lane
// distance 1, then 2); every lane of the warp must take part.
__device__ __forceinline__ void quad_transpose4(uint32_t (&a)[4], int w) {
#pragma unroll
  for (int m = 1; m <= 2; m <<= 1) {
    const bool hi = (w & m) != 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c & m) continue;
      const uint32_t send = hi ? a[c] : a[c | m];
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
      if (hi) a[c] = recv;
      else a[c | m] = recv;
    }
  }
}

// 4 x 4 byte transpose inside four words: byte q of x[c] becomes byte c of
// x[q] (byte permutes only).
__device__ __forceinline__ void byte_transpose4(uint32_t (&x)[4]) {
  const uint32_t t0 = __byte_perm(x[0], x[1], 0x5140), t1 = __byte_perm(x[0], x[1], 0x7362);
  const uint32_t t2 = __byte_perm(x[2], x[3], 0x5140), t3 = __byte_perm(x[2], x[3], 0x7362);
  x[0] = __byte_perm(t0, t2, 0x5410);
  x[1] = __byte_perm(t0, t2, 0x7632);
  x[2] = __byte_perm(t1, t3, 0x5410);
  x[3] = __byte_perm(t1, t3, 0x7632);
}

// (x & m) | (y & ~m)
__device__ __forceinline__ uint32_t bit_select(uint32_t x, uint32_t y, uint32_t m) {
  return (x & m) | (y & ~m);
}

// Keep flags of the four bytes of a at once, for a threshold t in 1..256:
// bit 8 c + 7 of the result is set iff byte c is below t; the other bits are
// unspecified.  With u = 256 - t, byte c is below t iff byte c + u stays below
// 256, i.e. the byte-wise sum does not carry out of bit 7: the low seven bits
// of each byte are added without carries between bytes, and the carry out is
// the majority of the two high bits and the carry into bit 7.
// u_lo7 = (u & 0x7F) * 0x01010101, u_all = u * 0x01010101.
__device__ __forceinline__ uint32_t keep_flags4(uint32_t a, uint32_t u_lo7, uint32_t u_all) {
  const uint32_t s7 = (a & 0x7F7F7F7Fu) + u_lo7;
  return ~((a & u_all) | (a & s7) | (u_all & s7));
}

// Four words of keep flags (bit 8 c + 7 of f_s) into one: the flag of byte c
// of f_s goes to bit 8 c + 7 - s; bits 8 c .. 8 c + 3 are unspecified.
__device__ __forceinline__ uint32_t merge_flags4(uint32_t f0, uint32_t f1, uint32_t f2,
                                                 uint32_t f3) {
  const uint32_t x = bit_select(f0, f1 >> 1, 0x80808080u);  // bits 8c+7, 8c+6
  const uint32_t y = bit_select(f2 >> 2, f3 >> 3, 0x20202020u);  // bits 8c+5, 8c+4
  return bit_select(x, y, 0xC0C0C0C0u);
}

// A 16-bit pair mask from keep flags: the low half is all ones iff bit 7 of
// byte 2 k of flags is set, the high half iff bit 7 of byte 2 k + 1 is (byte
// permute with replication of the selected byte's sign bit).
__device__ __forceinline__ uint32_t pair_keep_mask(uint32_t flags, int k) {
  uint32_t m;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(m) : "r"(flags), "r"(k ? 0xBBAAu : 0x9988u));
  return m;
}

// A 32-bit mask from keep flags: all ones iff bit 7 of byte c of flags is set.
__device__ __forceinline__ uint32_t word_keep_mask(uint32_t flags, int c) {
  uint32_t m;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(m) : "r"(flags), "r"((8u | c) * 0x1111u));
  return m;
}

// ---------------------------------------------------------------------------
// small numeric helpers (hardware instructions, no library math)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two fp32 lanes in one 64-bit register: (lo, hi).
__device__ __forceinline__ unsigned long long f2pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// a * b + c on both lanes
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long fadd2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long fmul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log2(x) (hardware approximation, relative error about 2^-22), x > 0.
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) return pack_bf16x2(lo, hi);
  else return pack_f16x2(lo, hi);
}

// The two 16-bit values of a pair back to fp32 (exact).
template <bool BF16>
__device__ __forceinline__ void unpack2(uint32_t w, float& lo, float& hi) {
  if constexpr (BF16) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
  } else {
    uint16_t a = static_cast<uint16_t>(w), b = static_cast<uint16_t>(w >> 16);
    asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(a));
    asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(b));
  }
}

// Two fp32 values to two e4m3 bytes (round to nearest even, saturating to
// +-448): lo in bits 0..7, hi in bits 8..15.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return static_cast<uint32_t>(r);
}
// Four fp32 values to one word of e4m3 bytes, a0 in bits 0..7.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a0, float a1, float a2, float a3) {
  return pack_e4m3x2(a0, a1) | (pack_e4m3x2(a2, a3) << 16);
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core operand reads, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

}  // namespace fa
