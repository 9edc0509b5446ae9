// Backward exact attention on sm_100a, by recomputation.
//
// "How Flash Attention Works" (swarnava.dev), section "The Backward Pass:
// Recomputation Instead of Stored Activations": only O and the per-row
// statistics are kept from the forward pass; the score tiles are recomputed
// tile by tile inside one fused kernel.  The statistic kept here is the
// log-sum-exp LSE_i, so P_ij = exp(scale * s_ij - LSE_i) is rebuilt exactly.
// With D_i = <dO_i, O_i> (the softmax-backward row term), the gradients are
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dQ = scale dS K,
//   dK = scale dS^T Q.
//
// Three kernels:
//  1. fa_bwd_pre: D_i = sum_c dO_ic O_ic (fp32) and zero the fp32 dQ
//     accumulator;
//  2. fa_bwd_kernel (persistent, one CTA per SM, 512 threads): a work unit is
//     (batch*head, 128-key tile j).  K_j and V_j stay in shared memory while
//     the query tiles i (i >= j when causal) stream past:
//       S^T  = K_j Q_i^T      (tcgen05, TMEM region A, keys on lanes)
//       P^T  = exp2(c S^T - LSE_i log2 e)  (warps 0-7, one key row and half
//                              the queries per thread; to region B as 16-bit)
//       dP^T = V_j dO_i^T     (region A, once S^T has been loaded out of it)
//       dS^T = P^T * (dP^T - D_i)  (warps 0-7, from dP^T and the 16-bit P^T;
//                              to a swizzled shared-memory tile)
//       dV_j += P^T dO_i,  dK_j += dS^T Q_i   (TMEM accumulators)
//       dQ_i  = dS K_j     (region B, once dV has read P^T out of it; warps
//                           8-11 add it into the fp32 accumulator in global
//                           memory with TMA reduce-adds)
//     warp 12 issues the MMAs, warp 13 the TMA loads, warp 14 stages LSE_i
//     and D_i in shared memory; warps 8-11 also write dK_j (times scale) and
//     dV_j at the end of the unit;
//  3. fa_bwd_post: dQ = scale * accumulator, rounded to 16-bit.
//
// TMEM columns: region A [0,128) holds S^T(i), then dP^T(i); region B
// [128,256) holds P^T(i) (16-bit, columns 0-31 and 64-95 of the region; with
// dropout the unmasked copy in 32-63 and 96-127), then dQ(i); dV [256,256+d),
// dK [256+d,256+2d).  Each region is handed on as soon as its contents have
// been read, so no MMA waits for work that does not produce its operands.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

template <int D>
struct BwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kPanelBytes = 128 * 64 * 2;
  static constexpr int kPanels = D / 64;
  static constexpr int kK = 0;
  static constexpr int kV = kTileBytes;
  static constexpr int kSlot = 2 * kTileBytes;         // Q_i in slots 0/1 (alternating), dO_i in 2
  static constexpr int kSlots = 3;
  static constexpr int kDS = kSlot + kSlots * kTileBytes;  // dS^T, 128 x 128 16-bit
  static constexpr int kSTG = kDS + 128 * 128 * 2;     // dQ staging: two [128][32] fp32
  static constexpr int kLSE = kSTG + 2 * 32 * 128 * 4; // 2 stages x 128 fp32
  static constexpr int kDSUM = kLSE + 2 * 128 * 4;     // 2 stages x 128 fp32
  static constexpr int kBar = kDSUM + 2 * 128 * 4;
  static constexpr int kBarBytes = 256;
  static constexpr int kUsed = kBar + kBarBytes;
  static constexpr int kSmemMax = 232448;              // sm_100 per-block opt-in maximum
  static constexpr int kSmemBytes = (kUsed + 1024 <= kSmemMax) ? kUsed + 1024 : kSmemMax;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColA = 0;    // S^T(i), then dP^T(i)
  static constexpr uint32_t kColB = 128;  // P^T(i) (16-bit), then dQ(i)
  static constexpr uint32_t kColDV = 256;
  static constexpr uint32_t kColDK = 256 + D;
};

struct BwdUnit {
  int bh, j, L, i0, ni;
  int nq;             // query tiles of the slice that are computed
  int z, row0, rows;  // slice placement (SliceInfo)
  bool skip;          // packed key tile past its sequence: no role does anything
};

// Register split: 512 threads launched at 128 registers (launch bounds 512,1);
// the softmax warpgroups keep their P^T values between the two phases and the
// dQ warpgroup holds a whole dQ^T row (128 fp32) before staging it, so they
// take 144 each; the MMA/TMA/LSE warpgroup keeps 80: 2 * 144 + 144 + 80 =
// 4 * 128.
constexpr int kBwdLaunchRegs = 128;
constexpr int kBwdSoftmaxRegs = 144;
constexpr int kBwdDqRegs = 144;
constexpr int kBwdOtherRegs = 80;
static_assert(2 * kBwdSoftmaxRegs + kBwdDqRegs + kBwdOtherRegs <= 4 * kBwdLaunchRegs,
              "register split");

// Unit (bh, key tile j).  The work order hands out key tiles mirrored
// (j = n-1-idx), so the long tile of a causal super-unit (small j) runs first.
// The unit visits the ni query tiles i in [i0, nq) that see key tile j (with
// SPARSE, those the block mask allows), in ascending order; every role walks
// the same list with bwd_next_i.
template <bool PACKED, bool SPARSE>
__device__ __forceinline__ BwdUnit bwd_decode(int bh, int idx, const BwdParams& p) {
  BwdUnit w;
  w.bh = bh;
  w.j = p.n_ktiles - 1 - idx;
  const SliceInfo si = slice_info<PACKED>(bh, p, kErrDeviceSeqlen);
  w.z = si.z;
  w.row0 = si.row0;
  w.rows = si.rows;
  w.L = si.L;
  const int nq = min((si.rows + kBlockM - 1) / kBlockM, p.n_ktiles);  // query tiles computed
  w.nq = nq;
  w.i0 = p.causal ? w.j : 0;
  // a key tile past L only gets zeros (fixed length) or nothing (packed)
  w.ni = (w.j * kBlockN < si.L) ? max(nq - w.i0, 0) : 0;
  if constexpr (SPARSE) {
    int n = 0;
    for (int i = w.i0; i < w.i0 + w.ni; ++i) n += tile_allowed(p.block_mask, p.n_ktiles, i, w.j);
    w.ni = n;  // a key tile no query tile sees still writes zero dK, dV
  }
  w.skip = PACKED && w.ni == 0;
  return w;
}

// The next query tile >= i of the unit's list.
template <bool SPARSE>
__device__ __forceinline__ int bwd_next_i(const BwdParams& p, const BwdUnit& w, int i) {
  if constexpr (SPARSE) {
    while (i < w.nq && !tile_allowed(p.block_mask, p.n_ktiles, i, w.j)) ++i;
  }
  return i;
}

// Longest-first order of a packed batch's backward work (the table is built
// once per call by fa_bwd_rank into the workspace).  A sequence of L rows has
// n = ceil(L / 128) key tiles; for each head its key tiles are paired with
// their mirror (tile m with tile n-1-m, equal cost under a causal mask, and
// every key tile costs the same without one), so listing the sequences by
// length, longest first, lists the super-units by cost.  Dealing them to the
// CTAs in snake order (CTA c takes positions r G + c for even r and
// r G + G-1-c for odd r) keeps CTAs busy where the head-major order over
// max_seqlen would leave those with short sequences idle.  cursor (this
// role's, starting at 0) only moves forward.
__device__ __forceinline__ bool packed_bwd_item(int k, const BwdParams& p, int& cursor,
                                                WorkItem& wi) {
  const int* len = p.rank;
  const int* seq = p.rank + p.B;
  const int* pre = p.rank + 2 * p.B;
  const int r = k >> 1;
  const long long pos = static_cast<long long>(r) * gridDim.x +
                        ((r & 1) ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                                 : static_cast<int>(blockIdx.x));
  if (pos >= pre[p.B]) return false;
  while (pre[cursor + 1] <= pos) ++cursor;
  const int b = seq[cursor];
  const int n = (len[b] + kBlockN - 1) / kBlockN;
  const int half = (n + 1) / 2;
  const int off = static_cast<int>(pos - pre[cursor]);
  const int h = off / half;
  const int m = off - h * half;
  wi.bh = b * p.H + h;
  const int a = n - 1 - m;
  // first half: key tile m (the longer one under a causal mask); second: its
  // mirror.  bwd_decode takes the unit index n_ktiles - 1 - j of key tile j.
  const int j = (k & 1) == 0 ? m : (m != a ? a : -1);
  wi.idx = j < 0 ? -1 : p.n_ktiles - 1 - j;
  return true;
}

template <int D, bool BF16, bool PACKED, bool SPARSE, bool DROPOUT>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdo,
                  const __grid_constant__ CUtensorMap tmdq, const BwdParams p) {
  using Lay = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from smem_raw by pointer arithmetic so
  // that the compiler keeps every derived pointer in the shared space
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  if (smem + Lay::kUsed > smem_raw + Lay::kSmemBytes) {
    // the dynamic shared-memory window is not aligned well enough: refuse
    if (threadIdx.x == 0) record_error(kErrDeviceLayout, 0);
    return;
  }
  uint8_t* sK = smem + Lay::kK;
  uint8_t* sV = smem + Lay::kV;
  uint8_t* sSlot = smem + Lay::kSlot;
  uint8_t* sDS = smem + Lay::kDS;
  uint8_t* sSTG = smem + Lay::kSTG;
  float* sLSE = reinterpret_cast<float*>(smem + Lay::kLSE);
  float* sDSUM = reinterpret_cast<float*>(smem + Lay::kDSUM);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* slot_full = bars + 2;   // [3]
  uint64_t* slot_empty = bars + 5;  // [3]
  uint64_t* ld_full = bars + 8;     // [2]
  uint64_t* ld_empty = bars + 10;   // [2]
  uint64_t* s_full = bars + 12;
  uint64_t* dp_full = bars + 13;
  uint64_t* p_full = bars + 14;
  uint64_t* ds_empty = bars + 15;
  uint64_t* dq_full = bars + 16;
  uint64_t* dq_empty = bars + 17;
  uint64_t* dkv_full = bars + 18;
  uint64_t* dkv_empty = bars + 19;
  uint64_t* drain = bars + 20;
  uint64_t* ds_full = bars + 21;
  uint64_t* s_read = bars + 22;   // the first softmax phase has loaded S^T out of region A
  uint64_t* dp_read = bars + 23;  // the second phase has loaded dP^T out of region A
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const WaitCtl wc{abort_flag, p.wait_ns};  // every pipeline wait of this CTA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < Lay::kSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ld_full[s], 32);
      mbar_init(&ld_empty[s], 256);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(ds_empty, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(dkv_full, 1);
    mbar_init(dkv_empty, 128);
    mbar_init(drain, 1);
    mbar_init(s_read, 256);
    mbar_init(dp_read, 256);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // this CTA's k-th work item, in the same order for every role
  int cursor = 0;
  auto next_item = [&](int k, WorkItem& wi) -> bool {
    if (PACKED && p.rank != nullptr) return packed_bwd_item(k, p, cursor, wi);
    return work_item(k, p.n_ktiles, p.B * p.H, wi);
  };

  if (warp >= 12) {
  regs_decrease<kBwdOtherRegs>();
  if (warp == 13) {
    // ------------------------------------------------------------- TMA loads
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      tma_prefetch_desc(&tmdo);
      int nunit = 0, lt = 0;  // lt: query tiles loaded (Q_lt -> slot lt & 1, dO_lt -> slot 2)
      int issued[3] = {0, 0, 0};  // loads issued into each Q/dO slot (for the drain)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        WorkItem wi;
        if (!next_item(k, wi)) break;
        if (wi.idx < 0) continue;
        const BwdUnit w = bwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
        if (w.skip) continue;
        ok = mbar_wait(kv_empty, (nunit & 1) ^ 1, wc, 20);
        if (!ok) break;
        mbar_arrive_expect_tx(kv_full, 2 * Lay::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < Lay::kPanels; ++pn) {
          tma_load_3d(sK + pn * Lay::kPanelBytes, &tmk, kv_full, pn * 64, w.row0 + w.j * kBlockN,
                      w.z);
          tma_load_3d(sV + pn * Lay::kPanelBytes, &tmv, kv_full, pn * 64, w.row0 + w.j * kBlockN,
                      w.z);
        }
        ++nunit;
        int i = w.i0 - 1;  // walks the unit's query tiles
        for (int idx = 0; idx < w.ni && ok; ++idx) {
          i = bwd_next_i<SPARSE>(p, w, i + 1);
          for (int t = 0; t < 2 && ok; ++t) {  // Q_i, then dO_i
            const int slot = t == 0 ? (lt & 1) : 2;
            const int use = t == 0 ? (lt >> 1) : lt;  // earlier loads into this slot
            ok = mbar_wait(&slot_empty[slot], (use & 1) ^ 1, wc, 21);
            if (!ok) break;
            mbar_arrive_expect_tx(&slot_full[slot], Lay::kTileBytes);
#pragma unroll
            for (int pn = 0; pn < Lay::kPanels; ++pn)
              tma_load_3d(sSlot + slot * Lay::kTileBytes + pn * Lay::kPanelBytes,
                          t == 0 ? &tmq : &tmdo, &slot_full[slot], pn * 64,
                          w.row0 + i * kBlockM, w.z);
            FA_TRACE_AT(lt, t == 0 ? 21 : 23);
            ++issued[slot];
          }
          ++lt;
        }
      }
      // Never leave with copies in flight: wait for the last load issued into
      // every barrier (the n-th use of a slot completes its phase n & 1;
      // already complete on the normal path).
      if (nunit > 0) mbar_wait_drain(kv_full, (nunit - 1) & 1, 200000000ull);
      for (int s = 0; s < 3; ++s)
        if (issued[s] > 0) mbar_wait_drain(&slot_full[s], (issued[s] - 1) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 14) {
    // ------------------------------------------------ LSE_i, D_i -> shared memory
    int seq = 0;
    bool ok = true;
    const float log2e = 1.4426950408889634f;
    for (int k = 0; ok; ++k) {
      WorkItem wi;
      if (!next_item(k, wi)) break;
      if (wi.idx < 0) continue;
      const BwdUnit w = bwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
      if (w.skip) continue;
      const size_t base = static_cast<size_t>(w.z) * p.N + w.row0;
      int i = w.i0 - 1;  // walks the unit's query tiles
      for (int idx = 0; idx < w.ni && ok; ++idx) {
        i = bwd_next_i<SPARSE>(p, w, i + 1);
        const int st = seq & 1;
        ok = mbar_wait_warp(&ld_empty[st], ((seq >> 1) & 1) ^ 1, wc, 22);
        if (!ok) break;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ql = lane * 4 + e;
          const int q = i * kBlockM + ql;
          // rows past the computed ones (past N, or past a packed sequence):
          // LSE = +inf makes P = 0 there, D = 0, so they add exactly zero to
          // dK, dV and dQ.  D is kept negated so the second softmax phase
          // forms dP - D with one add.
          const bool live = q < w.rows;
          sLSE[st * 128 + ql] = live ? p.lse[base + q] * log2e : INFINITY;
          sDSUM[st * 128 + ql] = live ? -p.dsum[base + q] : 0.f;
        }
        mbar_arrive(&ld_full[st]);
        if (lane == 0) FA_TRACE_AT(seq, 9);
        ++seq;
      }
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_f16(BF16, 128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t kIdTS = idesc_f16(BF16, 128, D, false, true);    // dV, dK (B MN-major)
      // dQ = dS K_j (M = queries, N = d): a TMEM lane holds one query row
      constexpr uint32_t kIdDQ = idesc_f16(BF16, 128, D, true, true);
      // Low descriptor words of every operand tile, K-major (_k) or MN-major
      // (_m) view; the grouped MMAs derive the K steps from them.
      const uint32_t aSlot = smem_addr(sSlot);
      const uint32_t lK_k = sdesc_lo(smem_addr(sK), false), lK_m = sdesc_lo(smem_addr(sK), true);
      const uint32_t lV_k = sdesc_lo(smem_addr(sV), false);
      const uint32_t lQ0_k = sdesc_lo(aSlot, false), lQ0_m = sdesc_lo(aSlot, true);
      const uint32_t lQ1_k = sdesc_lo(aSlot + Lay::kTileBytes, false),
                     lQ1_m = sdesc_lo(aSlot + Lay::kTileBytes, true);
      const uint32_t lO_k = sdesc_lo(aSlot + 2 * Lay::kTileBytes, false),
                     lO_m = sdesc_lo(aSlot + 2 * Lay::kTileBytes, true);
      const uint32_t lS_k = sdesc_lo(smem_addr(sDS), false), lS_m = sdesc_lo(smem_addr(sDS), true);
      int nunit = 0, it = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        WorkItem wi;
        if (!next_item(k, wi)) break;
        if (wi.idx < 0) continue;
        const BwdUnit w = bwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
        if (w.skip) continue;
        ok = mbar_wait(kv_full, nunit & 1, wc, 23);
        if (!ok) break;
        tc_fence_after();
        // The epilogue of the previous unit must have read dV/dK before this
        // unit writes them, and before dkv_full is committed again (so that
        // barrier never runs two phases ahead of its waiter, also for units
        // with no query tiles).
        bool dkv_free = nunit == 0;
        // Software pipeline over the query tiles of the unit.  TMEM region A
        // holds S^T(i), then dP^T(i); region B holds P^T(i), then dQ(i):
        //   dP(i) once the first softmax phase has loaded S^T(i) out of A,
        //   dV(i) once it has written P^T(i) into B,
        //   S(i+1) once the second phase has loaded dP^T(i) out of A,
        //   dK(i), then dQ(i) into B (dV(i), issued before it, has read
        //   P^T(i)) once dS^T(i) is in shared memory.
        // No MMA waits for the exponentials of the tile it overwrites, nor for
        // the read-out of dQ (the first phase of the next tile waits for that
        // before it writes P^T into B).
        auto issue_s = [&](int t) -> bool {  // S^T(t) = K_j Q_t^T, Q_t in slot t & 1
          if (t > 0 && !mbar_wait(dp_read, (t - 1) & 1, wc, 37)) return false;
          if (!mbar_wait(&slot_full[t & 1], (t >> 1) & 1, wc, 24)) return false;
          FA_TRACE_AT(t, 28);
          tc_fence_after();
          umma_ss_group<D / 16, false, false>(tmem + Lay::kColA, lK_k, (t & 1) ? lQ1_k : lQ0_k,
                                              kIdS, 0u);
          umma_commit(s_full);
          return true;
        };
        if (w.ni > 0) ok = issue_s(it);
        for (int idx = 0; idx < w.ni && ok; ++idx) {
          FA_TRACE_AT(it, 0);
          // dP^T = V_j dO_i^T into region A
          ok = mbar_wait(s_read, it & 1, wc, 25);
          if (ok) ok = mbar_wait(&slot_full[2], it & 1, wc, 35);
          if (!ok) break;
          tc_fence_after();
          FA_TRACE_AT(it, 1);
          umma_ss_group<D / 16, false, false>(tmem + Lay::kColA, lV_k, lO_k, kIdS, 0u);
          umma_commit(dp_full);
          // dV_j += P^T dO_i once the first softmax phase wrote P^T
          ok = mbar_wait(p_full, it & 1, wc, 26);
          if (!ok) break;
          tc_fence_after();
          FA_TRACE_AT(it, 2);
          if (!dkv_free) {
            ok = mbar_wait(dkv_empty, (nunit - 1) & 1, wc, 27);
            if (!ok) break;
            tc_fence_after();
            dkv_free = true;
          }
          // (A = P^T in TMEM region B, 16 queries = 8 columns; queries 64..127
          // sit 64 columns further)
          umma_ts_group8<true, true>(tmem + Lay::kColDV, tmem + Lay::kColB, lO_m, kIdTS,
                                     idx > 0 ? 1u : 0u);
          umma_commit(&slot_empty[2]);  // dO_i: dP and dV done
          FA_TRACE_AT(it, 13);
          if (idx + 1 < w.ni) {
            ok = issue_s(it + 1);
            if (!ok) break;
          }
          FA_TRACE_AT(it, 14);
          // dQ and dK_j += dS^T Q_i once the second phase wrote dS^T
          ok = mbar_wait(ds_full, it & 1, wc, 36);
          if (!ok) break;
          tc_fence_after();
          FA_TRACE_AT(it, 8);
          // dK_j += dS^T Q_i: A = dS^T K-major, B = Q_i MN-major.  Issued
          // before dQ so that Q_i's slot, the one the next-but-one query tile
          // loads into, is released one contraction earlier.
          umma_ss_group<8, false, true>(tmem + Lay::kColDK, lS_k, (it & 1) ? lQ1_m : lQ0_m, kIdTS,
                                        idx > 0 ? 1u : 0u);
          umma_commit(&slot_empty[it & 1]);  // Q_i: S and dK done
          // dQ = dS K_j into region B: A = dS^T read MN-major (queries
          // contiguous), B = K_j read MN-major (d contiguous)
          umma_ss_group<8, true, true>(tmem + Lay::kColB, lS_m, lK_m, kIdDQ, 0u);
          umma_commit(dq_full);
          umma_commit(ds_empty);             // dK and dQ have read dS^T
          FA_TRACE_AT(it, 3);
          ++it;
        }
        if (!ok) break;
        if (!dkv_free) {
          ok = mbar_wait(dkv_empty, (nunit - 1) & 1, wc, 34);
          if (!ok) break;
        }
        umma_commit(dkv_full);
        umma_commit(kv_empty);
        ++nunit;
      }
      umma_commit(drain);
      mbar_wait_drain(drain, 0, 200000000ull);
    }
    __syncwarp();
  }
#ifdef FA_TRACE
  if (warp == 15 && lane == 0 && blockIdx.x == 0) {
    // Trace builds only: observe when each tensor-core phase of CTA 0
    // completes (waits only, never arrives; gives up quietly).
    auto seen = [&](uint64_t* bar, uint32_t parity) {
      const uint32_t a = smem_addr(bar);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(a, parity))
        if (globaltimer_ns() - t0 > 20000000ull) return false;
      return true;
    };
    int it = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      WorkItem wi;
      if (!next_item(k, wi)) break;
      if (wi.idx < 0) continue;
      const BwdUnit w = bwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
      if (w.skip) continue;
      if (w.ni > 0) {
        ok = seen(s_full, it & 1);
        FA_TRACE_AT(it, 16);
      }
      for (int idx = 0; idx < w.ni && ok; ++idx) {
        ok = ok && seen(dp_full, it & 1);
        FA_TRACE_AT(it, 17);
        ok = ok && seen(&slot_empty[2], it & 1);
        FA_TRACE_AT(it, 18);
        if (idx + 1 < w.ni) {
          ok = ok && seen(s_full, (it + 1) & 1);
          FA_TRACE_AT(it + 1, 16);
        }
        ok = ok && seen(&slot_empty[it & 1], (it >> 1) & 1);
        FA_TRACE_AT(it, 19);
        ok = ok && seen(dq_full, it & 1);
        FA_TRACE_AT(it, 20);
        ++it;
      }
    }
  }
#endif
  } else if (warp < 8) {
    regs_increase<kBwdSoftmaxRegs>();
    // ------------------------- P^T and dS^T: key row per thread, half the queries
    const int half = warp >> 2;              // queries [64 half, 64 half + 64)
    const int r = ((warp & 3) << 5) | lane;  // key row in the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tA = tmem + lane_off + Lay::kColA;  // S^T, then dP^T
    const uint32_t tB = tmem + lane_off + Lay::kColB;  // P^T (16-bit), then dQ
    // dS^T row r, queries of this half: panel `half` of the swizzled tile
    const uint32_t ds_row = smem_addr(sDS) + half * 16384 + r * 128;
    const float cl = p.scale_log2;
    const uint32_t u_drop = 256u - min(p.keep_t, 256u);  // dropout keep test (keep_flags4)
    const uint32_t u_lo7 = (u_drop & 0x7Fu) * 0x01010101u, u_all = u_drop * 0x01010101u;
    const unsigned long long inv_keep2 = f2pack(p.inv_keep, p.inv_keep);
    int it = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      WorkItem wi;
      if (!next_item(k, wi)) break;
      if (wi.idx < 0) continue;
      const BwdUnit w = bwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
      if (w.skip) continue;
      const bool key_ok = w.j * kBlockN + r < w.L;
      int i = w.i0 - 1;  // walks the unit's query tiles
      for (int idx = 0; idx < w.ni && ok; ++idx) {
        i = bwd_next_i<SPARSE>(p, w, i + 1);
        const int st = it & 1;  // LSE/D staging advances with the iteration count
        // dropout: keep flags of this key for the half's 64 queries
        // (keep_flags_key64), made while S^T is computed; the first phase
        // writes only kept P^T, the second scales the kept dP^T by 256 / t
        uint32_t drop_keep[2] = {~0u, ~0u};
        if constexpr (DROPOUT)
          keep_flags_key64(p, w.bh, w.j * kBlockN + r, i * kBlockM + 64 * half, lane & 3, u_lo7,
                           u_all, drop_keep);
        // ---- phase 1: P^T = 2^(c S^T - LSE_i log2 e) from S^T (region A),
        // to region B as 16-bit for the dV product
        ok = mbar_wait_warp(&ld_full[st], (it >> 1) & 1, wc, 28) &&
             mbar_wait_warp(s_full, it & 1, wc, 29);
        if (!ok) break;
        tc_fence_after();
        if (threadIdx.x == FA_TRACE_SM_THREAD) FA_TRACE_AT(it, 4);
        // a query tile on the causal diagonal hides keys above the query
        const int diag_lim = (p.causal && i == w.j) ? r : -1;  // visible iff q_local >= r
        const float* lse2 = sLSE + st * 128;
        const float* dsm = sDSUM + st * 128;
        uint32_t pp[32];               // P^T as dV sees it (dropped scores zero), 16-bit pairs
        uint32_t pu[DROPOUT ? 32 : 1];  // dropout: P^T before the mask, for the second phase
        {
          uint32_t sr[64];  // S^T of this key row, the half's 64 queries
          tmem_ld64(tA + 64 * half, sr);
          // region A may now take dP^T(i)
          tc_fence_before();
          mbar_arrive(s_read);
          if (threadIdx.x == FA_TRACE_SM_THREAD) FA_TRACE_AT(it, 10);
          // the exponentials, P^T to 16-bit pairs; MASKED: the per-score
          // visibility test (causal diagonal tile, keys past the valid length)
          auto exps = [&](auto masked_tag) {
            constexpr bool MASKED = decltype(masked_tag)::value;
#pragma unroll
            for (int e = 0; e < 64; e += 4) {
              const int q0 = 64 * half + e;  // query inside the tile
              const float4 l4 = *reinterpret_cast<const float4*>(lse2 + q0);
              const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
              float pv[4];
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) {
                const float x = fmaf(__uint_as_float(sr[e + k4]), cl, -lv[k4]);
                if constexpr (MASKED) {
                  const bool vis = key_ok && (q0 + k4 >= diag_lim);
                  pv[k4] = vis ? ex2_approx(x) : 0.f;
                } else {
                  pv[k4] = ex2_approx(x);
                }
              }
              pp[e >> 1] = pack2<BF16>(pv[0], pv[1]);
              pp[(e >> 1) + 1] = pack2<BF16>(pv[2], pv[3]);
              if constexpr (DROPOUT) {
                // P^T as dV sees it: dropped scores are zero.  Queries e .. e + 3
                // = 32 h + 16 e' + 4 s + c share one shift of the flags
                pu[e >> 1] = pp[e >> 1];
                pu[(e >> 1) + 1] = pp[(e >> 1) + 1];
                const uint32_t fl = drop_keep[e >> 5] << (((e >> 2) & 3) + 4 * ((e >> 4) & 1));
                pp[e >> 1] &= pair_keep_mask(fl, 0);
                pp[(e >> 1) + 1] &= pair_keep_mask(fl, 1);
              }
            }
          };
          if constexpr (DROPOUT) {
            // with dropout a copy without the test serves the tiles off the
            // causal diagonal (measured ~10 % faster there; the dense kernels
            // measured no gain, fp16 a loss, so they keep the one loop)
            if (key_ok && diag_lim < 0) exps(std::false_type{});
            else exps(std::true_type{});
          } else {
            exps(std::true_type{});
          }
        }
        // region B still holds dQ(i-1) until the dQ warps have read it
        if (it > 0) {
          ok = mbar_wait_warp(dq_empty, (it - 1) & 1, wc, 38);
          if (!ok) break;
        }
        tc_fence_after();
        // P^T of the half's queries [64 half, 64 half + 64): columns 64 half ..
        // 64 half + 31 of region B (16 queries per 8 columns); with dropout the
        // unmasked copy goes to the next 32 columns
        tmem_st_n<32>(tB + 64 * half, pp);
        if constexpr (DROPOUT) tmem_st_n<32>(tB + 64 * half + 32, pu);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
        if (threadIdx.x == FA_TRACE_SM_THREAD) FA_TRACE_AT(it, 15);
        // ---- phase 2: dS^T = P^T * (dP^T - D_i) from dP^T (region A) and the
        // 16-bit P^T (region B), to shared memory
        ok = mbar_wait_warp(dp_full, it & 1, wc, 30);
        if (ok && it > 0) ok = mbar_wait_warp(ds_empty, (it - 1) & 1, wc, 31);
        if (!ok) break;
        tc_fence_after();
        if (threadIdx.x == FA_TRACE_SM_THREAD) FA_TRACE_AT(it, 11);
        uint32_t dr[64];  // dP^T of this key row, the half's 64 queries
        tmem_ld64(tA + 64 * half, dr);
        uint32_t pq[32];  // P^T, 16-bit pairs (unmasked with dropout)
        tmem_ld32(tB + 64 * half + (DROPOUT ? 32 : 0), pq);
        // region A may now take S^T(i+1)
        tc_fence_before();
        mbar_arrive(dp_read);
        if (threadIdx.x == FA_TRACE_SM_THREAD) FA_TRACE_AT(it, 12);
        uint32_t dd[16];
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const int q0 = 64 * half + e;
          const float4 nd = *reinterpret_cast<const float4*>(dsm + q0);  // -D
          if constexpr (DROPOUT) {  // dP of the kept scores (scaled by 256 / t below)
            const uint32_t fl = drop_keep[e >> 5] << (((e >> 2) & 3) + 4 * ((e >> 4) & 1));
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) dr[e + k4] &= word_keep_mask(fl, k4);
          }
          float pf[4];
          unpack2<BF16>(pq[e >> 1], pf[0], pf[1]);
          unpack2<BF16>(pq[(e >> 1) + 1], pf[2], pf[3]);
          // packed pairs: (dP - D) then P (dP - D)
          // (with dropout, dP of the kept scores times 256 / t, minus D)
          const auto dr01 = f2pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1]));
          const auto dr23 = f2pack(__uint_as_float(dr[e + 2]), __uint_as_float(dr[e + 3]));
          const auto x01 = DROPOUT ? ffma2(dr01, inv_keep2, f2pack(nd.x, nd.y))
                                   : fadd2(dr01, f2pack(nd.x, nd.y));
          const auto x23 = DROPOUT ? ffma2(dr23, inv_keep2, f2pack(nd.z, nd.w))
                                   : fadd2(dr23, f2pack(nd.z, nd.w));
          float gv[4];
          f2unpack(fmul2(f2pack(pf[0], pf[1]), x01), gv[0], gv[1]);
          f2unpack(fmul2(f2pack(pf[2], pf[3]), x23), gv[2], gv[3]);
          dd[(e & 31) >> 1] = pack2<BF16>(gv[0], gv[1]);
          dd[((e & 31) >> 1) + 1] = pack2<BF16>(gv[2], gv[3]);
          if (threadIdx.x == FA_TRACE_SM_THREAD && (e & 15) == 12) FA_TRACE_AT(it, 24 + (e >> 4));
          if ((e & 31) == 28) {
            // 32 queries done: four 16-byte units of the 128-byte swizzled row
            // (units 4 cc .. 4 cc + 3 of panel `half`, cc = e / 32)
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
              const uint32_t unit = ((e >> 5) * 4 + w4) ^ (r & 7);
              st_shared_v4(ds_row + unit * 16, dd[4 * w4], dd[4 * w4 + 1], dd[4 * w4 + 2],
                           dd[4 * w4 + 3]);
            }
          }
        }
        if (threadIdx.x == FA_TRACE_SM_THREAD) FA_TRACE_AT(it, 22);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(ds_full);
        mbar_arrive(&ld_empty[st]);
        if (threadIdx.x == FA_TRACE_SM_THREAD) FA_TRACE_AT(it, 5);
        ++it;
      }
    }
  } else {
    regs_increase<kBwdDqRegs>();
    // --------------------------- dQ read-out and reduce-add; dK_j, dV_j epilogue
    const int r = ((warp & 3) << 5) | lane;  // TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int it = 0, nunit = 0, stage_round = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      WorkItem wi;
      if (!next_item(k, wi)) break;
      if (wi.idx < 0) continue;
      const BwdUnit w = bwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
      if (w.skip) continue;
      const size_t base = static_cast<size_t>(w.z) * p.N + w.row0;
      int i = w.i0 - 1;  // walks the unit's query tiles
      for (int idx = 0; idx < w.ni && ok; ++idx) {
        i = bwd_next_i<SPARSE>(p, w, i + 1);
        // the four warps share named barrier 1 below: they go on or stop together
        ok = named_bar_and(1, 128, mbar_wait_warp(dq_full, it & 1, wc, 32));
        if (!ok) break;
        tc_fence_after();
        if (threadIdx.x == 256) FA_TRACE_AT(it, 6);
        // Lane r holds row r of dQ_i (one query, d contiguous).  Read it all,
        // release the TMEM columns, then D / 32 rounds: each stages a
        // [128][32] fp32 column block of the tile in one of two 16 KB buffers
        // (128-byte rows whose 16-byte units are permuted by the row as the
        // 128-byte TMA swizzle expects, so the vector stores of a warp hit
        // distinct banks) and reduce-adds it into the accumulator with one TMA
        // transfer (the TMA path sustains more reduce bandwidth per SM than
        // per-thread reds); staging a round overlaps the previous transfer.
        // Rows past N are clipped by the transfer.
        {
          const bool leader = warp == 8 && lane == 0;
          uint32_t v[D];
          if constexpr (D == 128) tmem_ld64x2(tmem + lane_off + Lay::kColB, v);
          else tmem_ld64(tmem + lane_off + Lay::kColB, v);
          if (threadIdx.x == 256) FA_TRACE_AT(it, 29);
          tc_fence_before();
          mbar_arrive(dq_empty);
#pragma unroll
          for (int rd = 0; rd < D / 32; ++rd) {
            uint8_t* stg = sSTG + (stage_round & 1) * 16384;
            if (stage_round >= 2) {
              // the transfer that used this buffer two rounds ago must have
              // read it
              if (leader) bulk_wait_read_one();
              named_bar_sync(1, 128);
            }
            const uint32_t row = smem_addr(stg) + r * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              st_shared_v4(row + ((u ^ (r & 7)) << 4), v[rd * 32 + 4 * u], v[rd * 32 + 4 * u + 1],
                           v[rd * 32 + 4 * u + 2], v[rd * 32 + 4 * u + 3]);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (leader) {
              tma_reduce_add_3d(&tmdq, stg, rd * 32, w.row0 + i * kBlockM, w.z);
              bulk_commit_group();
            }
            ++stage_round;
          }
        }
        if (threadIdx.x == 256) FA_TRACE_AT(it, 7);
        ++it;
      }
      if (!ok) break;
      ok = named_bar_and(1, 128, mbar_wait_warp(dkv_full, nunit & 1, wc, 33));
      if (!ok) break;
      tc_fence_after();
      const int key = w.j * kBlockN + r;
      const bool keep = key < w.L;  // padded keys get exactly zero
      const bool store = key < w.rows;
      const size_t off = (base + (store ? key : 0)) * (D * 2);
      uint8_t* dvrow = reinterpret_cast<uint8_t*>(p.dv) + off;
      uint8_t* dkrow = reinterpret_cast<uint8_t*>(p.dk) + off;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t col = part == 0 ? Lay::kColDV : Lay::kColDK;
        const float mul = part == 0 ? (DROPOUT ? p.inv_keep : 1.f) : p.scale;
        uint8_t* rowp = part == 0 ? dvrow : dkrow;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          if (w.ni > 0) {
            tmem_ld32(tmem + lane_off + col + c * 32, v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = keep ? __uint_as_float(v[2 * e]) * mul : 0.f;
            const float b = keep ? __uint_as_float(v[2 * e + 1]) * mul : 0.f;
            pk[e] = pack2<BF16>(a, b);
          }
          if (store) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              st_global_v4(rowp + c * 64 + v4 * 16, pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2],
                           pk[4 * v4 + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(dkv_empty);
      ++nunit;
    }
    // every reduce-add issued must have completed before the kernel ends
    if (warp == 8 && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

// D_i = <dO_i, O_i> in fp32 from the stored 16-bit values; zero the fp32 dQ
// accumulator.  D/8 threads per row, 16-byte loads.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre(const uint4* __restrict__ o,
                                                  const uint4* __restrict__ dout,
                                                  float* __restrict__ dsum,
                                                  float4* __restrict__ dq_acc, long long rows) {
  constexpr int T = D / 8;
  const long long total = rows * T;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  // whole warps iterate together so the row-group shuffles see every lane
  for (long long wbase = blockIdx.x * static_cast<long long>(blockDim.x) + (threadIdx.x & ~31);
       wbase < total; wbase += stride) {
    const long long g = wbase + (threadIdx.x & 31);
    const bool live = g < total;
    float s = 0.f;
    if (live) {
      const uint4 a = o[g];
      const uint4 b = dout[g];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 fa, fb;
        if constexpr (BF16) {
          fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
          fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
        } else {
          fa = __half22float2(*reinterpret_cast<const __half2*>(&av[e]));
          fb = __half22float2(*reinterpret_cast<const __half2*>(&bv[e]));
        }
        s = fmaf(fa.x, fb.x, s);
        s = fmaf(fa.y, fb.y, s);
      }
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      dq_acc[2 * g] = z;
      dq_acc[2 * g + 1] = z;
    }
#pragma unroll
    for (int m = T / 2; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m, T);
    if (live && (g & (T - 1)) == 0) dsum[g / T] = s;
  }
}

// dQ = scale * accumulator -> 16-bit; 8 values per thread.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_post(const float4* __restrict__ acc,
                                                   uint4* __restrict__ dq, float scale,
                                                   long long n8) {
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < n8;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = acc[2 * g];
    const float4 b = acc[2 * g + 1];
    uint4 r;
    r.x = pack2<BF16>(a.x * scale, a.y * scale);
    r.y = pack2<BF16>(a.z * scale, a.w * scale);
    r.z = pack2<BF16>(b.x * scale, b.y * scale);
    r.w = pack2<BF16>(b.z * scale, b.w * scale);
    dq[g] = r;
  }
}

// The longest-first table of a packed batch (see packed_bwd_item): lengths
// as slice_info clamps them, sequences ranked by length (ties by index), and
// the running count of super-units over the ranking.  One block.
__global__ void __launch_bounds__(1024) fa_bwd_rank(const BwdParams p) {
  int* len = p.rank;
  int* seq = p.rank + p.B;
  int* pre = p.rank + 2 * p.B;
  for (int b = threadIdx.x; b < p.B; b += blockDim.x)
    len[b] = slice_info<true>(b * p.H, p, kErrDeviceSeqlen).L;
  __syncthreads();
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    const int lb = len[b];
    int rank = 0;
    for (int o = 0; o < p.B; ++o) rank += (len[o] > lb) || (len[o] == lb && o < b);
    seq[rank] = b;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int i = 0; i < p.B; ++i) {
      pre[i] = acc;
      acc += p.H * (((len[seq[i]] + kBlockN - 1) / kBlockN + 1) / 2);
    }
    pre[p.B] = acc;
  }
}

cudaError_t launch_bwd_rank(const BwdParams& p, cudaStream_t stream) {
  fa_bwd_rank<<<1, 1024, 0, stream>>>(p);
  return cudaGetLastError();
}

static int elementwise_grid(long long n8, int num_sms) {
  return static_cast<int>(std::max<long long>(1, std::min<long long>((n8 + 255) / 256, num_sms * 16ll)));
}

cudaError_t launch_bwd_pre(int d, bool bf16, const BwdParams& p, int num_sms,
                           cudaStream_t stream) {
  const long long rows = total_rows(p);
  const int grid = elementwise_grid(rows * d / 8, num_sms);
  const uint4* o = static_cast<const uint4*>(p.o);
  const uint4* dout = static_cast<const uint4*>(p.dout);
  float4* acc = reinterpret_cast<float4*>(p.dq_acc);
  if (d == 128) {
    if (bf16) fa_bwd_pre<128, true><<<grid, 256, 0, stream>>>(o, dout, p.dsum, acc, rows);
    else fa_bwd_pre<128, false><<<grid, 256, 0, stream>>>(o, dout, p.dsum, acc, rows);
  } else {
    if (bf16) fa_bwd_pre<64, true><<<grid, 256, 0, stream>>>(o, dout, p.dsum, acc, rows);
    else fa_bwd_pre<64, false><<<grid, 256, 0, stream>>>(o, dout, p.dsum, acc, rows);
  }
  return cudaGetLastError();
}

template <int D, bool BF16, bool PACKED, bool SPARSE, bool DROPOUT>
static cudaError_t launch_bwd_main_t(const CUtensorMap& tmq, const CUtensorMap& tmk,
                                     const CUtensorMap& tmv, const CUtensorMap& tmdo,
                                     const CUtensorMap& tmdq, const BwdParams& p, int num_sms,
                                     cudaStream_t stream) {
  using Lay = BwdLayout<D>;
  auto kern = fa_bwd_kernel<D, BF16, PACKED, SPARSE, DROPOUT>;
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  // the register split in the kernel assumes exactly this launch allocation
  if (attr.numRegs != kBwdLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.n_units < num_sms ? p.n_units : num_sms;
  kern<<<grid, 512, Lay::kSmemBytes, stream>>>(tmq, tmk, tmv, tmdo, tmdq, p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_main(int d, bool bf16, const CUtensorMap& tmq, const CUtensorMap& tmk,
                            const CUtensorMap& tmv, const CUtensorMap& tmdo,
                            const CUtensorMap& tmdq, const BwdParams& p, int num_sms,
                            cudaStream_t stream) {
  const int mode = p.cu_seqlens != nullptr ? 1
                   : p.block_mask != nullptr ? 2
                   : p.keep_t < 256u        ? 3
                                            : 0;
#define FA_BWD_LAUNCH(DD, BB, PP, SS, RR) \
  launch_bwd_main_t<DD, BB, PP, SS, RR>(tmq, tmk, tmv, tmdo, tmdq, p, num_sms, stream)
#define FA_BWD_MODES(DD, BB)                                                \
  (mode == 1   ? FA_BWD_LAUNCH(DD, BB, true, false, false)                  \
   : mode == 2 ? FA_BWD_LAUNCH(DD, BB, false, true, false)                  \
   : mode == 3 ? FA_BWD_LAUNCH(DD, BB, false, false, true)                  \
               : FA_BWD_LAUNCH(DD, BB, false, false, false))
  if (d == 128) return bf16 ? FA_BWD_MODES(128, true) : FA_BWD_MODES(128, false);
  return bf16 ? FA_BWD_MODES(64, true) : FA_BWD_MODES(64, false);
#undef FA_BWD_MODES
#undef FA_BWD_LAUNCH
}

cudaError_t launch_bwd_post(int d, bool bf16, const BwdParams& p, int num_sms,
                            cudaStream_t stream) {
  const long long n8 = total_rows(p) * d / 8;
  const int grid = elementwise_grid(n8, num_sms);
  const float4* acc = reinterpret_cast<const float4*>(p.dq_acc);
  uint4* dq = static_cast<uint4*>(p.dq);
  if (bf16) fa_bwd_post<true><<<grid, 256, 0, stream>>>(acc, dq, p.scale, n8);
  else fa_bwd_post<false><<<grid, 256, 0, stream>>>(acc, dq, p.scale, n8);
  return cudaGetLastError();
}

}  // namespace fa
