// Forward exact attention on sm_100a: tiled, online softmax, nothing N x N
// ever leaves the SM.
//
// What is computed follows "How Flash Attention Works" (swarnava.dev):
//  * section "Tiling Q, K, and V for Fast On-Chip Memory": a block of query
//    rows stays on chip while K and V blocks stream past it; causal and
//    padding masks are applied per tile, boundary tiles take the ragged edge;
//  * section "Online Softmax Without the Full Score Matrix": each K/V tile
//    updates a running row max and row sum, and the partial output is
//    rescaled when the max grows;
//  * section "Kernel Fusion and Incremental Output Accumulation": scores,
//    masking, softmax statistics and the V-weighted accumulation all happen
//    in one kernel, and only O and per-row statistics (here the log-sum-exp)
//    reach HBM.
//
// B200 mapping (one persistent CTA per SM, 384 threads):
//  * a work unit is (batch*head, pair of 128-row query tiles); the two tiles
//    share every K/V tile that is loaded, and their softmax work ping-pongs
//    so the tensor core always has the other tile's MMA to run;
//  * warp 9 (one thread) issues TMA loads: Q tiles once per unit, K and V
//    tiles through a ring of shared-memory slots guarded by mbarriers;
//  * warp 8 (one thread) issues tcgen05 MMAs: S = Q K^T into TMEM, then
//    O += P V with P read straight from TMEM;
//  * warps 0-3 and 4-7 are the softmax warpgroups of query tile 0 and 1: a
//    thread owns one query row (TMEM lane), so row max and row sum need no
//    shuffles; they write P (16-bit) over S in TMEM, rescale O in TMEM when
//    the running max moves by more than the lazy threshold, and finally
//    normalise O and store O and LSE with 16-byte vector stores.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 and O1 at 256 + t*d.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

// Packed batches of at most this many sequences are scheduled longest
// first (more fall back to the head-major order of work_item).
constexpr int kRankMaxSeqs = 512;

// Longest-first order of a packed batch's work.  The super-units of a
// sequence (for each head, query-tile pair m with its mirror, as in
// work_item) all cost about the same, so listing the sequences by length,
// longest first, lists the super-units by cost; dealing them to the CTAs in
// snake order (CTA c takes positions r G + c for even r and r G + G-1-c for
// odd r) balances the CTAs where head-major order leaves those with short
// sequences idle.  The table is built in shared memory by the whole CTA
// before the roles split, and every role walks it with its own cursor.
struct PackedOrder {
  const int* len;   // [B] sequence lengths (as slice_info clamps them)
  const int* seq;   // [B] sequence of each rank
  const int* pre;   // [B + 1] super-units before each rank
};

__device__ __forceinline__ int fwd_pairs(int L) { return ((L + kBlockM - 1) / kBlockM + 1) / 2; }

__device__ void packed_order_build(const FwdParams& p, int* len, int* seq, int* pre) {
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
      acc += p.H * ((fwd_pairs(len[seq[i]]) + 1) / 2);
    }
    pre[p.B] = acc;
  }
}

// Work item k of this CTA in the longest-first order; false past the end.
// cursor (this role's, starting at 0) only moves forward.
__device__ __forceinline__ bool packed_work_item(int k, const FwdParams& p, const PackedOrder& o,
                                                 int& cursor, WorkItem& wi) {
  const int r = k >> 1;
  const long long pos = static_cast<long long>(r) * gridDim.x +
                        ((r & 1) ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                                 : static_cast<int>(blockIdx.x));
  if (pos >= o.pre[p.B]) return false;
  while (o.pre[cursor + 1] <= pos) ++cursor;
  const int b = o.seq[cursor];
  const int pairs = fwd_pairs(o.len[b]);
  const int half = (pairs + 1) / 2;
  const int off = static_cast<int>(pos - o.pre[cursor]);
  const int h = off / half;
  const int m = off - h * half;
  wi.bh = b * p.H + h;
  const int a = pairs - 1 - m;
  wi.idx = (k & 1) == 0 ? a : (m != a ? m : -1);
  return true;
}

template <int D, int ESZ>
struct FwdLayout {
  static constexpr int kRowBytes = D * ESZ;            // ESZ = element bytes (2, or 1 for e4m3)
  static constexpr int kTileBytes = kBlockM * kRowBytes;  // one 128-row, d-wide tile
  static constexpr int kPanelBytes = 128 * 128;        // 128 rows x 128 bytes: one swizzle panel
  static constexpr int kPanels = kRowBytes / 128;
  static constexpr int kPanelElems = 128 / ESZ;        // row elements inside one panel
  static constexpr int kSlots = (kTileBytes == 32768) ? 4 : 8;  // K/V ring depth
  static constexpr int kQ0 = 0;
  static constexpr int kSlot0 = 2 * kTileBytes;
  static constexpr int kBar = kSlot0 + kSlots * kTileBytes;
  static constexpr int kBarBytes = 512;
  // packed batches: sequence lengths, sequences ranked by length and the
  // running count of super-units over the ranking (see PackedOrder)
  static constexpr int kRank = kBar + kBarBytes;
  static constexpr int kRankBytes = (3 * kRankMaxSeqs + 1) * 4;
  static constexpr int kSmemBytes = kRank + kRankBytes + 1024;  // + slack to align to 1024
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
};

// Register split: 384 threads launched at 168 registers (launch bounds 384,1);
// the two softmax warpgroups take 184, the MMA/TMA warpgroup keeps 136:
// 2 * 184 + 136 = 3 * 168 (no spills at this split).
constexpr int kFwdLaunchRegs = 168;
constexpr int kFwdSoftmaxRegs = 184;
constexpr int kFwdOtherRegs = 136;
static_assert(2 * kFwdSoftmaxRegs + kFwdOtherRegs <= 3 * kFwdLaunchRegs, "register split");

struct FwdUnit {
  int bh, qt0, L, jend0, jend1;
  int z, row0, rows;    // slice placement (SliceInfo)
  int jlast0, jlast1;   // last key tile each query tile computes, -1 for none
};

// Unit (bh, pair): query tiles 2 pair and 2 pair + 1 of slice bh.  A query
// tile that starts at or past the slice's computed rows has no work.  Query
// tile t computes the key tiles j < jend_t (causal / key-length limit) that
// the block mask allows (SPARSE); the unit streams the union of the two
// lists in ascending order.
template <bool SPARSE>
__device__ __forceinline__ bool fwd_need(const FwdParams& p, const FwdUnit& w, int t, int j) {
  if (j >= (t == 0 ? w.jend0 : w.jend1)) return false;
  if constexpr (SPARSE) return tile_allowed(p.block_mask, p.n_qtiles, w.qt0 + t, j);
  return true;
}

// Smallest key tile >= j that either query tile computes; max(jend) if none.
template <bool SPARSE>
__device__ __forceinline__ int fwd_next(const FwdParams& p, const FwdUnit& w, int j) {
  const int jmax = max(w.jend0, w.jend1);
  if constexpr (SPARSE) {
    while (j < jmax && !fwd_need<SPARSE>(p, w, 0, j) && !fwd_need<SPARSE>(p, w, 1, j)) ++j;
  }
  return j < jmax ? j : jmax;
}

template <bool PACKED, bool SPARSE>
__device__ __forceinline__ FwdUnit fwd_decode(int bh, int pair, const FwdParams& p) {
  FwdUnit w;
  w.bh = bh;
  const SliceInfo si = slice_info<PACKED>(bh, p, kErrDeviceSeqlen);
  w.z = si.z;
  w.row0 = si.row0;
  w.rows = si.rows;
  w.L = si.L;
  const int nkb = (si.L + kBlockN - 1) / kBlockN;
  const int nq = (si.rows + kBlockM - 1) / kBlockM;
  w.qt0 = 2 * pair;
  int je[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = w.qt0 + t;
    if (qt < nq && qt < p.n_qtiles) je[t] = p.causal ? min(nkb, qt + 1) : nkb;
    else je[t] = 0;
  }
  w.jend0 = je[0];
  w.jend1 = je[1];
  int jl[2] = {je[0] - 1, je[1] - 1};
  if constexpr (SPARSE) {
#pragma unroll
    for (int t = 0; t < 2; ++t)
      while (jl[t] >= 0 && !tile_allowed(p.block_mask, p.n_qtiles, w.qt0 + t, jl[t])) --jl[t];
  }
  w.jlast0 = jl[0];
  w.jlast1 = jl[1];
  return w;
}

template <int D, bool BF16, bool PACKED, bool SPARSE, bool DROPOUT, bool FP8>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const FwdParams p) {
  using Lay = FwdLayout<D, FP8 ? 1 : 2>;
  static_assert(!FP8 || (D == 128 && !PACKED && !SPARSE && !DROPOUT), "e4m3: dense, d = 128");
  constexpr int kSlots = Lay::kSlots;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from smem_raw by pointer arithmetic so
  // that the compiler keeps every derived pointer in the shared space
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sq = smem + Lay::kQ0;        // Q0, Q1 tiles
  uint8_t* skv = smem + Lay::kSlot0;    // K/V ring
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* q_full = bars;              // [2]
  uint64_t* q_empty = bars + 2;         // [2]
  uint64_t* kv_full = bars + 4;         // [kSlots]
  uint64_t* kv_empty = kv_full + kSlots;
  uint64_t* s_full = kv_empty + kSlots; // [2]
  uint64_t* p_full = s_full + 2;        // [2]
  uint64_t* o_full = p_full + 2;        // [2]
  uint64_t* drain = o_full + 2;         // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const WaitCtl wc{abort_flag, p.wait_ns};  // every pipeline wait of this CTA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&q_empty[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
    tmem_relinquish();
  }
  PackedOrder order{nullptr, nullptr, nullptr};
  const bool ranked = PACKED && p.B <= kRankMaxSeqs;
  if (ranked) {
    int* tab = reinterpret_cast<int*>(smem + Lay::kRank);
    order = PackedOrder{tab, tab + kRankMaxSeqs, tab + 2 * kRankMaxSeqs};
    packed_order_build(p, tab, tab + kRankMaxSeqs, tab + 2 * kRankMaxSeqs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // this CTA's k-th work item, in the same order for every role
  int cursor = 0;
  auto next_item = [&](int k, WorkItem& wi) -> bool {
    if (ranked) return packed_work_item(k, p, order, cursor, wi);
    return work_item(k, p.n_pairs, p.B * p.H, wi);
  };
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
  regs_decrease<kFwdOtherRegs>();
  if (warp == 9) {
    // ------------------------------------------------------------- TMA loads
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      int qload[2] = {0, 0};
      int kv_seq = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        WorkItem wi;
        if (!next_item(k, wi)) break;
        if (wi.idx < 0) continue;
        const FwdUnit w = fwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
        const int je[2] = {w.jend0, w.jend1};
        const int jl[2] = {w.jlast0, w.jlast1};
        for (int t = 0; t < 2 && ok; ++t) {
          if (jl[t] < 0) continue;
          ok = mbar_wait(&q_empty[t], (qload[t] & 1) ^ 1, wc, 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&q_full[t], Lay::kTileBytes);
#pragma unroll
          for (int pn = 0; pn < Lay::kPanels; ++pn)
            tma_load_3d(sq + t * Lay::kTileBytes + pn * Lay::kPanelBytes, &tmq, &q_full[t],
                        pn * Lay::kPanelElems, w.row0 + (w.qt0 + t) * kBlockM, w.z);
          ++qload[t];
        }
        const int jmax = max(je[0], je[1]);
        for (int j = fwd_next<SPARSE>(p, w, 0); j < jmax && ok; j = fwd_next<SPARSE>(p, w, j + 1)) {
          for (int kv = 0; kv < 2; ++kv) {
            const int slot = kv_seq % kSlots;
            const int round = kv_seq / kSlots;
            ok = mbar_wait(&kv_empty[slot], (round & 1) ^ 1, wc, 2);
            if (!ok) break;
            mbar_arrive_expect_tx(&kv_full[slot], Lay::kTileBytes);
            uint8_t* dst = skv + slot * Lay::kTileBytes;
#pragma unroll
            for (int pn = 0; pn < Lay::kPanels; ++pn)
              tma_load_3d(dst + pn * Lay::kPanelBytes, kv ? &tmv : &tmk, &kv_full[slot],
                          pn * Lay::kPanelElems, w.row0 + j * kBlockN, w.z);
            ++kv_seq;
          }
        }
      }
      // Never leave with copies in flight: wait for the last load issued into
      // every barrier (already complete on the normal path).
      for (int t = 0; t < 2; ++t)
        if (qload[t] > 0) mbar_wait_drain(&q_full[t], (qload[t] - 1) & 1, 200000000ull);
      for (int s = 0; s < kSlots; ++s) {
        if (kv_seq > s) {
          const int last = kv_seq - 1 - ((kv_seq - 1 - s) % kSlots);
          mbar_wait_drain(&kv_full[s], (last / kSlots) & 1, 200000000ull);
        }
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t kIdescQK =
          FP8 ? idesc_e4m3(128, 128, false, false) : idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t kIdescPV =
          FP8 ? idesc_e4m3(128, D, false, true) : idesc_f16(BF16, 128, D, false, true);
      const uint32_t sq_addr = smem_addr(sq);
      const uint32_t skv_addr = smem_addr(skv);
      int qload[2] = {0, 0};
      int pcnt[2] = {0, 0};
      int kv_seq = 0;
      bool ok = true;

      // Low descriptor words of the Q tiles and of the K/V ring, K-major and
      // MN-major (V); the grouped MMAs derive the K steps from them.
      constexpr uint32_t kTileLo = Lay::kTileBytes >> 4;
      const uint32_t lQ_k = sdesc_lo(sq_addr, false);
      const uint32_t lKV_k = sdesc_lo(skv_addr, false), lKV_m = sdesc_lo(skv_addr, true);
      // S_t = Q_t K^T: A = Q tile (K-major), B = K tile (K-major).
      auto issue_s = [&](int t, int kslot) {
        if constexpr (FP8)
          umma_ss_group4_e4m3(tmem + t * 128, lQ_k + t * kTileLo, lKV_k + kslot * kTileLo,
                              kIdescQK, 0u);
        else
          umma_ss_group<D / 16, false, false>(tmem + t * 128, lQ_k + t * kTileLo,
                                              lKV_k + kslot * kTileLo, kIdescQK, 0u);
      };
      // O_t += P_t V: A = P (TMEM, over S_t: 16-bit, 8 columns per 16 keys, or
      // e4m3, 8 columns per 32 keys), B = V tile read MN-major (d contiguous).
      auto issue_pv = [&](int t, int vslot, bool acc) {
        if constexpr (FP8)
          umma_ts_group4_e4m3(tmem + Lay::kColO + t * D, tmem + t * 128,
                              lKV_m + vslot * kTileLo, kIdescPV, acc ? 1u : 0u);
        else
          umma_ts_group8<true, false>(tmem + Lay::kColO + t * D, tmem + t * 128,
                                      lKV_m + vslot * kTileLo, kIdescPV, acc ? 1u : 0u);
      };
      for (int k = 0; ok; ++k) {
        WorkItem wi;
        if (!next_item(k, wi)) break;
        if (wi.idx < 0) continue;
        const FwdUnit w = fwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
        const int je[2] = {w.jend0, w.jend1};
        const int jl[2] = {w.jlast0, w.jlast1};
        const int jmax = max(je[0], je[1]);
        const int j0 = fwd_next<SPARSE>(p, w, 0);
        // nothing loaded: both tiles past a packed sequence, or masked out
        if ((PACKED || SPARSE) && j0 >= jmax) continue;
        for (int t = 0; t < 2 && ok; ++t) {
          if (jl[t] < 0) continue;
          ok = mbar_wait(&q_full[t], qload[t] & 1, wc, 3);
          ++qload[t];
        }
        if (!ok) break;
        tc_fence_after();
        // first K tile
        {
          const int slot = kv_seq % kSlots;
          ok = mbar_wait(&kv_full[slot], (kv_seq / kSlots) & 1, wc, 4);
          if (!ok) break;
          tc_fence_after();
          for (int t = 0; t < 2; ++t) {
            if (!fwd_need<SPARSE>(p, w, t, j0)) continue;
            issue_s(t, slot);
            umma_commit(&s_full[t]);
            if (j0 == jl[t]) umma_commit(&q_empty[t]);
          }
          umma_commit(&kv_empty[slot]);
          ++kv_seq;
        }
        int npv[2] = {0, 0};  // P.V issued per query tile in this unit
        for (int j = j0; j < jmax && ok;) {
          const int vslot = kv_seq % kSlots;
          ok = mbar_wait(&kv_full[vslot], (kv_seq / kSlots) & 1, wc, 5);
          if (!ok) break;
          tc_fence_after();
          ++kv_seq;
          const int jn = fwd_next<SPARSE>(p, w, j + 1);  // next streamed key tile
          const int kslot = kv_seq % kSlots;
          bool k_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            if (fwd_need<SPARSE>(p, w, t, j)) {
              ok = mbar_wait(&p_full[t], pcnt[t] & 1, wc, 6);
              if (!ok) break;
              FA_TRACE_AT(pcnt[t], t);
              ++pcnt[t];
              tc_fence_after();
              issue_pv(t, vslot, npv[t] > 0);
              ++npv[t];
              if (j == jl[t]) umma_commit(&o_full[t]);
            }
            if (jn < jmax && fwd_need<SPARSE>(p, w, t, jn)) {
              if (!k_ready) {
                ok = mbar_wait(&kv_full[kslot], (kv_seq / kSlots) & 1, wc, 7);
                if (!ok) break;
                tc_fence_after();
                k_ready = true;
              }
              issue_s(t, kslot);
              umma_commit(&s_full[t]);
              if (jn == jl[t]) umma_commit(&q_empty[t]);
            }
          }
          if (!ok) break;
          umma_commit(&kv_empty[vslot]);
          if (jn < jmax) {
            umma_commit(&kv_empty[kslot]);
            ++kv_seq;
          }
          j = jn;
        }
      }
      // every MMA issued must be complete before TMEM is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0, 200000000ull);
    }
    __syncwarp();
  }
  // warps 10 and 11 have no role
  } else {
    regs_increase<kFwdSoftmaxRegs>();
    // ------------------------------------------------------------- softmax
    const int t = warp >> 2;                 // query tile of the pair
    const int r = ((warp & 3) << 5) | lane;  // row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + Lay::kColO + t * D;
    const float c = p.scale_log2;
    const uint32_t u_drop = 256u - min(p.keep_t, 256u);  // dropout keep test (keep_flags4)
    const uint32_t u_lo7 = (u_drop & 0x7Fu) * 0x01010101u, u_all = u_drop * 0x01010101u;
    int scnt = 0, ocnt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      WorkItem wi;
      if (!next_item(k, wi)) break;
      if (wi.idx < 0) continue;
      const FwdUnit w = fwd_decode<PACKED, SPARSE>(wi.bh, wi.idx, p);
      const int jend = t == 0 ? w.jend0 : w.jend1;
      if (jend == 0) continue;
      const int qt = w.qt0 + t;
      const int row = qt * kBlockM + r;
      if (t == 0 && r == 0 && p.seqlens != nullptr) {
        const int raw = p.seqlens[w.bh / p.H];
        if (raw < 1 || raw > p.N) record_error(kErrDeviceSeqlen, 0);
      }
      if (SPARSE && (t == 0 ? w.jlast0 : w.jlast1) < 0) {
        // the block mask leaves these rows no key: O = 0, LSE = -inf
        if (row < w.rows) {
          const size_t idx = static_cast<size_t>(w.z) * p.N + w.row0 + row;
          uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) + idx * (D * 2);
#pragma unroll
          for (int c16 = 0; c16 < D * 2 / 16; ++c16) st_global_v4(orow + c16 * 16, 0u, 0u, 0u, 0u);
          p.lse[idx] = -INFINITY;
        }
        continue;
      }
      // e4m3 inputs: the query tile's descale and the largest V descale of
      // the slice's valid key tiles; key tile j's probabilities are scaled by
      // sv_j / sv_max before they are rounded to 8 bits, and O by sv_max at
      // the end, so one TMEM accumulator serves tiles of any V scale
      float sq_t = 1.f, sv_max = 1.f;
      const float* kds = nullptr;
      const float* vds = nullptr;
      if constexpr (FP8) {
        const size_t base = static_cast<size_t>(w.bh) * p.n_qtiles;
        kds = p.k_descale + base;
        vds = p.v_descale + base;
        sq_t = p.q_descale[base + qt];
        const int nkb = (w.L + kBlockN - 1) / kBlockN;
        sv_max = 0.f;
        for (int jv = 0; jv < nkb; ++jv) sv_max = fmaxf(sv_max, vds[jv]);
        if (!(sq_t > 0.f && sq_t < INFINITY && sv_max > 0.f && sv_max < INFINITY))
          record_error(kErrDeviceScale, 0);
      }
      float m = -INFINITY;  // running max, log2 units
      float l = 0.f;        // running sum of unnormalised probabilities
      int jj = 0;           // key tiles processed so far
      for (int j = 0; j < jend; ++j) {
        if (!fwd_need<SPARSE>(p, w, t, j)) continue;
        // dropout: keep flags of this row for key tile j (keep_flags_row128),
        // made while the tensor core computes S
        uint32_t drop_keep[4] = {~0u, ~0u, ~0u, ~0u};
        if constexpr (DROPOUT) {
          keep_flags_row128(p, w.bh, row, j, lane & 3, u_lo7, u_all, drop_keep);
          if (r == 0 && t == 0) FA_TRACE_AT(scnt, 15);
        }
        // scores of this tile are raw * cj in log2 units
        float cj = c, rho = 1.f, inv_rho = 1.f;
        if constexpr (FP8) {
          const float skj = kds[j], svj = vds[j];
          if (!(skj > 0.f && skj < INFINITY && svj > 0.f && svj < INFINITY))
            record_error(kErrDeviceScale, 1);
          cj = c * sq_t * skj;
          rho = svj / sv_max;
          inv_rho = sv_max / svj;
        }
        ok = mbar_wait_warp(&s_full[t], scnt & 1, wc, 8);
        if (!ok) break;
        if (r == 0) FA_TRACE_AT(scnt, 2 + 2 * t);
        ++scnt;
        tc_fence_after();
        uint32_t sr[128];  // raw scores q.k of this row, one TMEM load
        tmem_ld128(tS, sr);
        if (r == 0 && t == 0) FA_TRACE_AT(scnt - 1, 6);
        const int kbase = j * kBlockN;
        const bool need_mask = (p.causal && j == qt) || (kbase + kBlockN > w.L);
        if (need_mask) {
          const int lim = p.causal ? min(w.L, row + 1) : w.L;  // keys < lim are visible
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (kbase + i >= lim) sr[i] = __float_as_uint(-INFINITY);
        }
        // row max of the raw scores: four independent 3-input max chains,
        // chain q4 takes elements 8k + 2 q4 and 8k + 2 q4 + 1
        float mc[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          mc[q4] = fmaxf(__uint_as_float(sr[2 * q4]), __uint_as_float(sr[2 * q4 + 1]));
#pragma unroll
        for (int i = 8; i < 128; i += 8) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            mc[q4] = fmax3(mc[q4], __uint_as_float(sr[i + 2 * q4]), __uint_as_float(sr[i + 2 * q4 + 1]));
        }
        const float mx = fmax3(mc[0], mc[1], fmaxf(mc[2], mc[3])) * cj;  // log2 units (cj > 0)
        const float m_new = (mx > m + kRescaleThreshold) ? mx : m;
        const bool moved = m_new != m;
        if (r == 0 && t == 0) FA_TRACE_AT(scnt - 1, 7);
        const float alpha = moved ? ex2_approx(m - m_new) : 1.f;  // 0 when m was -inf
        l *= alpha;
        m = m_new;
        // O_t holds the sum up to the previous key tile (its MMA completed
        // before S_t(j) was committed) and PV_t(j) waits for p_full: when a
        // row's max moved, rescale O_t before that signal; rows that did not
        // move multiply by 1
        const bool rescale = jj > 0 && __any_sync(0xffffffffu, moved);
        auto rescale_o = [&]() {
#pragma unroll 1
          for (int cc = 0; cc < D / 16; ++cc) {
            uint32_t ro[16];
            tmem_ld16(tO + cc * 16, ro);
#pragma unroll
            for (int e = 0; e < 16; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
            tmem_st_n<16>(tO + cc * 16, ro);
          }
        };
        // p = 2^(c s - m): packed FMA on pairs, then ex2; row sum in fp32 over
        // four packed accumulators
        // e4m3: p rho_j = 2^(c s - m + log2 rho_j) is formed directly (the V
        // descale ratio rides in the exponent), and the row sum divides it back
        const float mu = (m == -INFINITY) ? 0.f : m;
        const float bias = FP8 ? lg2_approx(rho) - mu : -mu;
        const unsigned long long c2 = f2pack(cj, cj);
        const unsigned long long nm2 = f2pack(bias, bias);
        unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[FP8 ? 32 : 64];  // P as the A operand: 16-bit pairs or e4m3 quads
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const unsigned long long x2 =
              ffma2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, nm2);
          float x0, x1;
          f2unpack(x2, x0, x1);
          const unsigned long long p2 = f2pack(ex2_approx(x0), ex2_approx(x1));
          acc[i & 3] = fadd2(acc[i & 3], p2);
          float p0, p1;
          f2unpack(p2, p0, p1);
          if constexpr (FP8) {
            const uint32_t h = pack_e4m3x2(p0, p1);
            pk[i >> 1] = (i & 1) ? (pk[i >> 1] | (h << 16)) : h;
          } else {
            pk[i] = pack2<BF16>(p0, p1);
          }
          if constexpr (DROPOUT) {  // dropped scores leave the row sum, not P V
            // keys 2 i, 2 i + 1 = 32 h + 16 e + 4 s + c with c = 2 (i & 1)
            const int sh = ((i >> 1) & 3) + 4 * ((i >> 3) & 1);
            pk[i] &= pair_keep_mask(drop_keep[i >> 4] << sh, i & 1);
          }
          if (r == 0 && t == 0 && (i & 15) == 15) FA_TRACE_AT(scnt - 1, 8 + (i >> 4));
        }
        {
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f2unpack(acc[0], a0, a1);
          f2unpack(acc[1], b0, b1);
          f2unpack(acc[2], c0, c1);
          f2unpack(acc[3], d0, d1);
          const float sum = ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
          l += FP8 ? sum * inv_rho : sum;
        }
        if constexpr (FP8) tmem_st32(tS, pk);
        else tmem_st64(tS, pk);
        if (rescale) rescale_o();
        if (r == 0 && t == 0) FA_TRACE_AT(scnt - 1, 12);
        tmem_st_wait();
        if (r == 0 && t == 0) FA_TRACE_AT(scnt - 1, 14);
        tc_fence_before();
        mbar_arrive(&p_full[t]);
        if (r == 0) FA_TRACE_AT(scnt - 1, 3 + 2 * t);
        ++jj;
      }
      if (!ok) break;
      // epilogue: O / l -> 16-bit, LSE
      ok = mbar_wait_warp(&o_full[t], ocnt & 1, wc, 9);
      if (!ok) break;
      ++ocnt;
      tc_fence_after();
      // (with dropout the kept scores are scaled by 256 / t once, here; with
      // e4m3 inputs the V descale ratio is undone)
      const float inv_l = FP8 ? sv_max / l : (DROPOUT ? p.inv_keep / l : 1.f / l);
      const bool store = row < w.rows;
      const size_t orow_idx = static_cast<size_t>(w.z) * p.N + w.row0 + (store ? row : 0);
      // O rows are o_cols wide: D, or 64 for e4m3 inputs with d = 64, whose
      // columns 64..127 of the accumulator are zero (zero-filled V columns)
      const int o_cols = FP8 ? p.o_cols : D;
      uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) + orow_idx * (o_cols * 2);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        if (FP8 && cc * 32 >= o_cols) break;
        uint32_t ro[32];
        tmem_ld32(tO + cc * 32, ro);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack2<BF16>(__uint_as_float(ro[2 * i]) * inv_l, __uint_as_float(ro[2 * i + 1]) * inv_l);
        if (store) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            st_global_v4(orow + cc * 64 + v4 * 16, pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2],
                         pk[4 * v4 + 3]);
        }
      }
      if (store) p.lse[orow_idx] = (m + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

template <int D, bool BF16, bool PACKED, bool SPARSE, bool DROPOUT, bool FP8 = false>
static cudaError_t launch_fwd_t(const CUtensorMap& tmq, const CUtensorMap& tmk,
                                const CUtensorMap& tmv, const FwdParams& p, int num_sms,
                                cudaStream_t stream) {
  using Lay = FwdLayout<D, FP8 ? 1 : 2>;
  auto kern = fa_fwd_kernel<D, BF16, PACKED, SPARSE, DROPOUT, FP8>;
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  // the register split in the kernel assumes exactly this launch allocation
  if (attr.numRegs != kFwdLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.n_units < num_sms ? p.n_units : num_sms;
  kern<<<grid, 384, Lay::kSmemBytes, stream>>>(tmq, tmk, tmv, p);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int d, bool bf16, const CUtensorMap& tmq, const CUtensorMap& tmk,
                       const CUtensorMap& tmv, const FwdParams& p, int num_sms,
                       cudaStream_t stream) {
  const int mode = p.cu_seqlens != nullptr ? 1
                   : p.block_mask != nullptr ? 2
                   : p.keep_t < 256u        ? 3
                                            : 0;
#define FA_FWD_LAUNCH(DD, BB, PP, SS, RR) \
  launch_fwd_t<DD, BB, PP, SS, RR>(tmq, tmk, tmv, p, num_sms, stream)
#define FA_FWD_MODES(DD, BB)                                                \
  (mode == 1   ? FA_FWD_LAUNCH(DD, BB, true, false, false)                  \
   : mode == 2 ? FA_FWD_LAUNCH(DD, BB, false, true, false)                  \
   : mode == 3 ? FA_FWD_LAUNCH(DD, BB, false, false, true)                  \
               : FA_FWD_LAUNCH(DD, BB, false, false, false))
  if (d == 128) return bf16 ? FA_FWD_MODES(128, true) : FA_FWD_MODES(128, false);
  return bf16 ? FA_FWD_MODES(64, true) : FA_FWD_MODES(64, false);
#undef FA_FWD_MODES
#undef FA_FWD_LAUNCH
}

cudaError_t launch_fwd_e4m3(bool bf16, const CUtensorMap& tmq, const CUtensorMap& tmk,
                            const CUtensorMap& tmv, const FwdParams& p, int num_sms,
                            cudaStream_t stream) {
  return bf16 ? launch_fwd_t<128, true, false, false, false, true>(tmq, tmk, tmv, p, num_sms, stream)
              : launch_fwd_t<128, false, false, false, false, true>(tmq, tmk, tmv, p, num_sms,
                                                                    stream);
}

}  // namespace fa
