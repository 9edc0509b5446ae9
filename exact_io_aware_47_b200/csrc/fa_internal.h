// Parameters shared between the host launchers and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace fa {

constexpr int kBlockM = 128;  // query rows per tile (TMEM lanes)
constexpr int kBlockN = 128;  // keys per tile

// Lazy-rescale threshold in log2 units: the running row max is only moved
// when a tile's max exceeds it by more than this, so unnormalised
// probabilities stay below 2^8 and the final division by the row sum (taken
// with the same max) still yields the exact softmax.
constexpr float kRescaleThreshold = 8.0f;

// Two layouts share the kernels.  Fixed length: tensors [B, H, N, d], a
// (batch, head) slice is row block b * H + h of N rows.  Packed (cu_seqlens
// given): tensors [H, T, d] with the B sequences of head h back to back,
// sequence b in rows [cu_seqlens[b], cu_seqlens[b + 1]) of block h; N holds T
// and the tile counts come from max_seqlen.
struct FwdParams {
  void* o;                  // [B, H, N, d] or [H, T, d], 16-bit
  float* lse;               // [B, H, N] or [H, T] natural-log log-sum-exp
  const int32_t* seqlens;   // [B] valid key lengths (fixed length), or nullptr
  const int32_t* cu_seqlens;  // [B + 1] sequence offsets (packed), or nullptr
  int max_seqlen;           // packed: upper bound of every sequence length
  const uint8_t* block_mask;  // block-sparse: [n_qtiles][n_qtiles] tile mask, or nullptr
  // dropout (kernels instantiated with DROPOUT): Philox key, counter word 3,
  // 8-bit keep threshold t (1..256) and 256 / t
  uint32_t seed_lo, seed_hi, drop_offset, keep_t;
  float inv_keep;
  // e4m3 inputs (kernels instantiated with FP8): one descale factor per
  // 128-row tile, [B, H, n_qtiles] each; the tensors stand for code * descale
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
  int B, H, N;
  int o_cols;               // columns of O (d); the e4m3 kernel reads d = 64 inputs as 128
                            // columns, the TMA load filling columns 64..127 with zeros
  float scale_log2;         // scale * log2(e)
  int causal;
  int n_qtiles;             // ceil(N / 128)
  int n_pairs;              // ceil(n_qtiles / 2): a work unit is two query tiles
  int n_units;              // B * H * ceil(n_pairs / 2) super-units (see work_item)
  unsigned long long wait_ns;  // bound of one pipeline wait (kErrDeviceTimeout past it)
};

struct BwdParams {
  const void* q;            // [B, H, N, d] 16-bit
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;         // [B, H, N]
  void* dq;                 // [B, H, N, d] 16-bit outputs
  void* dk;
  void* dv;
  float* dsum;              // workspace [B, H, N]: D_i = <dO_i, O_i>
  float* dq_acc;            // workspace [B, H, N, d] fp32 accumulator
  const int32_t* seqlens;
  const int32_t* cu_seqlens;  // as in FwdParams
  int max_seqlen;
  const uint8_t* block_mask;  // as in FwdParams ([n_ktiles][n_ktiles])
  // packed batches: longest-first work order (workspace, built by
  // fa_bwd_rank): lengths [B], sequences by rank [B], super-units before each
  // rank [B + 1]; nullptr: head-major order
  int* rank;
  uint32_t seed_lo, seed_hi, drop_offset, keep_t;  // as in FwdParams
  float inv_keep;
  int B, H, N;
  float scale;
  float scale_log2;
  int causal;
  int n_ktiles;             // ceil(N / 128)
  int n_units;              // B * H * ceil(n_ktiles / 2) super-units (see work_item)
  unsigned long long wait_ns;  // bound of one pipeline wait (kErrDeviceTimeout past it)
};

// Work order of the persistent kernels.  A head's units (query-tile pairs in
// the forward, key tiles in the backward) are paired with their mirror: unit
// m and unit n-1-m form one super-unit, which costs the same for every m
// under a causal mask (long + short).  CTA c takes super-units c, c + grid,
// ... (head-major, so CTAs running together share K/V and dQ rows in L2) and
// runs the two halves back to back.  k counts the work items of this CTA;
// returns false past the end; idx < 0 marks the missing mirror of an odd
// middle unit.
// Where a (batch, head) slice lives and how long it is: rows [row0, row0 + L)
// of row block z (z = b * H + h, row0 = 0, L = seqlens[b] or N for fixed
// length; z = h, row0 = cu_seqlens[b] packed).  `rows` bounds the query rows
// that are computed and stored: N for fixed length (padded query rows are
// still computed), L packed (the rows after L belong to the next sequence).
// Out-of-range sequence descriptions are clamped and reported.  The kernels
// are instantiated per layout (PACKED), so the fixed-length code carries no
// trace of the packed one.
struct SliceInfo {
  int z, row0, L, rows;
};

template <bool PACKED, class P>
__device__ __forceinline__ SliceInfo slice_info(int bh, const P& p, int err_code) {
  SliceInfo s;
  const int b = bh / p.H;
  if constexpr (PACKED) {
    int s0 = p.cu_seqlens[b], s1 = p.cu_seqlens[b + 1];
    const int c0 = min(max(s0, 0), p.N);
    const int c1 = min(max(s1, c0), min(p.N, c0 + p.max_seqlen));
    if (c0 != s0 || c1 != s1) record_error(err_code, 1);
    s.z = bh - b * p.H;
    s.row0 = c0;
    s.L = c1 - c0;
    s.rows = s.L;
  } else {
    int L = p.N;
    if (p.seqlens != nullptr) {
      L = p.seqlens[b];
      L = L < 1 ? 1 : (L > p.N ? p.N : L);
    }
    s.z = bh;
    s.row0 = 0;
    s.L = L;
    s.rows = p.N;
  }
  return s;
}

// Rows of all (batch, head) slices together (the element-wise kernels).
template <class P>
__host__ __device__ inline long long total_rows(const P& p) {
  return p.cu_seqlens != nullptr ? static_cast<long long>(p.H) * p.N
                                 : static_cast<long long>(p.B) * p.H * p.N;
}

// Block-sparse attention (kernels instantiated with SPARSE): the 128 x 128
// score tile (query tile qt, key tile kt) is computed only if
// block_mask[qt * ntiles + kt] != 0, for every (batch, head) slice.
__device__ __forceinline__ bool tile_allowed(const uint8_t* block_mask, int ntiles, int qt, int kt) {
  return block_mask[static_cast<size_t>(qt) * ntiles + kt] != 0;
}

// Dropout keep bits of one 4 x 4 block of scores, as the four lanes of a quad
// need them.  The generator call for block (query block qb, key block kb) of
// slice bh uses counter (kb, qb, bh, offset); word w of its result belongs to
// query row 4 qb + w and byte c of that word to key 4 kb + c; a score is kept
// iff its byte is below keep_t.
//
// Forward (lanes = 4 consecutive query rows, lane w = row & 3): keep flags
// of this thread's row for the 128 keys of key tile j.  Group g of 16 keys
// (keys 16 g + 4 s + c) is the generator call with key block 32 j + 4 g + w;
// the eight calls run interleaved.  Key k = 32 h + 16 e + 4 s + c of the
// tile is bit 8 c + 7 - s - 4 e of m[h] (the byte-wise flags of keep_flags4,
// merged four words to one and two groups to one word): a pair of keys
// 2 i, 2 i + 1 sits in bits 8 c + 7 and 8 c + 15 of m[h] << (s + 4 e), the
// form pair_keep_mask reads.
template <class P>
__device__ __forceinline__ void keep_flags_row128(const P& p, int bh, int row, int j, int w,
                                                  uint32_t u_lo7, uint32_t u_all,
                                                  uint32_t (&m)[4]) {
  uint32_t a[8][4];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    a[g][0] = static_cast<uint32_t>(32 * j + 4 * g + w);
    a[g][1] = static_cast<uint32_t>(row >> 2);
    a[g][2] = static_cast<uint32_t>(bh);
    a[g][3] = p.drop_offset;
  }
  philox4x32_10_n<8>(a, p.seed_lo, p.seed_hi);
  uint32_t grp[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    quad_transpose4(a[g], w);  // a[g][s]: this row's word of key block 4 g + s
    grp[g] = merge_flags4(keep_flags4(a[g][0], u_lo7, u_all), keep_flags4(a[g][1], u_lo7, u_all),
                          keep_flags4(a[g][2], u_lo7, u_all), keep_flags4(a[g][3], u_lo7, u_all));
  }
#pragma unroll
  for (int h = 0; h < 4; ++h) m[h] = bit_select(grp[2 * h], grp[2 * h + 1] >> 4, 0xF0F0F0F0u);
}

// Backward (lanes = 4 consecutive keys, lane w = key & 3): keep flags of
// this thread's key for 64 queries q0 .. q0 + 63 (q0 a multiple of 64).
// Group g of 16 queries (q0 + 16 g + 4 s + c) is the generator call with
// query block q0 / 4 + 4 g + w.  Query
// q0 + 32 h + 16 e + 4 s + c is bit 8 c + 7 - s - 4 e of m[h], the layout of
// keep_flags_row128.
template <class P>
__device__ __forceinline__ void keep_flags_key64(const P& p, int bh, int key, int q0, int w,
                                                 uint32_t u_lo7, uint32_t u_all,
                                                 uint32_t (&m)[2]) {
  uint32_t a[4][4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    a[g][0] = static_cast<uint32_t>(key >> 2);
    a[g][1] = static_cast<uint32_t>((q0 >> 2) + 4 * g + w);
    a[g][2] = static_cast<uint32_t>(bh);
    a[g][3] = p.drop_offset;
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) philox4x32_10(a[g], p.seed_lo, p.seed_hi);
  uint32_t grp[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    byte_transpose4(a[g]);     // a[g][c] = key c's bytes of the 4 queries
    quad_transpose4(a[g], w);  // a[g][s] = this key's bytes of query block q0 / 4 + 4 g + s
    grp[g] = merge_flags4(keep_flags4(a[g][0], u_lo7, u_all), keep_flags4(a[g][1], u_lo7, u_all),
                          keep_flags4(a[g][2], u_lo7, u_all), keep_flags4(a[g][3], u_lo7, u_all));
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) m[h] = bit_select(grp[2 * h], grp[2 * h + 1] >> 4, 0xF0F0F0F0u);
}

struct WorkItem {
  int bh;   // batch * head
  int idx;  // unit index inside the head: n-1-m for the first half, m for the second
};

__device__ __forceinline__ bool work_item(int k, int per_head, int heads, WorkItem& wi) {
  const int half = (per_head + 1) >> 1;
  const int su = blockIdx.x + (k >> 1) * gridDim.x;
  if (su >= heads * half) return false;
  wi.bh = su / half;
  const int m = su - wi.bh * half;
  const int a = per_head - 1 - m;
  wi.idx = (k & 1) == 0 ? a : (m != a ? m : -1);
  return true;
}

// Host launchers (defined in the .cu files).  They assume validated
// arguments and return a cudaError_t from the launch.
cudaError_t launch_fwd(int d, bool bf16, const CUtensorMap& tmq, const CUtensorMap& tmk,
                       const CUtensorMap& tmv, const FwdParams& p, int num_sms,
                       cudaStream_t stream);
// e4m3 inputs (p.q_descale set), d = 128; bf16 selects the output type.
cudaError_t launch_fwd_e4m3(bool bf16, const CUtensorMap& tmq, const CUtensorMap& tmk,
                            const CUtensorMap& tmv, const FwdParams& p, int num_sms,
                            cudaStream_t stream);
// Per-tile e4m3 quantisation of a [rows_total / n_rows, n_rows, d] 16-bit tensor.
cudaError_t launch_quantize_e4m3(int d, bool bf16, const void* x, void* x8, float* descale,
                                 long long slices, int n_rows, int num_sms, cudaStream_t stream);

cudaError_t launch_bwd_pre(int d, bool bf16, const BwdParams& p, int num_sms,
                           cudaStream_t stream);
cudaError_t launch_bwd_main(int d, bool bf16, const CUtensorMap& tmq, const CUtensorMap& tmk,
                            const CUtensorMap& tmv, const CUtensorMap& tmdo,
                            const CUtensorMap& tmdq, const BwdParams& p, int num_sms,
                            cudaStream_t stream);
cudaError_t launch_bwd_post(int d, bool bf16, const BwdParams& p, int num_sms,
                            cudaStream_t stream);
// Packed batches of at most this many sequences get the longest-first
// backward order; the table takes 3 B + 1 ints of the workspace.
constexpr int kBwdRankMaxSeqs = 4096;
cudaError_t launch_bwd_rank(const BwdParams& p, cudaStream_t stream);

}  // namespace fa
