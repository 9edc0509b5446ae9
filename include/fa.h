/*
 * fa.h - C ABI of the B200 (sm_100a) exact tiled attention library
 *        (libfa_b200.so).
 *
 * Operation.  Exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T  [+ causal / key-padding mask]) V
 *
 * computed tile by tile with an online softmax, so that no N x N score or
 * probability matrix is ever written to device memory:
 *   - "How Flash Attention Works" (swarnava.dev), section "The Exact-Attention
 *     Idea": the result is the unchanged softmax(QK^T/sqrt(d))V, with causal
 *     masking when asked for;
 *   - same page, sections "Tiling Q, K, and V", "Online Softmax Without the
 *     Full Score Matrix" and "Kernel Fusion": query tiles stay on chip, K/V
 *     tiles stream past them, running row max and row sum rescale the partial
 *     output, only O and per-row statistics reach memory;
 *   - same page, section "The Backward Pass: Recomputation Instead of Stored
 *     Activations": the backward pass keeps only O and the per-row statistics
 *     and recomputes the score tiles;
 *   - "attn-flash-equivalence" (zenaique.com), opening answer: the output
 *     equals naive attention up to floating-point reduction order, so results
 *     agree with a float64 evaluation within rounding, not bit for bit.
 *
 * Conventions shared by every entry point.
 *   Layout.  Q, K, V, O, dO, dQ, dK, dV are dense, contiguous [B, H, N, d]
 *     tensors (d innermost), 16-bit (bf16 or fp16, all the same type).
 *     LSE is [B, H, N] float32, natural log:  LSE_i = ln sum_j exp(scale*s_ij)
 *     over the visible keys.  seqlens is a device int32 [B] array or NULL.
 *   Masks.  causal != 0 hides key j from query i when j > i (top-left
 *     aligned; queries and keys have the same length N).  seqlens[b] = L
 *     hides keys j >= L of batch b from every query (key padding); query rows
 *     i >= L are still computed.  1 <= L <= N is required; other values are
 *     clamped into range on the device and reported by fa_device_status().
 *   Sizes.  B, H, N >= 1; d in {64, 128}; B*H*N*d < 2^31.
 *   Scale.  finite and > 0 (typically 1/sqrt(d)).
 *   Memory.  All pointers are device pointers owned by the caller, 16-byte
 *     aligned.  The library allocates no device memory and keeps no state
 *     other than cached driver entry points, per-device properties and the
 *     wait bound of fa_set_wait_limit_ns().
 *   Streams.  stream is a cudaStream_t (NULL = legacy default stream).  Work
 *     is enqueued asynchronously; no entry point synchronises except
 *     fa_device_status().
 *   Errors.  Return FA_OK or an fa_status code.  Argument errors are found on
 *     the host before anything is launched.  Device-side conditions (bad
 *     seqlens values, a pipeline wait that timed out) are written to a device
 *     status word, read and cleared by fa_device_status().  The library never
 *     aborts the process and never traps on the device.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* null pointer, size < 1, bad scale or dtype    */
  FA_ERR_UNSUPPORTED = 2,     /* head dim not in {64, 128}, sizes too large     */
  FA_ERR_ALIGNMENT = 3,       /* a pointer is not 16-byte aligned               */
  FA_ERR_ARCH = 4,            /* current device is not an sm_100 (B200) GPU     */
  FA_ERR_CUDA = 5,            /* a CUDA runtime/driver call or launch failed    */
  FA_ERR_DEVICE_TIMEOUT = 6,  /* device: a pipeline wait gave up (fa_device_status) */
  FA_ERR_DEVICE_SEQLEN = 7,   /* device: seqlens[b] outside [1, N] (fa_device_status) */
  FA_ERR_WORKSPACE = 8,       /* backward workspace missing or too small        */
  FA_ERR_DEVICE_LAYOUT = 9,   /* device: shared-memory window misaligned, kernel refused (fa_device_status) */
  FA_ERR_SCRATCH_LIMIT = 10,  /* fa_bwd_noalloc: workspace would exceed its static array */
  FA_ERR_DEVICE_SCALE = 11    /* device: e4m3 descale not finite and > 0, or infinite or NaN
                                 input to fa_quantize_e4m3 (fa_device_status) */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/*
 * Forward pass.
 *   in : q, k, v       [B, H, N, d] 16-bit
 *   out: o             [B, H, N, d] 16-bit, rounded to nearest from fp32
 *        lse           [B, H, N] float32 log-sum-exp of the scaled scores
 *   Launches one persistent kernel on `stream`.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, float scale, int causal,
           const int32_t* seqlens, int dtype, void* stream);

/*
 * Bytes of device workspace fa_bwd needs: the row dots D = rowsum(dO * O)
 * (float32 [B, H, N]) and the float32 dQ accumulator ([B, H, N, d]), each
 * padded to 256 bytes.  Returns 0 for arguments fa_bwd would reject.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass of the loss <dO, O> (gradients of the forward above).
 *   in : q, k, v, o, dout  [B, H, N, d] 16-bit (o and lse from fa_fwd with the
 *        same arguments), lse [B, H, N] float32
 *   out: dq, dk, dv        [B, H, N, d] 16-bit; keys hidden by key padding get
 *        exactly zero dK and dV
 *   workspace: caller-owned device memory of at least
 *        fa_bwd_workspace_size(B, H, N, d) bytes, 256-byte aligned; its
 *        contents on entry do not matter and are overwritten.
 *   Launches three kernels on `stream` (row-dot preprocess, main, dQ convert).
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o,
           const void* dout, const float* lse, void* dq, void* dk, void* dv,
           void* workspace, size_t workspace_bytes,
           int B, int H, int N, int d, float scale, int causal,
           const int32_t* seqlens, int dtype, void* stream);

/*
 * The three stages fa_bwd runs, callable one by one (same arguments and
 * checks; fa_bwd is exactly these three calls in this order on one stream).
 *   fa_bwd_preprocess : workspace <- D_i = sum_c dO_ic O_ic (float32, from the
 *                       16-bit O and dO) and a zeroed float32 dQ accumulator.
 *   fa_bwd_main       : dk, dv written; float32 dQ accumulator reduce-added in
 *                       the workspace (needs the preprocess result).
 *   fa_bwd_postprocess: dq <- scale * accumulator, rounded to 16-bit.
 */
int fa_bwd_preprocess(const void* o, const void* dout, void* workspace,
                      size_t workspace_bytes, int B, int H, int N, int d,
                      int dtype, void* stream);
int fa_bwd_main(const void* q, const void* k, const void* v, const void* dout,
                const float* lse, void* dk, void* dv, void* workspace,
                size_t workspace_bytes, int B, int H, int N, int d, float scale,
                int causal, const int32_t* seqlens, int dtype, void* stream);
int fa_bwd_postprocess(void* workspace, size_t workspace_bytes, void* dq,
                       int B, int H, int N, int d, float scale, int dtype,
                       void* stream);

/*
 * Dropout on the attention probabilities, fused into both passes ("How Flash
 * Attention Works", sections "Why Standard Attention Becomes a GPU Memory
 * I/O Bottleneck": dropout comes after the softmax and before the product
 * with V; "Kernel Fusion and Incremental Output Accumulation": it is fused,
 * so the mask is regenerated, never stored).  Same layout, masks and checks
 * as fa_fwd / fa_bwd, plus:
 *   p_drop in [0, 1): scores are kept with probability t / 256, where
 *     t = round(256 (1 - p_drop)) (ties to even, clamped to [1, 256]), and
 *     kept probabilities are scaled by 256 / t:  O = (P * Z) V * 256 / t.
 *     LSE is that of the scores (unaffected by dropout).  t = 256 (p_drop
 *     below 1/512) runs the plain kernels.
 *   seed, offset: the keep mask Z is a function of (seed, offset, batch,
 *     head, query, key) only, from the counter-based generator Philox4x32-10
 *     (Salmon et al., SC 2011): the call with counter (key / 4, query / 4,
 *     b * H + h, offset) and key seed covers a 4 x 4 block; its word
 *     query % 4, byte key % 4 is compared with t.  fa_bwd_dropout must get
 *     the seed, offset and p_drop of the forward call.
 *   Gradients are those of the loss <dO, O> for that fixed mask.
 *   Returns FA_ERR_INVALID_ARG for p_drop outside [0, 1).
 */
int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int N, int d, float scale, int causal,
                   const int32_t* seqlens, float p_drop, uint64_t seed, uint32_t offset,
                   int dtype, void* stream);
int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv,
                   void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                   float scale, int causal, const int32_t* seqlens, float p_drop,
                   uint64_t seed, uint32_t offset, int dtype, void* stream);

/*
 * 8-bit (e4m3) inputs with per-tile scaling: the lower-precision path that
 * "How Flash Attention Works" (section "FlashAttention 2 and 3") names.
 *   Format.  e4m3 as in the OCP 8-bit floating-point specification (sign,
 *     4 exponent bits with bias 7, 3 mantissa bits, largest finite 448, no
 *     infinities); one byte per element.
 *   fa_quantize_e4m3: x [B, H, N, d] 16-bit (dtype FA_BF16 / FA_FP16, finite
 *     values) -> x8 [B, H, N, d] e4m3 codes and descale [B, H, ceil(N/128)]
 *     float32.  Tile t of a (batch, head) slice is rows 128 t .. 128 t + 127
 *     (the last tile may be short).  With amax = max |x| over the tile:
 *     descale = amax / 448 and each code = e4m3(x * (448 / amax)), both
 *     divisions and the product in fp32 rounded to nearest, the conversion
 *     round-to-nearest-even and saturating; a tile of zeros gets descale 1.
 *     d in {64, 128}.  An infinite or NaN input is reported as
 *     FA_ERR_DEVICE_SCALE (that tile's descale and codes are then unspecified).
 *   fa_fwd_e4m3: forward attention of Q, K, V given as e4m3 codes
 *     [B, H, N, d] with descales [B, H, ceil(N/128)] (any positive finite
 *     values; the quantiser's output is one choice): the tensors stand for
 *     code * descale of the row's tile.  Scores, masks, seqlens and LSE are
 *     as in fa_fwd, on those values.  For the product with V the
 *     probabilities of key tile j (against the running row max, which moves
 *     only by more than 8 in log2 units) are multiplied by
 *     sv_j / max sv (the largest V descale of the slice's valid key tiles;
 *     formed as 2^(c s - m + log2(sv_j / max sv))) and rounded to e4m3; the
 *     row sum uses them before rounding, divided back by sv_j / max sv; O =
 *     max sv * sum / l in out_dtype (FA_BF16 or FA_FP16) [B, H, N, d].
 *     d in {64, 128}: d = 64 runs the d = 128 kernel, whose loads fill
 *     columns 64..127 with zeros (same results, the d = 128 time).
 *     FA_ERR_UNSUPPORTED for other d.  Descale pointers must be
 *     4-byte aligned, the others 16-byte aligned.  A descale that is not
 *     finite and positive is reported as FA_ERR_DEVICE_SCALE (the results are
 *     then unspecified).
 *   Ownership and errors as in fa_fwd: the caller owns every buffer; nothing
 *   is allocated; the calls enqueue on `stream` and never synchronise.
 */
int fa_quantize_e4m3(const void* x, void* x8, float* descale, int B, int H, int N, int d,
                     int dtype, void* stream);
int fa_fwd_e4m3(const void* q8, const void* k8, const void* v8, const float* q_descale,
                const float* k_descale, const float* v_descale, void* o, float* lse,
                int B, int H, int N, int d, float scale, int causal,
                const int32_t* seqlens, int out_dtype, void* stream);

/*
 * Packed variable-length batches: B sequences of different lengths stored
 * back to back, with no padding rows.  Same method, masks and numerics as
 * fa_fwd / fa_bwd, with each sequence its own attention problem: queries of
 * sequence b see only keys of sequence b ("How Flash Attention Works",
 * section "Tiling Q, K, and V": the sequence is tiled and ragged edges are
 * masked per tile; here the edges are the sequence boundaries).
 *   Layout.  Q, K, V, O, dO, dQ, dK, dV are [H, T, d] 16-bit: head-major like
 *     the fixed-length tensors, with the B sequences of every head
 *     concatenated along the T rows.  LSE is [H, T] float32.  cu_seqlens is a
 *     device int32 [B + 1] array of row offsets: sequence b occupies rows
 *     cu_seqlens[b] .. cu_seqlens[b + 1] - 1 of every head, with
 *     0 = cu_seqlens[0] <= ... <= cu_seqlens[B] = T.  Empty sequences are
 *     allowed.  max_seqlen (host int) bounds every length; it sets the work
 *     decomposition, so a tight bound wastes no work.
 *   Masks.  causal != 0 hides key j from query i of the same sequence when
 *     j > i (positions counted from the sequence start).  Rows of other
 *     sequences never enter a sequence's result.  Rows outside
 *     [cu_seqlens[0], cu_seqlens[B]) belong to no sequence: o, lse, dk and
 *     dv leave them untouched, dq gets zeros there.
 *   Sizes.  B, H, T, max_seqlen >= 1; d in {64, 128}; H*T*d < 2^31;
 *     B*H*ceil(min(max_seqlen, T) / 128) < 2^31.  A cu_seqlens description
 *     that is out of range (decreasing, past T, a sequence longer than
 *     max_seqlen) is clamped on the device and reported by
 *     fa_device_status() as FA_ERR_DEVICE_SEQLEN.
 *   fa_bwd_varlen's workspace: fa_bwd_varlen_workspace_size(B, H, T, d)
 *     bytes, 256-byte aligned: the row dots and dQ accumulator of
 *     fa_bwd_workspace_size(1, H, T, d), then (for B <= 4096) the table of
 *     the longest-first work order.  It runs the three backward stages on
 *     `stream`, with a one-block kernel that ranks the sequences by length
 *     before the main kernel (B > 4096: head-major order, no table).
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int32_t* cu_seqlens, int B, int H, int T, int max_seqlen,
                  int d, float scale, int causal, int dtype, void* stream);
size_t fa_bwd_varlen_workspace_size(int B, int H, int T, int d);
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                  const void* dout, const float* lse, void* dq, void* dk, void* dv,
                  void* workspace, size_t workspace_bytes, const int32_t* cu_seqlens,
                  int B, int H, int T, int max_seqlen, int d, float scale, int causal,
                  int dtype, void* stream);

/*
 * Block-sparse attention ("sparse-attention-flashattention" glossary page,
 * definition: the original paper's block-sparse extension, a separate
 * configuration of the same exact attention).  Same layout, masks and
 * numerics as fa_fwd / fa_bwd, plus a tile mask: the 128 x 128 block of
 * scores (query tile qt, key tile kt) is computed only if
 * block_mask[qt * nt + kt] != 0, nt = ceil(N / 128); the softmax runs over
 * the scores that remain (block mask, causal and key-length masks together).
 * Skipped blocks cost no work: a K/V tile is loaded only if some query tile
 * of the CTA's pair needs it.
 *   block_mask: device uint8 [nt, nt], row-major, shared by every (batch,
 *     head) slice; no alignment requirement.
 *   Rows that are left no visible key get O = 0 and LSE = -inf, dQ = 0, and
 *     add nothing to dK and dV; keys no query sees get dK = dV = 0.
 *   fa_bwd_blocksparse: workspace as fa_bwd (fa_bwd_workspace_size); the
 *     mask must be the one the forward used; runs the three backward stages
 *     on `stream`.
 */
int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                       const uint8_t* block_mask, int B, int H, int N, int d, float scale,
                       int causal, const int32_t* seqlens, int dtype, void* stream);
int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       void* workspace, size_t workspace_bytes, const uint8_t* block_mask,
                       int B, int H, int N, int d, float scale, int causal,
                       const int32_t* seqlens, int dtype, void* stream);

/*
 * Backward pass that allocates nothing and takes no workspace.  The pages
 * have no counterpart: it exists for callers that cannot allocate device
 * memory for a workspace, such as plugin hosts that hand an operator only its
 * input and output buffers, or latency-critical paths that must not call
 * cudaMalloc (which may synchronise the device).
 *   Same arguments, results and checks as fa_bwd, minus the workspace.  The
 *   workspace is a static device array of fa_bwd_noalloc_max_bytes()
 *   (32 MiB) bytes inside the library, which every GPU that loads the
 *   library holds until the process exits.  Problems with
 *   fa_bwd_workspace_size(B, H, N, d) above that return FA_ERR_SCRATCH_LIMIT
 *   before anything is launched (for d = 128 that is about 64K rows B*H*N).
 *   All calls share the array: calls whose kernels overlap on the GPU (other
 *   streams, other host threads) race and give wrong results; serialise them.
 *   The array keeps the last call's contents; the preprocess stage rewrites
 *   everything the call reads, so no clearing is needed between calls.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any
 *   stream capture.  The address belongs to the device's primary context:
 *   after cudaDeviceReset() (or anything else that destroys that context)
 *   the looked-up address is stale, so do not call fa_bwd_noalloc again on
 *   that device in the same process.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, float scale, int causal,
                   const int32_t* seqlens, int dtype, void* stream);

/* Size in bytes of the static workspace fa_bwd_noalloc uses. */
size_t fa_bwd_noalloc_max_bytes(void);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device: FA_OK, FA_ERR_DEVICE_SEQLEN, FA_ERR_DEVICE_TIMEOUT,
 * FA_ERR_DEVICE_LAYOUT or FA_ERR_DEVICE_SCALE
 * (FA_ERR_CUDA if the synchronisation itself failed).  *detail, if not NULL,
 * receives the raw word (code | site << 8 | block << 16).
 */
int fa_device_status(void* stream, uint32_t* detail);

/*
 * Bound, in nanoseconds, of every pipeline wait inside the kernels launched
 * after this call, from any host thread (default 2e9 = 2 s; 0 restores the
 * default).  Returns the previous bound.
 *   Every wait of a kernel's producer/consumer pipeline (a warp waiting for
 *   a tile load, a tensor-core result or another warp's data) gives up after
 *   this long: it records FA_ERR_DEVICE_TIMEOUT, with the site of the wait,
 *   in the device status word, the CTA's other roles stop at their next
 *   wait, copies and tensor-core work already in flight are waited for, and
 *   the kernel returns, so the device stays usable; that call's outputs are
 *   unspecified.  In a correct pipeline no wait lasts more than microseconds,
 *   so the default only fires on a hang.  A bound far below a kernel's
 *   ordinary waits (say 1 ns) makes ordinary waits give up: that is how the
 *   timeout path is exercised without a fault.
 */
unsigned long long fa_set_wait_limit_ns(unsigned long long ns);

/* Static description of a status code.  Never NULL. */
const char* fa_status_string(int status);

/* Library ABI version: 100 * major + minor. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
