// C ABI of the library: argument checks, TMA descriptors, launches.
//
// Every check here runs on the host before anything is enqueued, so a bad
// call returns a status and leaves the device untouched.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool probed = false;
  bool is_sm100 = false;
  int num_sms = 0;
};

DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode = nullptr;

// Bound of every pipeline wait of the kernels launched from now on
// (fa_set_wait_limit_ns).
std::atomic<unsigned long long> g_wait_ns{kWaitTimeoutNs};

int current_device_info(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& di = g_devices[dev];
  if (!di.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    di.is_sm100 = (major == 10 && minor == 0);
    di.num_sms = sms;
    di.probed = true;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return FA_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *out = di;
  return di.is_sm100 ? FA_OK : FA_ERR_ARCH;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int H, int N, int d, float scale, int dtype) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long elems = static_cast<long long>(B) * H * N * d;
  if (elems >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// [B*H, N, d] view of a [B, H, N, d] 16-bit tensor; box = 64 columns x 128 rows,
// 128-byte swizzle (the layout the tcgen05 descriptors expect).  Rows past N
// inside a head read as zero.
int make_map(CUtensorMap* map, const void* ptr, int BH, int N, int d, int dtype) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      g_encode(map, dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
               3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// [B*H, N, d] e4m3 view: box = 128 columns (128 bytes) x 128 rows, 128-byte
// swizzle; in bytes the same tiles as the 16-bit d = 64 layout.  For d = 64
// the box runs past the row: the load fills columns 64..127 with zeros, so
// the d = 128 kernel computes the same S and an O whose last 64 columns are 0.
int make_map_e4m3(CUtensorMap* map, const void* ptr, int BH, int N, int d) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N) * d};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// [B*H, N, d] fp32 view of the dQ accumulator for TMA reduce-adds of 128 rows
// x 32 columns; rows past N inside a head are skipped.
int make_map_acc(CUtensorMap* map, void* ptr, int BH, int N, int d) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(N) * d * 4};
  // box: 32 columns (128 bytes) x 128 rows, read from a 128-byte-swizzled
  // shared tile
  const cuuint32_t box[3] = {32, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace
}  // namespace fa

using namespace fa;

namespace fa {
namespace {

// Forward for both layouts (cu_seqlens == nullptr: [B, H, N, d]; else packed
// [H, T = N, d]); arguments already checked except the pointers' alignment.
int fwd_core(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int N, int d, float scale, int causal, const int32_t* seqlens,
             const int32_t* cu_seqlens, int max_seqlen, int dtype, void* stream,
             const uint8_t* block_mask = nullptr, uint32_t keep_t = 256u, float inv_keep = 1.f,
             uint64_t seed = 0, uint32_t drop_offset = 0, const float* q_descale = nullptr,
             const float* k_descale = nullptr, const float* v_descale = nullptr) {
  const bool e4m3 = q_descale != nullptr;  // q, k, v are e4m3 codes; dtype is O's type
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) ||
      (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)))
    return FA_ERR_ALIGNMENT;
  DeviceInfo di;
  const int st = current_device_info(&di);
  if (st != FA_OK) return st;

  CUtensorMap tq, tk, tv;
  const int blocks = cu_seqlens ? H : B * H;  // row blocks of N rows
  if (e4m3) {
    if (make_map_e4m3(&tq, q, blocks, N, d) != FA_OK ||
        make_map_e4m3(&tk, k, blocks, N, d) != FA_OK ||
        make_map_e4m3(&tv, v, blocks, N, d) != FA_OK)
      return FA_ERR_CUDA;
  } else if (make_map(&tq, q, blocks, N, d, dtype) != FA_OK ||
             make_map(&tk, k, blocks, N, d, dtype) != FA_OK ||
             make_map(&tv, v, blocks, N, d, dtype) != FA_OK) {
    return FA_ERR_CUDA;
  }

  FwdParams p;
  p.o = o;
  p.lse = lse;
  p.seqlens = seqlens;
  p.cu_seqlens = cu_seqlens;
  p.max_seqlen = cu_seqlens ? max_seqlen : N;
  p.block_mask = block_mask;
  p.keep_t = keep_t;
  p.inv_keep = inv_keep;
  p.seed_lo = static_cast<uint32_t>(seed);
  p.seed_hi = static_cast<uint32_t>(seed >> 32);
  p.drop_offset = drop_offset;
  p.q_descale = q_descale;
  p.k_descale = k_descale;
  p.v_descale = v_descale;
  p.B = B;
  p.H = H;
  p.N = N;
  p.o_cols = d;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.n_qtiles = (p.max_seqlen + kBlockM - 1) / kBlockM;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.n_units = B * H * ((p.n_pairs + 1) / 2);
  p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  const cudaError_t e =
      e4m3 ? launch_fwd_e4m3(dtype == FA_BF16, tq, tk, tv, p, di.num_sms,
                             static_cast<cudaStream_t>(stream))
           : launch_fwd(d, dtype == FA_BF16, tq, tk, tv, p, di.num_sms,
                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Dropout rate -> 8-bit keep threshold t = round(256 (1 - p)) (ties to even),
// clamped to [1, 256], and the scale 256 / t of the kept scores.
int dropout_threshold(float p_drop, uint32_t* keep_t, float* inv_keep) {
  if (!(p_drop >= 0.f && p_drop < 1.f)) return FA_ERR_INVALID_ARG;
  double t = std::nearbyint(256.0 * (1.0 - static_cast<double>(p_drop)));
  t = t < 1.0 ? 1.0 : (t > 256.0 ? 256.0 : t);
  *keep_t = static_cast<uint32_t>(t);
  *inv_keep = static_cast<float>(256.0 / t);
  return FA_OK;
}

// Packed-layout argument checks shared by the forward and the backward: the
// [H, T, d] tensors as in check_common (B = 1, N = T), B >= 1 sequences, and
// the work-unit count B * H * ceil(max_seqlen / 128) within int range.
int check_varlen(const int32_t* cu_seqlens, int B, int H, int T, int max_seqlen, int d,
                 float scale, int dtype) {
  if (!cu_seqlens || B < 1 || max_seqlen < 1) return FA_ERR_INVALID_ARG;
  const int st = check_common(1, H, T, d, scale, dtype);
  if (st != FA_OK) return st;
  const long long tiles = (static_cast<long long>(max_seqlen < T ? max_seqlen : T) + 127) / 128;
  if (static_cast<long long>(B) * H * tiles >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int N, int d, float scale, int causal, const int32_t* seqlens,
                      int dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  const int st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  return fwd_core(q, k, v, o, lse, B, H, N, d, scale, causal, seqlens, nullptr, 0, dtype, stream);
}

extern "C" int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o,
                                  float* lse, const uint8_t* block_mask, int B, int H, int N,
                                  int d, float scale, int causal, const int32_t* seqlens,
                                  int dtype, void* stream) {
  if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID_ARG;
  const int st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  return fwd_core(q, k, v, o, lse, B, H, N, d, scale, causal, seqlens, nullptr, 0, dtype, stream,
                  block_mask);
}

extern "C" int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int H, int N, int d, float scale, int causal,
                              const int32_t* seqlens, float p_drop, uint64_t seed,
                              uint32_t offset, int dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  uint32_t keep_t;
  float inv_keep;
  st = dropout_threshold(p_drop, &keep_t, &inv_keep);
  if (st != FA_OK) return st;
  return fwd_core(q, k, v, o, lse, B, H, N, d, scale, causal, seqlens, nullptr, 0, dtype, stream,
                  nullptr, keep_t, inv_keep, seed, offset);
}

extern "C" int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                             const int32_t* cu_seqlens, int B, int H, int T, int max_seqlen,
                             int d, float scale, int causal, int dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  const int st = check_varlen(cu_seqlens, B, H, T, max_seqlen, d, scale, dtype);
  if (st != FA_OK) return st;
  return fwd_core(q, k, v, o, lse, B, H, T, d, scale, causal, nullptr, cu_seqlens,
                  max_seqlen < T ? max_seqlen : T, dtype, stream);
}

extern "C" int fa_fwd_e4m3(const void* q8, const void* k8, const void* v8, const float* q_descale,
                           const float* k_descale, const float* v_descale, void* o, float* lse,
                           int B, int H, int N, int d, float scale, int causal,
                           const int32_t* seqlens, int out_dtype, void* stream) {
  if (!q8 || !k8 || !v8 || !q_descale || !k_descale || !v_descale || !o || !lse)
    return FA_ERR_INVALID_ARG;
  const int st = check_common(B, H, N, d, scale, out_dtype);
  if (st != FA_OK) return st;
  const uintptr_t ds_bits = reinterpret_cast<uintptr_t>(q_descale) |
                            reinterpret_cast<uintptr_t>(k_descale) |
                            reinterpret_cast<uintptr_t>(v_descale);
  if (ds_bits & 3u) return FA_ERR_ALIGNMENT;
  return fwd_core(q8, k8, v8, o, lse, B, H, N, d, scale, causal, seqlens, nullptr, 0, out_dtype,
                  stream, nullptr, 256u, 1.f, 0, 0, q_descale, k_descale, v_descale);
}

extern "C" int fa_quantize_e4m3(const void* x, void* x8, float* descale, int B, int H, int N,
                                int d, int dtype, void* stream) {
  if (!x || !x8 || !descale) return FA_ERR_INVALID_ARG;
  const int st = check_common(B, H, N, d, 1.f, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(x) || !aligned16(x8) || (reinterpret_cast<uintptr_t>(descale) & 3u))
    return FA_ERR_ALIGNMENT;
  DeviceInfo di;
  const int dst = current_device_info(&di);
  if (dst != FA_OK) return dst;
  const cudaError_t e =
      launch_quantize_e4m3(d, dtype == FA_BF16, x, x8, descale, static_cast<long long>(B) * H, N,
                           di.num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.f, FA_BF16) != FA_OK) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  return round256(rows * sizeof(float)) + round256(rows * d * sizeof(float));
}

extern "C" size_t fa_bwd_varlen_workspace_size(int B, int H, int T, int d) {
  if (B < 1) return 0;
  const size_t base = fa_bwd_workspace_size(1, H, T, d);
  if (base == 0) return 0;
  // the longest-first order table: 3 B + 1 ints (batches of up to
  // kBwdRankMaxSeqs sequences; larger ones run in head-major order)
  const size_t table = B <= kBwdRankMaxSeqs ? round256((3ull * B + 1) * sizeof(int)) : 0;
  return base + table;
}

namespace fa {
namespace {

// Checks shared by the backward stages; fills the workspace carving.  With
// cu_seqlens the tensors are packed [H, T = N, d] (max_seqlen already clamped
// to T) and the workspace is that of fa_bwd_workspace_size(1, H, T, d).
int bwd_common(void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale,
               int dtype, const int32_t* seqlens, BwdParams* p, DeviceInfo* di,
               const int32_t* cu_seqlens = nullptr, int max_seqlen = 0) {
  int st = cu_seqlens ? check_varlen(cu_seqlens, B, H, N, max_seqlen, d, scale, dtype)
                      : check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  if ((seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) ||
      (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)))
    return FA_ERR_ALIGNMENT;
  const size_t need = cu_seqlens ? fa_bwd_varlen_workspace_size(B, H, N, d)
                                 : fa_bwd_workspace_size(B, H, N, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_ALIGNMENT;
  st = current_device_info(di);
  if (st != FA_OK) return st;
  const size_t rows = static_cast<size_t>(cu_seqlens ? 1 : B) * H * N;
  std::memset(p, 0, sizeof(*p));
  p->keep_t = 256u;  // no dropout unless a dropout entry point sets it
  p->inv_keep = 1.f;
  p->dsum = static_cast<float*>(workspace);
  p->dq_acc =
      reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round256(rows * sizeof(float)));
  // packed batches: the longest-first table after the accumulator
  p->rank = (cu_seqlens && B <= kBwdRankMaxSeqs)
                ? reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) +
                                         round256(rows * sizeof(float)) +
                                         round256(rows * d * sizeof(float)))
                : nullptr;
  p->seqlens = seqlens;
  p->cu_seqlens = cu_seqlens;
  p->max_seqlen = cu_seqlens ? max_seqlen : N;
  p->B = B;
  p->H = H;
  p->N = N;
  p->scale = scale;
  p->scale_log2 = scale * 1.4426950408889634f;
  p->n_ktiles = (p->max_seqlen + kBlockN - 1) / kBlockN;
  p->n_units = B * H * ((p->n_ktiles + 1) / 2);
  p->wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" int fa_bwd_preprocess(const void* o, const void* dout, void* workspace,
                                 size_t workspace_bytes, int B, int H, int N, int d, int dtype,
                                 void* stream) {
  if (!o || !dout) return FA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(dout)) return FA_ERR_ALIGNMENT;
  BwdParams p;
  DeviceInfo di;
  int st = bwd_common(workspace, workspace_bytes, B, H, N, d, 1.f, dtype, nullptr, &p, &di);
  if (st != FA_OK) return st;
  p.o = o;
  p.dout = dout;
  const cudaError_t e = launch_bwd_pre(d, dtype == FA_BF16, p, di.num_sms,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" int fa_bwd_main(const void* q, const void* k, const void* v, const void* dout,
                           const float* lse, void* dk, void* dv, void* workspace,
                           size_t workspace_bytes, int B, int H, int N, int d, float scale,
                           int causal, const int32_t* seqlens, int dtype, void* stream) {
  if (!q || !k || !v || !dout || !lse || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dk) || !aligned16(dv))
    return FA_ERR_ALIGNMENT;
  BwdParams p;
  DeviceInfo di;
  int st = bwd_common(workspace, workspace_bytes, B, H, N, d, scale, dtype, seqlens, &p, &di);
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv, tdo, tdq;
  const int BH = B * H;
  if (make_map(&tq, q, BH, N, d, dtype) != FA_OK || make_map(&tk, k, BH, N, d, dtype) != FA_OK ||
      make_map(&tv, v, BH, N, d, dtype) != FA_OK || make_map(&tdo, dout, BH, N, d, dtype) != FA_OK ||
      make_map_acc(&tdq, p.dq_acc, BH, N, d) != FA_OK)
    return FA_ERR_CUDA;
  p.q = q;
  p.k = k;
  p.v = v;
  p.dout = dout;
  p.lse = lse;
  p.dk = dk;
  p.dv = dv;
  p.causal = causal ? 1 : 0;
  const cudaError_t e = launch_bwd_main(d, dtype == FA_BF16, tq, tk, tv, tdo, tdq, p, di.num_sms,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" int fa_bwd_postprocess(void* workspace, size_t workspace_bytes, void* dq, int B, int H,
                                  int N, int d, float scale, int dtype, void* stream) {
  if (!dq) return FA_ERR_INVALID_ARG;
  if (!aligned16(dq)) return FA_ERR_ALIGNMENT;
  BwdParams p;
  DeviceInfo di;
  int st = bwd_common(workspace, workspace_bytes, B, H, N, d, scale, dtype, nullptr, &p, &di);
  if (st != FA_OK) return st;
  p.dq = dq;
  const cudaError_t e = launch_bwd_post(d, dtype == FA_BF16, p, di.num_sms,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv, void* workspace,
                      size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                      const int32_t* seqlens, int dtype, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  // validate everything before the first launch, so a rejected call enqueues nothing
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_ALIGNMENT;
  {
    BwdParams p;
    DeviceInfo di;
    const int st = bwd_common(workspace, workspace_bytes, B, H, N, d, scale, dtype, seqlens, &p, &di);
    if (st != FA_OK) return st;
  }
  int st = fa_bwd_preprocess(o, dout, workspace, workspace_bytes, B, H, N, d, dtype, stream);
  if (st != FA_OK) return st;
  st = fa_bwd_main(q, k, v, dout, lse, dk, dv, workspace, workspace_bytes, B, H, N, d, scale,
                   causal, seqlens, dtype, stream);
  if (st != FA_OK) return st;
  return fa_bwd_postprocess(workspace, workspace_bytes, dq, B, H, N, d, scale, dtype, stream);
}

namespace fa {
namespace {

// The three backward stages in one call for a variant (block mask, dropout,
// packed layout): p has passed bwd_common and carries the variant's fields;
// blocks x rows is the TMA view of the tensors (B*H x N, or H x T packed).
int bwd_variant_run(BwdParams& p, const DeviceInfo& di, const void* q, const void* k,
                    const void* v, const void* o, const void* dout, const float* lse, void* dq,
                    void* dk, void* dv, int blocks, int rows, int d, int causal, int dtype,
                    void* stream) {
  CUtensorMap tq, tk, tv, tdo, tdq;
  if (make_map(&tq, q, blocks, rows, d, dtype) != FA_OK ||
      make_map(&tk, k, blocks, rows, d, dtype) != FA_OK ||
      make_map(&tv, v, blocks, rows, d, dtype) != FA_OK ||
      make_map(&tdo, dout, blocks, rows, d, dtype) != FA_OK ||
      make_map_acc(&tdq, p.dq_acc, blocks, rows, d) != FA_OK)
    return FA_ERR_CUDA;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.causal = causal ? 1 : 0;
  const bool bf16 = dtype == FA_BF16;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_bwd_pre(d, bf16, p, di.num_sms, s) != cudaSuccess) return FA_ERR_CUDA;
  if (p.rank != nullptr && launch_bwd_rank(p, s) != cudaSuccess) return FA_ERR_CUDA;
  if (launch_bwd_main(d, bf16, tq, tk, tv, tdo, tdq, p, di.num_sms, s) != cudaSuccess)
    return FA_ERR_CUDA;
  return launch_bwd_post(d, bf16, p, di.num_sms, s) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

bool bwd_pointers_ok(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, const void* dq, const void* dk, const void* dv) {
  return q && k && v && o && dout && lse && dq && dk && dv;
}

bool bwd_pointers_aligned(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, const void* dq, const void* dk,
                          const void* dv) {
  return aligned16(q) && aligned16(k) && aligned16(v) && aligned16(o) && aligned16(dout) &&
         aligned16(lse) && aligned16(dq) && aligned16(dk) && aligned16(dv);
}

}  // namespace
}  // namespace fa

extern "C" int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o,
                                  const void* dout, const float* lse, void* dq, void* dk,
                                  void* dv, void* workspace, size_t workspace_bytes,
                                  const uint8_t* block_mask, int B, int H, int N, int d,
                                  float scale, int causal, const int32_t* seqlens, int dtype,
                                  void* stream) {
  if (!bwd_pointers_ok(q, k, v, o, dout, lse, dq, dk, dv) || !block_mask)
    return FA_ERR_INVALID_ARG;
  if (!bwd_pointers_aligned(q, k, v, o, dout, lse, dq, dk, dv)) return FA_ERR_ALIGNMENT;
  BwdParams p;
  DeviceInfo di;
  const int st = bwd_common(workspace, workspace_bytes, B, H, N, d, scale, dtype, seqlens, &p, &di);
  if (st != FA_OK) return st;
  p.block_mask = block_mask;
  return bwd_variant_run(p, di, q, k, v, o, dout, lse, dq, dk, dv, B * H, N, d, causal, dtype,
                         stream);
}

extern "C" int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                              float scale, int causal, const int32_t* seqlens, float p_drop,
                              uint64_t seed, uint32_t offset, int dtype, void* stream) {
  if (!bwd_pointers_ok(q, k, v, o, dout, lse, dq, dk, dv)) return FA_ERR_INVALID_ARG;
  if (!bwd_pointers_aligned(q, k, v, o, dout, lse, dq, dk, dv)) return FA_ERR_ALIGNMENT;
  uint32_t keep_t;
  float inv_keep;
  int st = dropout_threshold(p_drop, &keep_t, &inv_keep);
  if (st != FA_OK) return st;
  BwdParams p;
  DeviceInfo di;
  st = bwd_common(workspace, workspace_bytes, B, H, N, d, scale, dtype, seqlens, &p, &di);
  if (st != FA_OK) return st;
  p.keep_t = keep_t;
  p.inv_keep = inv_keep;
  p.seed_lo = static_cast<uint32_t>(seed);
  p.seed_hi = static_cast<uint32_t>(seed >> 32);
  p.drop_offset = offset;
  return bwd_variant_run(p, di, q, k, v, o, dout, lse, dq, dk, dv, B * H, N, d, causal, dtype,
                         stream);
}

extern "C" int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, void* dq, void* dk, void* dv,
                             void* workspace, size_t workspace_bytes, const int32_t* cu_seqlens,
                             int B, int H, int T, int max_seqlen, int d, float scale, int causal,
                             int dtype, void* stream) {
  if (!bwd_pointers_ok(q, k, v, o, dout, lse, dq, dk, dv)) return FA_ERR_INVALID_ARG;
  if (!bwd_pointers_aligned(q, k, v, o, dout, lse, dq, dk, dv)) return FA_ERR_ALIGNMENT;
  BwdParams p;
  DeviceInfo di;
  const int st = bwd_common(workspace, workspace_bytes, B, H, T, d, scale, dtype, nullptr, &p,
                            &di, cu_seqlens, max_seqlen < T ? max_seqlen : T);
  if (st != FA_OK) return st;
  return bwd_variant_run(p, di, q, k, v, o, dout, lse, dq, dk, dv, H, T, d, causal, dtype, stream);
}

// ---------------------------------------------------------------------------
// Backward pass without any allocation: the workspace is a static device
// array of the library.
//
// Some callers cannot hand the library a workspace: plugin hosts that give an
// operator only its input and output buffers and own every other byte of
// device memory, and latency-critical paths that must not call cudaMalloc
// (which may synchronise the device).  fa_bwd_noalloc serves them with a
// fixed scratch array that every GPU loading the library holds until the
// process exits.
// ---------------------------------------------------------------------------
namespace fa {
namespace {

constexpr size_t kStaticScratchBytes = 32ull << 20;  // 32 MiB per device
static __device__ __align__(256) uint8_t g_bwd_scratch[kStaticScratchBytes];

void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_bwd_scratch on the current device (host code cannot use
// the symbol itself: on the host it names a stand-in, not device memory).
// Looked up once per device, with that device current.
int static_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || ptr == nullptr)
      return FA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" size_t fa_bwd_noalloc_max_bytes(void) { return kStaticScratchBytes; }

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int B, int H, int N, int d, float scale, int causal,
                              const int32_t* seqlens, int dtype, void* stream) {
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == 0) {
    const int st = check_common(B, H, N, d, scale, dtype);
    return st != FA_OK ? st : FA_ERR_INVALID_ARG;
  }
  if (need > kStaticScratchBytes) return FA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const int st = static_scratch(&scratch);
  if (st != FA_OK) return st;
  // fa_bwd's preprocess rewrites the row dots and zeroes the dQ accumulator,
  // so whatever an earlier call left in the array does not matter.
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, scratch, kStaticScratchBytes, B, H, N, d,
                scale, causal, seqlens, dtype, stream);
}

extern "C" unsigned long long fa_set_wait_limit_ns(unsigned long long ns) {
  return g_wait_ns.exchange(ns == 0 ? kWaitTimeoutNs : ns);
}

extern "C" int fa_device_status(void* stream, uint32_t* detail) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int word = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return FA_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (detail) *detail = word;
  const unsigned code = word & 0xffu;
  if (code == kErrDeviceTimeout) return FA_ERR_DEVICE_TIMEOUT;
  if (code == kErrDeviceSeqlen) return FA_ERR_DEVICE_SEQLEN;
  if (code == kErrDeviceLayout) return FA_ERR_DEVICE_LAYOUT;
  if (code == kErrDeviceScale) return FA_ERR_DEVICE_SCALE;
  return word == 0 ? FA_OK : FA_ERR_CUDA;
}

extern "C" const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported shape (d must be 64 or 128; B*H*N*d < 2^31)";
    case FA_ERR_ALIGNMENT: return "pointer not aligned (16 bytes; workspace 256 bytes)";
    case FA_ERR_ARCH: return "current device is not sm_100 (B200)";
    case FA_ERR_CUDA: return "CUDA call or launch failed";
    case FA_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
    case FA_ERR_DEVICE_SEQLEN: return "seqlens value outside [1, N] (clamped on device)";
    case FA_ERR_WORKSPACE: return "backward workspace missing or too small";
    case FA_ERR_DEVICE_LAYOUT: return "kernel refused: shared-memory window misaligned";
    case FA_ERR_SCRATCH_LIMIT:
      return "problem needs more backward scratch than fa_bwd_noalloc's static array holds";
    case FA_ERR_DEVICE_SCALE: return "e4m3 descale factor not finite and positive, or infinite or NaN input";
    default: return "unknown status";
  }
}

extern "C" int fa_version(void) { return 100; }


#ifdef FA_TRACE
// Trace builds only: copy the device timeline (see FA_TRACE_AT) to the host.
extern "C" int fa_trace_read(unsigned long long* host, int n) {
  if (n > kTraceSlots) n = kTraceSlots;
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(host, g_trace, n * sizeof(unsigned long long)) != cudaSuccess)
    return FA_ERR_CUDA;
  static unsigned long long zeros[kTraceSlots];
  return cudaMemcpyToSymbol(g_trace, zeros, sizeof(zeros)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
#endif
