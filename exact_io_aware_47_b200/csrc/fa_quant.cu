// Per-tile e4m3 quantisation of a 16-bit [slices, n_rows, d] tensor, the
// producer of the 8-bit forward's inputs.
//
// For every 128-row tile of a slice (the last one may be ragged): amax = the
// largest magnitude in the tile, descale = amax / 448 and inv = 448 / amax,
// both fp32 divisions rounded to nearest; every element becomes
// e4m3(x * inv) (fp32 product, then round to nearest even, saturating).  A
// tile of zeros gets descale 1 and zero codes; a tile holding an infinite or
// NaN value is reported as FA_ERR_DEVICE_SCALE.  The format and the 448 bound
// are those of e4m3 in the OCP 8-bit floating-point specification; the pages
// ("How Flash Attention Works", section "FlashAttention 2 and 3") only name
// lower-precision paths.
//
// HBM-bound: 2 bytes read and 1 written per element.  One 256-thread CTA per
// tile, persistent over tiles; each thread keeps its d / 16 16-byte vectors of
// the tile in registers between the amax pass and the conversion, so the tile
// is read from HBM once.
#include <cuda_fp16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

constexpr int kQuantThreads = 256;

// max that propagates NaN (the library max drops it), so that a NaN input
// makes the tile's amax NaN and is reported like an infinite one
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ float abs_max8(const uint4& v, bool bf16, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float lo, hi;
    if (bf16) {
      lo = __uint_as_float(w[i] << 16);
      hi = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      lo = __low2float(h);
      hi = __high2float(h);
    }
    m = max_nan(m, max_nan(fabsf(lo), fabsf(hi)));
  }
  return m;
}

__device__ __forceinline__ uint2 to_e4m3x8(const uint4& v, bool bf16, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (bf16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      f[2 * i] = __low2float(h);
      f[2 * i + 1] = __high2float(h);
    }
  }
  uint2 r;
  r.x = pack_e4m3x4(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv), __fmul_rn(f[2], inv),
                    __fmul_rn(f[3], inv));
  r.y = pack_e4m3x4(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv), __fmul_rn(f[6], inv),
                    __fmul_rn(f[7], inv));
  return r;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kQuantThreads)
    fa_quantize_e4m3_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ x8,
                            float* __restrict__ descale, long long slices, int n_rows) {
  constexpr int kVecPerRow = D * 2 / 16;                       // 16-byte vectors per row
  constexpr int kVecPerThread = kBlockM * kVecPerRow / kQuantThreads;
  __shared__ float warp_max[kQuantThreads / 32];
  const int tiles_per_slice = (n_rows + kBlockM - 1) / kBlockM;
  const long long n_tiles = slices * tiles_per_slice;
  for (long long tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const long long s = tile / tiles_per_slice;
    const int t = static_cast<int>(tile - s * tiles_per_slice);
    const int rows = min(kBlockM, n_rows - t * kBlockM);
    const long long row0 = s * n_rows + static_cast<long long>(t) * kBlockM;
    const uint4* src = reinterpret_cast<const uint4*>(x + row0 * D * 2);
    uint2* dst = reinterpret_cast<uint2*>(x8 + row0 * D);
    uint4 v[kVecPerThread];
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < kVecPerThread; ++k) {
      const int idx = threadIdx.x + k * kQuantThreads;        // vector index inside the tile
      if (idx / kVecPerRow < rows) {
        v[k] = __ldcs(src + idx);                               // read once: streaming
        m = abs_max8(v[k], BF16, m);
      } else {
        v[k] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    float amax = warp_max[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) amax = max_nan(amax, warp_max[i]);
    __syncthreads();  // warp_max is rewritten by the next tile
    float inv = 0.f, ds = 1.f;
    if (amax > 0.f) {
      inv = __fdiv_rn(448.f, amax);
      ds = __fdiv_rn(amax, 448.f);
    }
    if (!(amax < INFINITY)) record_error(kErrDeviceScale, 2);   // an infinite or NaN input
    if (threadIdx.x == 0) descale[tile] = ds;
#pragma unroll
    for (int k = 0; k < kVecPerThread; ++k) {
      const int idx = threadIdx.x + k * kQuantThreads;
      if (idx / kVecPerRow < rows) __stcs(dst + idx, to_e4m3x8(v[k], BF16, inv));
    }
  }
}

cudaError_t launch_quantize_e4m3(int d, bool bf16, const void* x, void* x8, float* descale,
                                 long long slices, int n_rows, int num_sms, cudaStream_t stream) {
  const long long tiles = slices * ((n_rows + kBlockM - 1) / kBlockM);
  const long long cap = static_cast<long long>(num_sms) * (2048 / kQuantThreads);  // resident CTAs
  const int grid = static_cast<int>(tiles < cap ? tiles : cap);
  const uint8_t* xs = static_cast<const uint8_t*>(x);
  uint8_t* xd = static_cast<uint8_t*>(x8);
  if (d == 128) {
    if (bf16) fa_quantize_e4m3_kernel<128, true><<<grid, kQuantThreads, 0, stream>>>(xs, xd, descale, slices, n_rows);
    else fa_quantize_e4m3_kernel<128, false><<<grid, kQuantThreads, 0, stream>>>(xs, xd, descale, slices, n_rows);
  } else {
    if (bf16) fa_quantize_e4m3_kernel<64, true><<<grid, kQuantThreads, 0, stream>>>(xs, xd, descale, slices, n_rows);
    else fa_quantize_e4m3_kernel<64, false><<<grid, kQuantThreads, 0, stream>>>(xs, xd, descale, slices, n_rows);
  }
  return cudaGetLastError();
}

}  // namespace fa
