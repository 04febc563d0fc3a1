// Row-wise LayerNorm kernels (one warp per row, fp32 statistics).
//
// LayerNorm over the feature axis of a token: mean, biased variance of the
// deviations (two passes over registers), eps = 1e-5 inside the square root,
// then gamma * (x - mean) / sqrt(var + eps) + beta.
//
// One template serves every case: input rows are read through a row map
// (scratch rows with no residual row get zeros) and written densely.
//   bf16 x rows            -> fp16 rows    (LN1, tensor-core path)
//   fp32 residual rows y   -> fp16 rows    (LN2, tensor-core path)
//   fp32 rows              -> fp32 rows    (LN1 / LN2, fp32 path)
// An fp16 output beyond the fp16 range (or NaN) is reported in the device
// error word.
#pragma once

#include "common.cuh"

namespace bpt {

constexpr float kLnEps = 1e-5f;
constexpr int kLnWarps = 8;

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Loads 8 consecutive elements as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = __bfloat162float(h[k]);
}
__device__ __forceinline__ void load8(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* v) {
  uint4 w;
  w.x = pack_bf16x2(v[0], v[1]);
  w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]);
  w.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = w;
}
__device__ __forceinline__ void load8(const __half* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half* h = reinterpret_cast<const __half*>(&u);
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = __half2float(h[k]);
}
__device__ __forceinline__ void store8(__half* p, const float* v, bool& bad) {
  uint4 w;
  w.x = pack_f16x2(v[0], v[1], bad);
  w.y = pack_f16x2(v[2], v[3], bad);
  w.z = pack_f16x2(v[4], v[5], bad);
  w.w = pack_f16x2(v[6], v[7], bad);
  *reinterpret_cast<uint4*>(p) = w;
}
__device__ __forceinline__ void store8(float* p, const float* v, bool&) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// NV = 8-element chunks per lane (d <= 256 * NV, d % 8 == 0).
// gamma = ln[0..d), beta = ln[d..2d).
template <int NV, typename TIn, typename TOut, typename TP>
__global__ void __launch_bounds__(kLnWarps * 32)
    ln_rows_kernel(const TIn* __restrict__ in, const TP* __restrict__ ln, TOut* __restrict__ out,
                   long long rows, int d, RowMap in_map, uint32_t* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long s = static_cast<long long>(blockIdx.x) * kLnWarps + warp;
  if (s >= rows) return;
  const long long g = in_map.map(s);
  TOut* orow = out + s * d;
  bool bad = false;
  if (g < 0) {
    float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int c = (lane + 32 * q) * 8;
      if (c < d) store8(orow + c, z, bad);
    }
    return;
  }
  const TIn* irow = in + g * d;
  float v[NV][8];
  float sum = 0.f;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c = (lane + 32 * q) * 8;
    if (c < d) {
      load8(irow + c, v[q]);
#pragma unroll
      for (int k = 0; k < 8; ++k) sum += v[q][k];
    }
  }
  const float mean = warp_sum(sum) / static_cast<float>(d);
  float sq = 0.f;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c = (lane + 32 * q) * 8;
    if (c < d) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float t = v[q][k] - mean;
        sq += t * t;
      }
    }
  }
  const float var = warp_sum(sq) / static_cast<float>(d);
  const float rstd = 1.0f / sqrtf(var + kLnEps);
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c = (lane + 32 * q) * 8;
    if (c < d) {
      float gm[8], bt[8], o[8];
      load8(ln + c, gm);
      load8(ln + d + c, bt);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = (v[q][k] - mean) * rstd * gm[k] + bt[k];
      store8(orow + c, o, bad);
    }
  }
  if (bad) record_error(err, kErrRange, kSiteRangeLN);
}

// bf16 -> fp16 copies of the weight matrices, eight elements per thread and
// step (each segment's length is a multiple of 8).  Values within the fp16
// normal range convert exactly; magnitudes below 2^-14 become fp16 subnormals
// (absolute error <= 2^-25); anything beyond the fp16 range is reported.
struct CvtSegments {
  const __nv_bfloat16* src[6];
  __half* dst[6];
  long long n8_end[6];  // cumulative count of 8-element groups
  int count;
};

__global__ void __launch_bounds__(256) cvt_bf16_to_f16_kernel(const CvtSegments seg,
                                                             uint32_t* err) {
  const long long total = seg.n8_end[seg.count - 1];
  bool bad = false;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    int k = 0;
    while (i >= seg.n8_end[k]) ++k;
    const long long j = i - (k ? seg.n8_end[k - 1] : 0);
    float v[8];
    load8(seg.src[k] + 8 * j, v);
    store8(seg.dst[k] + 8 * j, v, bad);
  }
  if (bad) record_error(err, kErrRange, kSiteRangeWeights);
}

}  // namespace bpt
