// Backward pass of the BPT layer: the kernels that are not GEMMs.
//
// "Blockwise Parallel Transformer — BPT", section "The backward pass": the
// forward keeps the layer input, the layer output and the per-row softmax
// statistics (m, l); the backward recomputes each block's scores, attention
// output and FFN hidden from them and accumulates the gradients.  The GEMMs
// of the backward run on the pair GEMM (gemm_tc.cuh); this file holds
//   * row copies fp32 -> fp16 (GEMM operands),
//   * LayerNorm backward (one warp per row) and the deterministic column
//     sums of the bias, gamma and beta gradients,
//   * the attention backward's per-row terms (D = rowsum(dO * O) per head,
//     with the row's softmax statistics; the attention gradients themselves
//     run on the tensor cores, attn_bwd_tc.cuh).
// LayerNorm y = g * xh + b (standard calculus):
//   dx = rstd * (dxh - mean(dxh) - xh * mean(dxh * xh)),
//   dxh = dy * g,  dg = sum_rows dy * xh,  db = sum_rows dy.
#pragma once

#include "common.cuh"

namespace bpt {

__device__ __forceinline__ float ld_as_float(const float* p) { return *p; }
__device__ __forceinline__ float ld_as_float(const __half* p) { return __half2float(*p); }
__device__ __forceinline__ float ld_as_float(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Row copies of fp16 [., d] tensors between wave block rows and token rows
// (d % 8 == 0; row strides in elements, multiples of 8):
//   scatter = 0: out[r, :] = in[map(r), :], zeros where map(r) < 0;
//   scatter = 1: out[map(r), :] = in[r, :] where map(r) >= 0.
__global__ void rows_copy_f16_kernel(const __half* __restrict__ in, long long ld_in,
                                     __half* __restrict__ out, long long ld_out, long long rows,
                                     int d, RowMap map, int scatter) {
  const long long per_row = d / 8;
  const long long total = rows * per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / per_row;
    const int c = static_cast<int>(i - r * per_row) * 8;
    const long long g = map.map(r);
    if (scatter) {
      if (g >= 0)
        *reinterpret_cast<uint4*>(out + g * ld_out + c) =
            *reinterpret_cast<const uint4*>(in + r * ld_in + c);
    } else {
      *reinterpret_cast<uint4*>(out + r * ld_out + c) =
          g >= 0 ? *reinterpret_cast<const uint4*>(in + g * ld_in + c) : make_uint4(0, 0, 0, 0);
    }
  }
}

// out[r, :] = fp16(in[map(r), :]) for r < rows; d % 8 == 0.
__global__ void rows_f32_to_f16_kernel(const float* __restrict__ in, __half* __restrict__ out,
                                       long long rows, int d, RowMap map) {
  const long long per_row = d / 8;
  const long long total = rows * per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / per_row;
    const int c = static_cast<int>(i - r * per_row) * 8;
    const long long g = map.map(r);
    uint4 w = make_uint4(0, 0, 0, 0);
    if (g >= 0) {
      const float4 a = *reinterpret_cast<const float4*>(in + g * d + c);
      const float4 b = *reinterpret_cast<const float4*>(in + g * d + c + 4);
      w.x = pack_f16x2(a.x, a.y);
      w.y = pack_f16x2(a.z, a.w);
      w.z = pack_f16x2(b.x, b.y);
      w.w = pack_f16x2(b.z, b.w);
    }
    *reinterpret_cast<uint4*>(out + r * d + c) = w;
  }
}

// out[g, which*d + c] = fp16(in_which[g, c]) for which = 0, 1, 2 (dQ | dK | dV).
__global__ void pack3_f32_to_f16_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                        const float* __restrict__ c3, __half* __restrict__ out,
                                        long long rows, int d) {
  const long long per_row = 3LL * d / 8;
  const long long total = rows * per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / per_row;
    const int col = static_cast<int>(i - r * per_row) * 8;
    const int which = col / d, c = col - which * d;
    const float* src = (which == 0 ? a : which == 1 ? b : c3) + r * d + c;
    const float4 x = *reinterpret_cast<const float4*>(src);
    const float4 y = *reinterpret_cast<const float4*>(src + 4);
    uint4 w;
    w.x = pack_f16x2(x.x, x.y);
    w.y = pack_f16x2(x.z, x.w);
    w.z = pack_f16x2(y.x, y.y);
    w.w = pack_f16x2(y.z, y.w);
    *reinterpret_cast<uint4*>(out + r * 3LL * d + col) = w;
  }
}

// LayerNorm backward, one warp per local row r (g = map(r); rows beyond the
// sequence are skipped):
//   dx_ln = LN'(X[g]) applied to DY[r] (gamma from `gamma`)
//   OUT[g] = (accumulate ? OUT[g] : RES[g]) + dx_ln;  OUT16[r] = fp16(OUT[g]) if OUT16
//   rowstat[r] = (mean, rstd) of X[g]
template <typename TX, typename TG = __nv_bfloat16>
__global__ void ln_backward_kernel(const TX* __restrict__ X, const TG* __restrict__ gamma,
                                   const float* __restrict__ DY, const float* __restrict__ RES,
                                   float* __restrict__ OUT, __half* __restrict__ OUT16,
                                   float2* __restrict__ rowstat, long long rows, int d,
                                   RowMap map, int accumulate) {
  const int lane = threadIdx.x & 31;
  const long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  if (r >= rows) return;
  const long long g = map.map(r);
  if (g < 0) {
    if (rowstat && lane == 0) rowstat[r] = make_float2(0.f, 0.f);
    if (OUT16)
      for (int c = lane; c < d; c += 32) OUT16[r * d + c] = __float2half(0.f);
    return;
  }
  const TX* x = X + g * d;
  const float* dy = DY + r * d;
  float s = 0.f;
  for (int c = lane; c < d; c += 32) s += ld_as_float(x + c);
  const float mu = warp_sum(s) / d;
  float v = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float t = ld_as_float(x + c) - mu;
    v += t * t;
  }
  const float rstd = rsqrtf(warp_sum(v) / d + 1e-5f);
  float a = 0.f, b = 0.f;  // sum dxh, sum dxh * xh
  for (int c = lane; c < d; c += 32) {
    const float dxh = dy[c] * ld_as_float(gamma + c);
    a += dxh;
    b += dxh * (ld_as_float(x + c) - mu) * rstd;
  }
  a = warp_sum(a) / d;
  b = warp_sum(b) / d;
  float* out = OUT + g * d;
  const float* res = accumulate ? out : RES + g * d;
  for (int c = lane; c < d; c += 32) {
    const float xh = (ld_as_float(x + c) - mu) * rstd;
    const float dxh = dy[c] * ld_as_float(gamma + c);
    const float val = res[c] + rstd * (dxh - a - xh * b);
    out[c] = val;
    if (OUT16) OUT16[r * d + c] = __float2half(val);
  }
  if (rowstat && lane == 0) rowstat[r] = make_float2(mu, rstd);
}

// Four consecutive elements as fp32 (p 4-element aligned).
__device__ __forceinline__ float4 ld4_as_float(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 ld4_as_float(const __half* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 ld4_as_float(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// Column sums over `rows` rows split into row chunks, one partial per chunk:
//   part_a[chunk, c] = sum_r A[row(r), c]
//   part_b[chunk, c] = sum_r A[row(r), c] * (X[g(r), c] - mean_r) * rstd_r   (if X)
// A is indexed by the local row (a_global = 0) or by g = map(r) (a_global = 1).
// With a wave map a chunk is one query block (rows_per_chunk = map.blk), whose
// valid rows map to consecutive token rows; with the identity map, any run of
// rows.  Each thread sums four adjacent columns (d % 4 == 0) over its chunk's
// rows in order.
template <typename TA, typename TX>
__global__ void colsum_partial_kernel(const TA* __restrict__ A, int a_global,
                                      const TX* __restrict__ X, const float2* __restrict__ rowstat,
                                      float* __restrict__ part_a, float* __restrict__ part_b,
                                      long long rows, int d, int rows_per_chunk, RowMap map) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  const int chunk = blockIdx.y;
  if (c >= d) return;
  const long long r0 = static_cast<long long>(chunk) * rows_per_chunk;
  long long g0;  // token row of the chunk's first row
  int nv;        // rows of the chunk that exist
  if (map.identity) {
    g0 = r0;
    nv = static_cast<int>(min(static_cast<long long>(rows_per_chunk), rows - r0));
  } else {
    const long long item = map.item0 + r0 / map.blk;
    const long long b = item / map.nb;
    const long long pos0 = (item - b * map.nb) * map.blk;
    g0 = b * map.N + pos0;
    nv = static_cast<int>(min(static_cast<long long>(map.blk), map.N - pos0));
  }
  float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int i = 0; i < nv; ++i) {
    const float4 a = ld4_as_float(A + (a_global ? g0 + i : r0 + i) * d + c);
    sa.x += a.x;
    sa.y += a.y;
    sa.z += a.z;
    sa.w += a.w;
    if (X) {
      const float2 st = rowstat[r0 + i];
      const float4 x = ld4_as_float(X + (g0 + i) * d + c);
      sb.x += a.x * (x.x - st.x) * st.y;
      sb.y += a.y * (x.y - st.x) * st.y;
      sb.z += a.z * (x.z - st.x) * st.y;
      sb.w += a.w * (x.w - st.x) * st.y;
    }
  }
  *reinterpret_cast<float4*>(part_a + static_cast<long long>(chunk) * d + c) = sa;
  if (X) *reinterpret_cast<float4*>(part_b + static_cast<long long>(chunk) * d + c) = sb;
}

// out[c] += sum over chunks of part[chunk, c], chunks in order (deterministic).
__global__ void colsum_reduce_kernel(const float* __restrict__ part, int chunks, int d,
                                     float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
  float s = 0.f;
  for (int k = 0; k < chunks; ++k) s += part[static_cast<long long>(k) * d + c];
  out[c] += s;
}

// Per (head t, local row r) the two numbers the attention backward needs for
// query row r, stored per 128-row block as 128 a' then 128 -D (1 KB runs a
// bulk copy can fetch):
//   qs[((t * blocks + r / 128) * 2 + 0) * 128 + r % 128] = -(m + ln l) log2 e
//   qs[((t * blocks + r / 128) * 2 + 1) * 128 + r % 128] = -D,
// D = sum over head t's columns of dO[r, c] * O[r, c], (m, l) the forward's
// softmax statistics of the row's global position (stats [B][h][N]);
// P = 2^(S scale log2 e + a') is then the row's probability.  Rows past the
// sequence get a' = -inf, D = 0, which makes their probabilities 0.  One
// warp per row; rows is a multiple of 128.
__global__ void attn_row_terms_kernel(const __half* __restrict__ dO, const __half* __restrict__ O,
                                      const float2* __restrict__ stats, float* __restrict__ qs,
                                      long long rows, int d, int h, RowMap map) {
  const int lane = threadIdx.x & 31;
  const long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  if (r >= rows) return;
  const long long g = map.map(r);
  const int dk = d / h;
  const long long b = g >= 0 ? g / map.N : 0, pos = g >= 0 ? g - b * map.N : 0;
  const long long blocks = rows / 128;
  for (int t = 0; t < h; ++t) {
    float s = 0.f;
    for (int c = lane; c < dk; c += 32)
      s += __half2float(dO[r * d + t * dk + c]) * __half2float(O[r * d + t * dk + c]);
    s = warp_sum(s);
    if (lane == 0) {
      float a = -INFINITY, nd = 0.f;
      if (g >= 0) {
        const float2 ml = stats[(b * h + t) * map.N + pos];
        a = -(ml.x * 1.4426950408889634f + log2f(ml.y));
        nd = -s;
      }
      float* blk = qs + (t * blocks + r / 128) * 256;
      blk[r % 128] = a;
      blk[128 + r % 128] = nd;
    }
  }
}

}  // namespace bpt
