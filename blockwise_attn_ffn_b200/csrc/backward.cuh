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
//   * the attention backward: the row terms D = rowsum(dO * O) per head and
//     the dQ and dK/dV kernels, which recompute P = exp(s - m) / l from the
//     saved statistics.  These run on CUDA cores in fp32 arithmetic on fp16
//     operands (64-row tiles).
// Formulas (standard calculus), per head with s = q.k / sqrt(d_k):
//   P = exp(s - m) / l,  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//   dQ = dS K / sqrt(d_k),  dK = dS^T Q / sqrt(d_k);
//   LayerNorm y = g * xh + b: dx = rstd * (dxh - mean(dxh) - xh * mean(dxh * xh)),
//   dxh = dy * g,  dg = sum_rows dy * xh,  db = sum_rows dy.
#pragma once

#include "common.cuh"

namespace bpt {

__device__ __forceinline__ float ld_as_float(const float* p) { return *p; }
__device__ __forceinline__ float ld_as_float(const __half* p) { return __half2float(*p); }
__device__ __forceinline__ float ld_as_float(const __nv_bfloat16* p) { return __bfloat162float(*p); }

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
template <typename TX>
__global__ void ln_backward_kernel(const TX* __restrict__ X, const __nv_bfloat16* __restrict__ gamma,
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
    const float dxh = dy[c] * __bfloat162float(gamma[c]);
    a += dxh;
    b += dxh * (ld_as_float(x + c) - mu) * rstd;
  }
  a = warp_sum(a) / d;
  b = warp_sum(b) / d;
  float* out = OUT + g * d;
  const float* res = accumulate ? out : RES + g * d;
  for (int c = lane; c < d; c += 32) {
    const float xh = (ld_as_float(x + c) - mu) * rstd;
    const float dxh = dy[c] * __bfloat162float(gamma[c]);
    const float val = res[c] + rstd * (dxh - a - xh * b);
    out[c] = val;
    if (OUT16) OUT16[r * d + c] = __float2half(val);
  }
  if (rowstat && lane == 0) rowstat[r] = make_float2(mu, rstd);
}

// Column sums over `rows` rows split into row chunks, one partial per chunk:
//   part_a[chunk, c] = sum_r A[row(r), c]
//   part_b[chunk, c] = sum_r A[row(r), c] * (X[g(r), c] - mean_r) * rstd_r   (if X)
// A is indexed by the local row (a_global = 0) or by g = map(r) (a_global = 1).
template <typename TA, typename TX>
__global__ void colsum_partial_kernel(const TA* __restrict__ A, int a_global,
                                      const TX* __restrict__ X, const float2* __restrict__ rowstat,
                                      float* __restrict__ part_a, float* __restrict__ part_b,
                                      long long rows, int d, int rows_per_chunk, RowMap map) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int chunk = blockIdx.y;
  if (c >= d) return;
  const long long r0 = static_cast<long long>(chunk) * rows_per_chunk;
  const long long r1 = min(rows, r0 + rows_per_chunk);
  float sa = 0.f, sb = 0.f;
  for (long long r = r0; r < r1; ++r) {
    const long long g = map.map(r);
    if (g < 0) continue;
    const float a = ld_as_float(A + (a_global ? g : r) * d + c);
    sa += a;
    if (X) {
      const float2 st = rowstat[r];
      sb += a * (ld_as_float(X + g * d + c) - st.x) * st.y;
    }
  }
  part_a[static_cast<long long>(chunk) * d + c] = sa;
  if (X) part_b[static_cast<long long>(chunk) * d + c] = sb;
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

// D[r, t] = sum over head t's columns of dO[r, c] * O[r, c]; one warp per row.
__global__ void attn_row_dot_kernel(const __half* __restrict__ dO, const __half* __restrict__ O,
                                    float* __restrict__ D, long long rows, int d, int h) {
  const int lane = threadIdx.x & 31;
  const long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  if (r >= rows) return;
  const int dk = d / h;
  for (int t = 0; t < h; ++t) {
    float s = 0.f;
    for (int c = lane; c < dk; c += 32)
      s += __half2float(dO[r * d + t * dk + c]) * __half2float(O[r * d + t * dk + c]);
    s = warp_sum(s);
    if (lane == 0) D[r * h + t] = s;
  }
}

// ------------------------------------------------- attention gradients --
struct AttnBwdParams {
  const __half* qkv;     // [B*N, 3d] fp16: Q | K | V per token (global rows)
  const __half* o;       // [count * 128, d] fp16, this wave's block rows
  const __half* dO;      // [count * 128, d] fp16, this wave's block rows
  const float* D;        // [count * 128, h] rowsum(dO * O) per head
  const float2* stats;   // [B][h][N] (m, l) from the forward
  float* dq;             // [B*N, d] written for this wave's rows
  float* dk;             // [B*N, d] accumulated (+=)
  float* dv;             // [B*N, d] accumulated (+=)
  int N, nb, h, d, causal, item0, count, seqs;
  float scale;           // 1 / sqrt(d_k)
};

constexpr int kBwdRows = 64;  // query / key tile of the SIMT attention backward

template <int DK>
struct AttnBwdSmem {
  static constexpr int TILE = kBwdRows * DK;              // floats
  static constexpr int PT = kBwdRows * (kBwdRows + 1);    // floats, padded
  static constexpr int DQ_BYTES = (4 * TILE + PT + 3 * kBwdRows) * 4;
  static constexpr int DKV_BYTES = (4 * TILE + 2 * PT + 3 * kBwdRows) * 4;
};

__device__ __forceinline__ void load_tile_f16(float* dst, const __half* src, long long ld,
                                              int col0, int dk, long long row0, int nrows_valid) {
  // dst[r][c] = src[(row0 + r) * ld + col0 + c] for r < nrows_valid, else 0
  for (int t = threadIdx.x; t < kBwdRows * dk; t += blockDim.x) {
    const int r = t / dk, c = t - (t / dk) * dk;
    dst[t] = r < nrows_valid ? __half2float(src[(row0 + r) * ld + col0 + c]) : 0.f;
  }
}

// dQ for one 64-row query tile of the wave and one head.  256 threads: row
// r = tid / 4 of the tile, sub = tid % 4 takes key columns sub, sub + 4, ...
template <int DK>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const AttnBwdParams p) {
  extern __shared__ float smf[];
  using S = AttnBwdSmem<DK>;
  float* sQ = smf;
  float* sdO = sQ + S::TILE;
  float* sK = sdO + S::TILE;
  float* sV = sK + S::TILE;
  float* sS = sV + S::TILE;          // dS [64][65]
  float* sM = sS + S::PT;            // m, l, D per row
  float* sL = sM + kBwdRows;
  float* sD = sL + kBwdRows;
  const int head = blockIdx.y;
  const int q = blockIdx.x;                       // 64-row tile of the wave
  const int item = p.item0 + q / 2;
  const int bidx = item / p.nb, iblk = item - (item / p.nb) * p.nb;
  const int pos0 = iblk * 128 + (q & 1) * kBwdRows;
  const long long lrow0 = static_cast<long long>(q / 2) * 128 + (q & 1) * kBwdRows;
  const int nvalid = max(0, min(kBwdRows, p.N - pos0));
  const long long g0 = static_cast<long long>(bidx) * p.N + pos0;
  const long long ld3 = 3LL * p.d;
  const int r = threadIdx.x >> 2, sub = threadIdx.x & 3;
  if (nvalid == 0) return;
  load_tile_f16(sQ, p.qkv, ld3, head * DK, DK, g0, nvalid);
  load_tile_f16(sdO, p.dO, p.d, head * DK, DK, lrow0, nvalid);
  if (threadIdx.x < kBwdRows) {
    const int rr = threadIdx.x;
    const bool ok = rr < nvalid;
    const float2 st = ok ? p.stats[(static_cast<long long>(bidx) * p.h + head) * p.N + pos0 + rr]
                         : make_float2(0.f, 1.f);
    sM[rr] = st.x;
    sL[rr] = st.y;
    sD[rr] = ok ? p.D[(lrow0 + rr) * p.h + head] : 0.f;
  }
  float acc[DK / 4];
#pragma unroll
  for (int t = 0; t < DK / 4; ++t) acc[t] = 0.f;
  const int pos = pos0 + r;
  const int kend = p.causal ? min(p.N, pos0 + kBwdRows) : p.N;
  for (int k0 = 0; k0 < kend; k0 += kBwdRows) {
    __syncthreads();
    const int kvalid = min(kBwdRows, p.N - k0);
    const long long gk = static_cast<long long>(bidx) * p.N + k0;
    load_tile_f16(sK, p.qkv, ld3, p.d + head * DK, DK, gk, kvalid);
    load_tile_f16(sV, p.qkv, ld3, 2 * p.d + head * DK, DK, gk, kvalid);
    __syncthreads();
    const float m = sM[r], linv = 1.0f / sL[r], Dr = sD[r];
#pragma unroll 4
    for (int t = 0; t < kBwdRows / 4; ++t) {
      const int kk = sub + 4 * t;
      const int kp = k0 + kk;
      float ds = 0.f;
      if (r < nvalid && kk < kvalid && (!p.causal || kp <= pos)) {
        float sc = 0.f, dp = 0.f;
        for (int c = 0; c < DK; ++c) {
          sc = fmaf(sQ[r * DK + c], sK[kk * DK + c], sc);
          dp = fmaf(sdO[r * DK + c], sV[kk * DK + c], dp);
        }
        const float pr = expf(sc * p.scale - m) * linv;
        ds = pr * (dp - Dr);
      }
      sS[r * (kBwdRows + 1) + kk] = ds;
    }
    __syncwarp();
#pragma unroll
    for (int t = 0; t < DK / 4; ++t) {
      const int c = sub + 4 * t;
      float a = 0.f;
      for (int kk = 0; kk < kBwdRows; ++kk) a = fmaf(sS[r * (kBwdRows + 1) + kk], sK[kk * DK + c], a);
      acc[t] += a;
    }
  }
  if (r < nvalid) {
    float* dst = p.dq + (g0 + r) * p.d + head * DK;
#pragma unroll
    for (int t = 0; t < DK / 4; ++t) dst[sub + 4 * t] = acc[t] * p.scale;
  }
}

// dK, dV contributions of this wave's query rows to one 64-key tile of one
// head and sequence (grid: key tiles x heads x sequences of the wave).
// 256 threads: key row k = tid / 4, sub = tid % 4 takes query columns sub,
// sub + 4, ... of each query tile, and head columns sub, sub + 4, ... of the
// accumulators.
template <int DK>
__global__ void __launch_bounds__(256) attn_bwd_dkv_kernel(const AttnBwdParams p) {
  extern __shared__ float smf[];
  using S = AttnBwdSmem<DK>;
  float* sQ = smf;
  float* sdO = sQ + S::TILE;
  float* sK = sdO + S::TILE;
  float* sV = sK + S::TILE;
  float* sP = sV + S::TILE;          // P^T [64 keys][65]
  float* sS = sP + S::PT;            // dS^T [64 keys][65]
  float* sM = sS + S::PT;
  float* sL = sM + kBwdRows;
  float* sD = sL + kBwdRows;
  const int head = blockIdx.y;
  const int bidx = (p.seqs > 0 ? p.item0 / p.nb + static_cast<int>(blockIdx.z) : p.item0 / p.nb);
  const int k0 = blockIdx.x * kBwdRows;
  if (k0 >= p.N) return;
  // this wave's query positions in sequence bidx: [qlo, qhi)
  int qlo, qhi;
  long long lbase;  // wave scratch row of position 0 of this sequence
  if (p.seqs > 0) {
    qlo = 0;
    qhi = p.N;
    lbase = static_cast<long long>(bidx * p.nb - p.item0) * 128;
  } else {
    const int i0 = p.item0 - bidx * p.nb;
    qlo = i0 * 128;
    qhi = min(p.N, (i0 + p.count) * 128);
    lbase = -static_cast<long long>(qlo);
  }
  const int qstart = p.causal ? max(qlo, k0 - (k0 % kBwdRows)) : qlo;
  if (qstart >= qhi) return;
  const int kvalid = min(kBwdRows, p.N - k0);
  const long long ld3 = 3LL * p.d;
  const long long gk = static_cast<long long>(bidx) * p.N + k0;
  const int k = threadIdx.x >> 2, sub = threadIdx.x & 3;
  load_tile_f16(sK, p.qkv, ld3, p.d + head * DK, DK, gk, kvalid);
  load_tile_f16(sV, p.qkv, ld3, 2 * p.d + head * DK, DK, gk, kvalid);
  float ak[DK / 4], av[DK / 4];
#pragma unroll
  for (int t = 0; t < DK / 4; ++t) ak[t] = av[t] = 0.f;
  const int kp = k0 + k;
  for (int q0 = qstart; q0 < qhi; q0 += kBwdRows) {
    __syncthreads();
    const int qvalid = min(kBwdRows, qhi - q0);
    const long long gq = static_cast<long long>(bidx) * p.N + q0;
    load_tile_f16(sQ, p.qkv, ld3, head * DK, DK, gq, qvalid);
    load_tile_f16(sdO, p.dO, p.d, head * DK, DK, lbase + q0, qvalid);
    if (threadIdx.x < kBwdRows) {
      const int rr = threadIdx.x;
      const bool ok = rr < qvalid;
      const float2 st = ok ? p.stats[(static_cast<long long>(bidx) * p.h + head) * p.N + q0 + rr]
                           : make_float2(0.f, 1.f);
      sM[rr] = st.x;
      sL[rr] = st.y;
      sD[rr] = ok ? p.D[(lbase + q0 + rr) * p.h + head] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kBwdRows / 4; ++t) {
      const int rr = sub + 4 * t;
      const int qp = q0 + rr;
      float pr = 0.f, ds = 0.f;
      if (k < kvalid && rr < qvalid && (!p.causal || kp <= qp)) {
        float sc = 0.f, dp = 0.f;
        for (int c = 0; c < DK; ++c) {
          sc = fmaf(sQ[rr * DK + c], sK[k * DK + c], sc);
          dp = fmaf(sdO[rr * DK + c], sV[k * DK + c], dp);
        }
        pr = expf(sc * p.scale - sM[rr]) / sL[rr];
        ds = pr * (dp - sD[rr]);
      }
      sP[k * (kBwdRows + 1) + rr] = pr;
      sS[k * (kBwdRows + 1) + rr] = ds;
    }
    __syncwarp();
#pragma unroll
    for (int t = 0; t < DK / 4; ++t) {
      const int c = sub + 4 * t;
      float a = 0.f, b = 0.f;
      for (int rr = 0; rr < kBwdRows; ++rr) {
        a = fmaf(sP[k * (kBwdRows + 1) + rr], sdO[rr * DK + c], a);
        b = fmaf(sS[k * (kBwdRows + 1) + rr], sQ[rr * DK + c], b);
      }
      av[t] += a;
      ak[t] += b;
    }
  }
  if (k < kvalid) {
    float* dkr = p.dk + (gk + k) * p.d + head * DK;
    float* dvr = p.dv + (gk + k) * p.d + head * DK;
#pragma unroll
    for (int t = 0; t < DK / 4; ++t) {
      dkr[sub + 4 * t] += ak[t] * p.scale;
      dvr[sub + 4 * t] += av[t];
    }
  }
}

}  // namespace bpt
