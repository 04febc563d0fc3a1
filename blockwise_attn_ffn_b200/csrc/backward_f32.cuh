// Backward pass of the BPT layer for fp32 layers, on the CUDA cores.
//
// "Blockwise Parallel Transformer — BPT", section "The backward pass": the
// same schedule as the bf16 path (waves of query blocks recomputed from x and
// the saved (m, l), gradients accumulated wave by wave), every product and
// sum in fp32 FFMA: the fp32 path serves the small layers whose oracle
// comparison needs 1e-4-level agreement, so simple SIMT kernels suffice:
//   gemm_f32_gen_kernel       C (+)= op(A) op(B), either operand transposed
//   gather_rows_f32_kernel    wave rows of a global [M, d] tensor
//   bias_gelu_keep_f32_kernel Hpre += b_1, H = GELU(Hpre)
//   gelu_grad_mul_f32_kernel  dHpre = dH * GELU'(Hpre)
//   attn_row_terms_f32_kernel per (row, head): (-(m + ln l) log2 e, -D)
//   attn_bwd_dq_f32_kernel    one warp per (wave row, head): dQ
//   attn_bwd_dkv_f32_kernel   one warp per (key row, head): dK, dV (+=)
// With s = q.k / sqrt(d_k), P = exp(s - m) / l = 2^(s log2 e + a'),
// D = rowsum(dO * O): dP = dO V^T, dS = P (dP - D), dV = P^T dO,
// dK = dS^T Q / sqrt(d_k), dQ = dS K / sqrt(d_k).
#pragma once

#include "common.cuh"

namespace bpt {

struct GemmGenF32 {
  int M, N, K;
  const float* A;
  long long lda;
  int a_t;  // 0: A[m * lda + k]; 1: A[k * lda + m]
  const float* B;
  long long ldb;
  int b_t;  // 0: B[k * ldb + n]; 1: B[n * ldb + k]
  float* C;
  long long ldc;
  int acc;  // 1: C += ; 0: C =
};

// 64 x 64 tile per CTA, k-steps of 16 staged in shared memory, 4 x 4
// outputs per thread.
__global__ void __launch_bounds__(256) gemm_f32_gen_kernel(const GemmGenF32 p) {
  __shared__ float sA[16][64 + 4];
  __shared__ float sB[16][64 + 4];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += 16) {
    for (int t = threadIdx.x; t < 64 * 16; t += 256) {
      int m, k;
      if (p.a_t) {
        m = t & 63;
        k = t >> 6;
      } else {
        k = t & 15;
        m = t >> 4;
      }
      const int gm = m0 + m, gk = k0 + k;
      float a = 0.f;
      if (gm < p.M && gk < p.K)
        a = p.a_t ? p.A[static_cast<long long>(gk) * p.lda + gm]
                  : p.A[static_cast<long long>(gm) * p.lda + gk];
      sA[k][m] = a;
      int n;
      if (p.b_t) {
        k = t & 15;
        n = t >> 4;
      } else {
        n = t & 63;
        k = t >> 6;
      }
      const int gn = n0 + n, gk2 = k0 + k;
      float b = 0.f;
      if (gn < p.N && gk2 < p.K)
        b = p.b_t ? p.B[static_cast<long long>(gn) * p.ldb + gk2]
                  : p.B[static_cast<long long>(gk2) * p.ldb + gn];
      sB[k][n] = b;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sB[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= p.N) continue;
      float* c = p.C + static_cast<long long>(gm) * p.ldc + gn;
      *c = p.acc ? *c + acc[i][j] : acc[i][j];
    }
  }
}

// dst[r, :] = src[map(r), :] (zeros for rows past the sequence)
__global__ void gather_rows_f32_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                       long long rows, int d, RowMap map) {
  const long long total = rows * d;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / d, c = i - r * d;
    const long long g = map.map(r);
    dst[i] = g >= 0 ? src[g * d + c] : 0.f;
  }
}

// Hpre += b_1 (per column); H = GELU(Hpre)
__global__ void bias_gelu_keep_f32_kernel(float* __restrict__ hpre, const float* __restrict__ b1,
                                          float* __restrict__ hh, long long rows, int d_ff) {
  const long long total = rows * d_ff;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float z = hpre[i] + b1[i % d_ff];
    hpre[i] = z;
    hh[i] = gelu_erf(z);
  }
}

// dh *= GELU'(hpre)
__global__ void gelu_grad_mul_f32_kernel(float* __restrict__ dh, const float* __restrict__ hpre,
                                         long long n) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    dh[i] *= gelu_erf_grad(hpre[i]);
}

// rt[t * rows + r] = (-(m + ln l) log2 e, -D) for wave row r, head t, with
// D = sum over head t's columns of dO[r] * O[r] and (m, l) the forward's
// statistics of the row's position (stats [B][h][N]); (-inf, 0) for rows past
// the sequence.  One warp per row.
__global__ void attn_row_terms_f32_kernel(const float* __restrict__ dO, const float* __restrict__ O,
                                          const float2* __restrict__ stats,
                                          float2* __restrict__ rt, long long rows, int d, int h,
                                          RowMap map) {
  const int lane = threadIdx.x & 31;
  const long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  if (r >= rows) return;
  const long long g = map.map(r);
  const int dk = d / h;
  const long long b = g >= 0 ? g / map.N : 0, pos = g >= 0 ? g - b * map.N : 0;
  for (int t = 0; t < h; ++t) {
    float s = 0.f;
    for (int c = lane; c < dk; c += 32) s += dO[r * d + t * dk + c] * O[r * d + t * dk + c];
    s = warp_sum(s);
    if (lane == 0) {
      float2 v = make_float2(-INFINITY, 0.f);
      if (g >= 0) {
        const float2 ml = stats[(b * h + t) * map.N + pos];
        v = make_float2(-(ml.x * 1.4426950408889634f + log2f(ml.y)), -s);
      }
      rt[t * rows + r] = v;
    }
  }
}

struct AttnBwdF32Params {
  const float* qkv;   // [B*N, 3d] (Q | K | V per row)
  const float* dO;    // [rows, d] this wave's block rows
  const float2* rt;   // [h][rows] row terms
  float* dq;          // [B*N, d] written (this wave's query rows)
  float* dk;          // [B*N, d] accumulated
  float* dv;          // [B*N, d] accumulated
  long long rows;     // wave rows
  int N, d, h, causal;
  float scale;        // 1 / sqrt(d_k)
  RowMap map;
};

// d_k <= 128: a lane holds columns lane, lane + 32, lane + 64, lane + 96.
constexpr int kF32BwdCols = 4;

// One warp per (wave row r, head t): dQ[r] = scale * sum_j dS_rj k_j.
__global__ void attn_bwd_dq_f32_kernel(const AttnBwdF32Params p) {
  const int lane = threadIdx.x & 31;
  const long long w = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  if (w >= p.rows * p.h) return;
  const long long r = w / p.h;
  const int t = static_cast<int>(w - r * p.h);
  const long long g = p.map.map(r);
  if (g < 0) return;
  const int dk = p.d / p.h;
  const long long b = g / p.N, qpos = g - b * p.N;
  const long long ld = 3LL * p.d;
  float q[kF32BwdCols], o[kF32BwdCols], acc[kF32BwdCols];
#pragma unroll
  for (int i = 0; i < kF32BwdCols; ++i) {
    const int c = lane + 32 * i;
    q[i] = c < dk ? p.qkv[g * ld + t * dk + c] : 0.f;
    o[i] = c < dk ? p.dO[r * p.d + t * dk + c] : 0.f;
    acc[i] = 0.f;
  }
  const float2 term = p.rt[static_cast<long long>(t) * p.rows + r];
  const float c2 = p.scale * 1.4426950408889634f;
  const long long kend = p.causal ? qpos + 1 : p.N;
  for (long long j = 0; j < kend; ++j) {
    const float* kr = p.qkv + (b * p.N + j) * ld + p.d + t * dk;
    const float* vr = kr + p.d;
    float sk = 0.f, sv = 0.f, kk[kF32BwdCols];
#pragma unroll
    for (int i = 0; i < kF32BwdCols; ++i) {
      const int c = lane + 32 * i;
      kk[i] = c < dk ? kr[c] : 0.f;
      sk += q[i] * kk[i];
      sv += o[i] * (c < dk ? vr[c] : 0.f);
    }
    sk = warp_sum(sk);
    sv = warp_sum(sv);
    const float pr = exp2f(fmaf(sk, c2, term.x));
    const float ds = pr * (sv + term.y);
#pragma unroll
    for (int i = 0; i < kF32BwdCols; ++i) acc[i] = fmaf(ds, kk[i], acc[i]);
  }
#pragma unroll
  for (int i = 0; i < kF32BwdCols; ++i) {
    const int c = lane + 32 * i;
    if (c < dk) p.dq[g * p.d + t * dk + c] = acc[i] * p.scale;
  }
}

// One warp per (key row gk of the batch, head t): over this wave's query rows
// that see it, dV[gk] += sum P dO and dK[gk] += scale * sum dS q.
__global__ void attn_bwd_dkv_f32_kernel(const AttnBwdF32Params p, long long key_rows) {
  const int lane = threadIdx.x & 31;
  const long long w = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  if (w >= key_rows * p.h) return;
  const long long gk = w / p.h;
  const int t = static_cast<int>(w - gk * p.h);
  const int dk = p.d / p.h;
  const long long b = gk / p.N, kpos = gk - b * p.N;
  const long long ld = 3LL * p.d;
  float kk[kF32BwdCols], vv[kF32BwdCols], ak[kF32BwdCols], av[kF32BwdCols];
#pragma unroll
  for (int i = 0; i < kF32BwdCols; ++i) {
    const int c = lane + 32 * i;
    kk[i] = c < dk ? p.qkv[gk * ld + p.d + t * dk + c] : 0.f;
    vv[i] = c < dk ? p.qkv[gk * ld + 2 * p.d + t * dk + c] : 0.f;
    ak[i] = av[i] = 0.f;
  }
  const float c2 = p.scale * 1.4426950408889634f;
  bool any = false;
  for (long long r = 0; r < p.rows; ++r) {
    const long long g = p.map.map(r);
    if (g < 0 || g / p.N != b) continue;
    if (p.causal && g - b * p.N < kpos) continue;
    any = true;
    const float* qr = p.qkv + g * ld + t * dk;
    const float* orow = p.dO + r * p.d + t * dk;
    float sq = 0.f, so = 0.f, qv[kF32BwdCols], ov[kF32BwdCols];
#pragma unroll
    for (int i = 0; i < kF32BwdCols; ++i) {
      const int c = lane + 32 * i;
      qv[i] = c < dk ? qr[c] : 0.f;
      ov[i] = c < dk ? orow[c] : 0.f;
      sq += qv[i] * kk[i];
      so += ov[i] * vv[i];
    }
    sq = warp_sum(sq);
    so = warp_sum(so);
    const float2 term = p.rt[static_cast<long long>(t) * p.rows + r];
    const float pr = exp2f(fmaf(sq, c2, term.x));
    const float ds = pr * (so + term.y);
#pragma unroll
    for (int i = 0; i < kF32BwdCols; ++i) {
      av[i] = fmaf(pr, ov[i], av[i]);
      ak[i] = fmaf(ds, qv[i], ak[i]);
    }
  }
  if (!any) return;
#pragma unroll
  for (int i = 0; i < kF32BwdCols; ++i) {
    const int c = lane + 32 * i;
    if (c < dk) {
      p.dv[gk * p.d + t * dk + c] += av[i];
      p.dk[gk * p.d + t * dk + c] += ak[i] * p.scale;
    }
  }
}

}  // namespace bpt
