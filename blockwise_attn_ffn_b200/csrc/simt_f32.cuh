// fp32 path: CUDA-core (FFMA) kernels for float32 inputs.
//
// TF32 tensor cores (unit roundoff 2^-11) cannot hold a 1e-4 absolute error
// on this layer, so the fp32 path computes every product and sum in fp32 on
// the CUDA cores.  Same block schedule and epilogues as the bf16 path:
//   gemm_f32_kernel: C = A B with the four epilogues of the tensor-core GEMM
//   attn_f32_kernel: blockwise online-softmax attention, 64-row query blocks
#pragma once

#include "common.cuh"

namespace bpt {

struct GemmF32Params {
  int M, N, K;
  int n_sub;          // columns of each concatenated B matrix
  const float* A;     // [M, K]
  const float* B[3];  // [K, n_sub] each
  int epi;            // GemmEpi
  float* out;         // kEpiStoreF16 / kEpiGeluBias (fp32 here): [M, ld_out]; else residual rows
  long long ld_out;
  const float* resid;  // kEpiResidX: x
  long long ld_resid;
  const float* bias;
  RowMap map;
};

constexpr int kF32Tile = 64, kF32BK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(const GemmF32Params p) {
  __shared__ float sA[kF32BK][kF32Tile + 4];
  __shared__ float sB[kF32BK][kF32Tile + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * kF32Tile, n0 = blockIdx.x * kF32Tile;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += kF32BK) {
    for (int t = threadIdx.x; t < kF32Tile * kF32BK; t += 256) {
      const int mm = t / kF32BK, kk = t % kF32BK;
      const int gm = m0 + mm, gk = k0 + kk;
      sA[kk][mm] = (gm < p.M && gk < p.K) ? p.A[static_cast<long long>(gm) * p.K + gk] : 0.f;
      const int nn = t % kF32Tile, kb = t / kF32Tile;
      const int gn = n0 + nn, gkb = k0 + kb;
      float bv = 0.f;
      if (gn < p.N && gkb < p.K) {
        const int which = gn / p.n_sub;
        bv = p.B[which][static_cast<long long>(gkb) * p.n_sub + (gn - which * p.n_sub)];
      }
      sB[kb][nn] = bv;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kF32BK; ++kk) {
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
    const long long row = m0 + ty * 4 + i;
    if (row >= p.M) continue;
    long long g = row;
    if (p.epi == kEpiResidX || p.epi == kEpiBiasAccum) {
      g = p.map.map(row);
      if (g < 0) continue;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      if (col >= p.N) continue;
      const float v = acc[i][j];
      if (p.epi == kEpiStoreF16) {
        p.out[row * p.ld_out + col] = v;
      } else if (p.epi == kEpiGeluBias) {
        const float z = v + p.bias[col];
        p.out[row * p.ld_out + col] = 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
      } else if (p.epi == kEpiResidX) {
        p.out[g * p.ld_out + col] = p.resid[g * p.ld_resid + col] + v;
      } else {
        float* o = p.out + g * p.ld_out + col;
        *o = *o + v + p.bias[col];
      }
    }
  }
}

struct AttnF32Params {
  const float* qkv;  // [B*N, 3d]
  float* o;          // [count * blk, d]
  int N, nb, h, d, causal, item0, blk;
  float scale;       // 1 / sqrt(d_k)
  float* stats;      // nullable: per-row softmax statistics [B][h][N][2] (m, l)
};

constexpr int kF32AttnRows = 64;     // query / key-value block
constexpr int kF32AttnMaxDk = 128;

// One CTA per (block item, head); 256 threads = 64 rows x 4 threads.
// Dynamic shared memory: Q, K, V tiles [64][d_k] and P [64][65].
__global__ void __launch_bounds__(256) attn_f32_kernel(const AttnF32Params p) {
  extern __shared__ float sm[];
  const int dk = p.d / p.h;
  float* sQ = sm;
  float* sK = sQ + kF32AttnRows * dk;
  float* sV = sK + kF32AttnRows * dk;
  float* sP = sV + kF32AttnRows * dk;  // [64][65]
  const int item = p.item0 + blockIdx.x / p.h;
  const int head = blockIdx.x % p.h;
  const int bidx = item / p.nb, iblk = item % p.nb;
  const int r = threadIdx.x >> 2, sub = threadIdx.x & 3;
  const long long ld = 3LL * p.d;
  const float* base = p.qkv + static_cast<long long>(bidx) * p.N * ld;
  const int q0 = iblk * kF32AttnRows;

  for (int t = threadIdx.x; t < kF32AttnRows * dk; t += 256) {
    const int rr = t / dk, cc = t % dk;
    const int pos = q0 + rr;
    sQ[t] = pos < p.N ? base[pos * ld + head * dk + cc] : 0.f;
  }
  float m = -INFINITY, l = 0.f;
  float o[kF32AttnMaxDk / 4];
#pragma unroll
  for (int t = 0; t < kF32AttnMaxDk / 4; ++t) o[t] = 0.f;
  const int qpos = q0 + r;
  const int n_kv = p.causal ? iblk + 1 : p.nb;
  for (int j = 0; j < n_kv; ++j) {
    const int k0 = j * kF32AttnRows;
    __syncthreads();
    for (int t = threadIdx.x; t < kF32AttnRows * dk; t += 256) {
      const int rr = t / dk, cc = t % dk;
      const int pos = k0 + rr;
      sK[t] = pos < p.N ? base[pos * ld + p.d + head * dk + cc] : 0.f;
      sV[t] = pos < p.N ? base[pos * ld + 2 * p.d + head * dk + cc] : 0.f;
    }
    __syncthreads();
    float s[16];
    float mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const int kk = sub + 4 * t;
      const int kpos = k0 + kk;
      const bool allowed = kpos < p.N && (!p.causal || kpos <= qpos);
      float acc = 0.f;
      for (int c = 0; c < dk; ++c) acc = fmaf(sQ[r * dk + c], sK[kk * dk + c], acc);
      s[t] = allowed ? acc * p.scale : -INFINITY;
      mx = fmaxf(mx, s[t]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    // a row with no allowed key so far keeps m = -inf and weight 0
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    float rs = 0.f;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const float pv = (m_new == -INFINITY || s[t] == -INFINITY) ? 0.f : expf(s[t] - m_new);
      sP[r * 65 + sub + 4 * t] = pv;
      rs += pv;
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l = alpha * l + rs;
    m = m_new;
    __syncwarp();
    for (int t = 0; t < dk / 4; ++t) {
      const int c = sub + 4 * t;
      float acc = 0.f;
      for (int kk = 0; kk < kF32AttnRows; ++kk) acc = fmaf(sP[r * 65 + kk], sV[kk * dk + c], acc);
      o[t] = alpha * o[t] + acc;
    }
  }
  const long long srow = static_cast<long long>(item - p.item0) * kF32AttnRows + r;
  float* dst = p.o + srow * p.d + head * dk;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  for (int t = 0; t < dk / 4; ++t) dst[sub + 4 * t] = o[t] * inv;
  if (p.stats != nullptr && sub == 0 && qpos < p.N) {
    float* st = p.stats + ((static_cast<long long>(bidx) * p.h + head) * p.N + qpos) * 2;
    st[0] = m;
    st[1] = l;
  }
}

}  // namespace bpt
