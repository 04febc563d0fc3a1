// Blockwise causal / non-causal attention for one query block and one head per
// CTA, on the tcgen05 tensor cores (the BPT inner loop).
//
// For query block i of sequence b and head t, the CTA keeps the online-softmax
// state (running reference max m, running sum l, accumulator o) and walks the
// key/value blocks j = 0..i (causal; blocks j > i are never loaded or scored)
// or j = 0..nb-1.  Per step: S = Q K_j^T into tensor memory (UMMA), softmax
// warps turn S into P = exp(S/sqrt(d_k) - m) in bf16 and l += rowsum(P), then
// O += P V_j (UMMA, accumulator in tensor memory).  When the running max grows
// by more than 2^8 in exp2 units the accumulator O is rescaled by
// alpha = exp(m_old - m_new); smaller growth keeps the old reference, which is
// exact (o / l does not depend on the reference) and keeps P <= 2^8.
// Finally o / l is written in bf16 to the wave's block scratch, head t's
// columns.
//
// Operand layout (all 128-byte swizzled, loaded by 3-D TMA over the QKV buffer
// viewed as [B][N][3d]): Q and K tiles are K-major (d_k contiguous), V is the
// MN-major B operand of P V (d_k contiguous), P is written by the softmax
// warps in K-major swizzled form.  Tensor memory: S double buffer at columns
// 0..255, O at 256..256+d_k.
//
// Warp roles (256 threads): warp 0 TMA, warp 1 UMMA issue, warp 2 tensor
// memory owner, warps 4..7 softmax (thread = query row).
#pragma once

#include "common.cuh"

namespace bpt {

struct AttnParams {
  int N;         // tokens per sequence
  int nb;        // query blocks per sequence
  int h;         // heads
  int d;         // model width (row stride of Q, K and V is 3d)
  int causal;
  int item0;     // first flattened block item (batch * nb + block) of the wave
  int count;     // block items in the wave
  int seqs;      // >0: the wave is `seqs` whole sequences; 0: part of one sequence
  __nv_bfloat16* o;  // [count * 128, d] block scratch
  float scale_log2;  // log2(e) / sqrt(d_k)
  uint32_t* err;
};

template <int D>
struct AttnTile {
  static constexpr int BQ = 128;
  static constexpr int BKV = 128;
  static constexpr int KST = (D == 128) ? 2 : 3;  // K/V pipeline stages
  static constexpr int CHUNK = BQ * 128;           // one 64-column swizzled chunk: 16 KB
  static constexpr int Q_BYTES = BQ * D * 2;
  static constexpr int KV_BYTES = BKV * D * 2;
  static constexpr int P_BYTES = BQ * BKV * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_P = OFF_V + KST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_O = 256;
};

// Block item processed by CTA rank `rank`: longest work first under a causal
// mask (descending query block), so the grid drains evenly.
__device__ __forceinline__ int attn_item_for_rank(const AttnParams& p, int rank) {
  if (!p.causal) return p.item0 + rank;
  if (p.seqs == 0) return p.item0 + p.count - 1 - rank;
  const int b0 = p.item0 / p.nb;
  const int i = p.nb - 1 - rank / p.seqs;
  const int b = b0 + rank % p.seqs;
  return b * p.nb + i;
}

template <int D>
__global__ void __launch_bounds__(256, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap mapQKV, const AttnParams p) {
  using T = AttnTile<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t k_full0 = smem_u32(bars + 1);
  const uint32_t k_empty0 = smem_u32(bars + 1 + T::KST);
  const uint32_t v_full0 = smem_u32(bars + 1 + 2 * T::KST);
  const uint32_t v_empty0 = smem_u32(bars + 1 + 3 * T::KST);
  const uint32_t s_full0 = smem_u32(bars + 1 + 4 * T::KST);
  const uint32_t p_full = smem_u32(bars + 3 + 4 * T::KST);
  const uint32_t pv_done = smem_u32(bars + 4 + 4 * T::KST);
  const uint32_t drain = smem_u32(bars + 5 + 4 * T::KST);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = blockIdx.x / p.h;
  const int head = blockIdx.x - rank * p.h;
  const int item = attn_item_for_rank(p, rank);
  const int bidx = item / p.nb;
  const int iblk = item - bidx * p.nb;
  const int n_kv = p.causal ? iblk + 1 : p.nb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < T::KST; ++s) {
      mbar_init(k_full0 + 8 * s, 1);
      mbar_init(k_empty0 + 8 * s, 1);
      mbar_init(v_full0 + 8 * s, 1);
      mbar_init(v_empty0 + 8 * s, 1);
    }
    mbar_init(s_full0, 1);
    mbar_init(s_full0 + 8, 1);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&tmem_base_sh), T::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  const int colQ = head * D, colK = p.d + head * D, colV = 2 * p.d + head * D;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&mapQKV);
    int armed_k[T::KST], armed_v[T::KST];
    for (int s = 0; s < T::KST; ++s) armed_k[s] = armed_v[s] = -1;
    mbar_arrive_expect_tx(q_full, T::Q_BYTES);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_load_3d(smem_u32(smem + T::OFF_Q + c * T::CHUNK), &mapQKV, q_full, colQ + 64 * c,
                  iblk * T::BQ, bidx);
    for (int j = 0; j < n_kv; ++j) {
      const int st = j % T::KST;
      const uint32_t ph = (j / T::KST) & 1;
      if (!mbar_wait(k_empty0 + 8 * st, ph ^ 1u, abort_flag, p.err, kSiteAttnProducer)) break;
      mbar_arrive_expect_tx(k_full0 + 8 * st, T::KV_BYTES);
      armed_k[st] = static_cast<int>(ph);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(smem_u32(smem + T::OFF_K + st * T::KV_BYTES + c * T::CHUNK), &mapQKV,
                    k_full0 + 8 * st, colK + 64 * c, j * T::BKV, bidx);
      if (!mbar_wait(v_empty0 + 8 * st, ph ^ 1u, abort_flag, p.err, kSiteAttnProducer)) break;
      mbar_arrive_expect_tx(v_full0 + 8 * st, T::KV_BYTES);
      armed_v[st] = static_cast<int>(ph);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(smem_u32(smem + T::OFF_V + st * T::KV_BYTES + c * T::CHUNK), &mapQKV,
                    v_full0 + 8 * st, colV + 64 * c, j * T::BKV, bidx);
    }
    mbar_wait_drain(q_full, 0, p.err);
    for (int s = 0; s < T::KST; ++s) {
      if (armed_k[s] >= 0) mbar_wait_drain(k_full0 + 8 * s, static_cast<uint32_t>(armed_k[s]), p.err);
      if (armed_v[s] >= 0) mbar_wait_drain(v_full0 + 8 * s, static_cast<uint32_t>(armed_v[s]), p.err);
    }
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------- UMMA issue
    constexpr uint32_t idesc_s = idesc_bf16_f32(T::BQ, T::BKV, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(T::BQ, D, false, true);
    const uint32_t sQ = smem_u32(smem + T::OFF_Q);
    const uint32_t sP = smem_u32(smem + T::OFF_P);
    bool ok = mbar_wait(q_full, 0, abort_flag, p.err, kSiteAttnMma);
    auto issue_s = [&](int j) -> bool {
      const int st = j % T::KST;
      if (!mbar_wait(k_full0 + 8 * st, (j / T::KST) & 1, abort_flag, p.err, kSiteAttnMma))
        return false;
      tc_fence_after();
      const uint32_t sK = smem_u32(smem + T::OFF_K + st * T::KV_BYTES);
      const uint32_t d_tmem = tmem + static_cast<uint32_t>((j & 1) * T::BKV);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * T::CHUNK + (k & 3) * 32;
        umma_bf16(d_tmem, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024),
                  idesc_s, k > 0 ? 1u : 0u);
      }
      umma_commit(s_full0 + 8 * (j & 1));
      umma_commit(k_empty0 + 8 * st);
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int j = 0; j < n_kv && ok; ++j) {
      if (j + 1 < n_kv && !issue_s(j + 1)) break;
      if (!mbar_wait(p_full, j & 1, abort_flag, p.err, kSiteAttnMma)) break;
      const int st = j % T::KST;
      if (!mbar_wait(v_full0 + 8 * st, (j / T::KST) & 1, abort_flag, p.err, kSiteAttnMma)) break;
      tc_fence_after();
      const uint32_t sV = smem_u32(smem + T::OFF_V + st * T::KV_BYTES);
#pragma unroll
      for (int k = 0; k < T::BKV / 16; ++k) {
        const uint32_t offp = (k >> 2) * T::CHUNK + (k & 3) * 32;
        umma_bf16(tmem + T::TM_O, sdesc_sw128(sP + offp, 16, 1024),
                  sdesc_sw128(sV + k * 2048, T::CHUNK, 1024), idesc_o, (j | k) != 0 ? 1u : 0u);
      }
      umma_commit(pv_done);
      umma_commit(v_empty0 + 8 * st);
    }
    umma_commit(drain);
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int e = warp - 4;
    const int r = e * 32 + lane;  // query row within the block
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(e * 32) << 16);
    const float c = p.scale_log2;
    float m_run = -INFINITY;  // reference max (raw score units)
    float l = 0.f;
    bool ok = true;
    uint8_t* sP = smem + T::OFF_P;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(s_full0 + 8 * (j & 1), (j >> 1) & 1, abort_flag, p.err, kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t t_s = t_lane + static_cast<uint32_t>((j & 1) * T::BKV);
      // Key columns allowed for this row: causal diagonal block keeps keys
      // <= r; a ragged last block (non-causal) keeps keys < N.
      int lim = T::BKV;
      if (p.causal && j == iblk) lim = r + 1;
      if (!p.causal) {
        const int rem = p.N - j * T::BKV;
        if (rem < lim) lim = rem;
      }
      float mx = -INFINITY;
#pragma unroll 1
      for (int cc = 0; cc < T::BKV / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_s + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (cc * 32 + k < lim) mx = fmaxf(mx, __uint_as_float(v[k]));
      }
      float m_new = m_run;
      bool need = false;
      if (mx > m_run) {
        need = (m_run == -INFINITY) || ((mx - m_run) * c > 8.0f);
        if (need) m_new = mx;
      }
      const bool warp_need = __any_sync(0xffffffffu, need) && j > 0;
      const float alpha = need ? (m_run == -INFINITY ? 0.f : ex2_approx((m_run - m_new) * c)) : 1.f;
      const float mref = m_new * c;
      uint32_t pk[64];
      float rs = 0.f;
#pragma unroll
      for (int cc = 0; cc < T::BKV / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_s + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const float p0 = (cc * 32 + k < lim) ? ex2_approx(fmaf(__uint_as_float(v[k]), c, -mref)) : 0.f;
          const float p1 =
              (cc * 32 + k + 1 < lim) ? ex2_approx(fmaf(__uint_as_float(v[k + 1]), c, -mref)) : 0.f;
          const uint32_t packed = pack_bf16x2(p0, p1);
          pk[cc * 16 + k / 2] = packed;
          // the row sum uses the bf16-rounded weights that enter P V
          const __nv_bfloat162 pb = *reinterpret_cast<const __nv_bfloat162*>(&packed);
          rs += __bfloat162float(pb.x) + __bfloat162float(pb.y);
        }
      }
      l = alpha * l + rs;
      m_run = m_new;
      if (j > 0) {
        // P V of the previous step has finished: the P buffer is free and O
        // holds every earlier block.
        if (!mbar_wait(pv_done, (j - 1) & 1, abort_flag, p.err, kSiteAttnSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // P row r -> swizzled K-major tile: 64-key chunk kc, 16-byte unit u.
#pragma unroll
      for (int u16 = 0; u16 < 16; ++u16) {
        const int kc = u16 >> 3, u = u16 & 7;
        uint4 w = make_uint4(pk[u16 * 4 + 0], pk[u16 * 4 + 1], pk[u16 * 4 + 2], pk[u16 * 4 + 3]);
        *reinterpret_cast<uint4*>(sP + kc * T::CHUNK + r * 128 + ((u ^ (r & 7)) << 4)) = w;
      }
      if (warp_need) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_lane + T::TM_O + cc * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
          tmem_st_32x32b_x32(t_lane + T::TM_O + cc * 32, v);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(pv_done, (n_kv - 1) & 1, abort_flag, p.err, kSiteAttnSoftmax)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const long long srow = static_cast<long long>(item - p.item0) * T::BQ + r;
      __nv_bfloat16* dst = p.o + srow * p.d + head * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + T::TM_O + cc * 32, v);
        tmem_ld_wait();
        uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[q * 8 + 0]) * inv_l, __uint_as_float(v[q * 8 + 1]) * inv_l);
          w.y = pack_bf16x2(__uint_as_float(v[q * 8 + 2]) * inv_l, __uint_as_float(v[q * 8 + 3]) * inv_l);
          w.z = pack_bf16x2(__uint_as_float(v[q * 8 + 4]) * inv_l, __uint_as_float(v[q * 8 + 5]) * inv_l);
          w.w = pack_bf16x2(__uint_as_float(v[q * 8 + 6]) * inv_l, __uint_as_float(v[q * 8 + 7]) * inv_l);
          d4[q] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, T::TMEM_COLS);
}

}  // namespace bpt
