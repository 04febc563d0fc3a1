// Blockwise attention with 64-row query blocks (b = 64): each K/V tile
// brought in serves 64 query rows ("Blockwise Parallel Transformer — BPT",
// section "Choosing the block size: arithmetic intensity": the FLOPs done per
// byte re-read equal the block's row count).  The point of the block-size
// series below the default b = 256 and b = 128.
//
// One CTA per (64-row query block, head); two CTAs fit one SM (256 TMEM
// columns and about 100 KB of shared memory each), so one CTA's softmax
// overlaps the other's products on the SM's tensor core.  Per key block j
// (128 keys), with the online-softmax state of the pair kernel:
//
//   S = Q K_j^T      UMMA M = 64 (SS): the accumulator fills TMEM lanes
//                    0..15 of each 32-lane quarter (row 16 q + i at lane
//                    32 q + i), 128 fp32 columns
//   P = exp2(...)    softmax warp q, lanes 0..15 (lanes 16..31 hold nothing);
//                    P in fp16 into shared memory, 128-byte swizzled K-major
//   O += P V_j       UMMA M = 64 (SS), O in TMEM columns 128..
//
// P lives in shared memory, so S_j+1 is issued as soon as the softmax warps
// have read S_j (before their exponentials), and P_j+1 waits only for PV_j.
// The softmax arithmetic (lazy reference maximum, MUFU / FMA-pipe exp2
// groups, partial sums, rescale) is that of attn_pair_tc_kernel, so a query
// row gets bitwise the output of the b = 128 / 256 kernels.
//
// Warp roles (256 threads): 0 TMA, 1 UMMA issue, 2 TMEM owner, 3 idle,
// 4..7 softmax.  Every wait is bounded.
#pragma once

#include "attn_pair_tc.cuh"

namespace bpt {

template <int D>
struct AttnB64Cfg {
  static constexpr int BQ = 64;
  static constexpr int BKV = 128;
  static constexpr int QTILE = 64 * D * 2;    // [D/64][64 rows][64]
  static constexpr int QCHUNK = 64 * 128;     // 8 KB: one 64-column chunk of Q or P
  static constexpr int KTILE = 128 * D * 2;   // [D/64][128 rows][64]
  static constexpr int KCHUNK = 128 * 128;    // 16 KB
  static constexpr int NSLOT = D == 128 ? 2 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = QTILE;         // [2][64 rows][64 keys]
  static constexpr int OFF_RING = OFF_P + 2 * QCHUNK;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * KTILE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t TM_O = 128;
};

template <int D, int EMU>
__global__ void __launch_bounds__(256, 2)
    attn_b64_tc_kernel(const __grid_constant__ CUtensorMap mapQ64,
                       const __grid_constant__ CUtensorMap mapQKV, const AttnPairParams p) {
  using C = AttnB64Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t ring_full0 = smem_u32(bars + 1);
  const uint32_t ring_empty0 = smem_u32(bars + 1 + C::NSLOT);
  const uint32_t s_full = smem_u32(bars + 1 + 2 * C::NSLOT);   // S_j landed
  const uint32_t s_read = smem_u32(bars + 2 + 2 * C::NSLOT);   // softmax read S_j (4 warps)
  const uint32_t p_ready = smem_u32(bars + 3 + 2 * C::NSLOT);  // P_j stored (4 warps)
  const uint32_t pv_done = smem_u32(bars + 4 + 2 * C::NSLOT);  // PV_j complete
  const uint32_t drain = smem_u32(bars + 5 + 2 * C::NSLOT);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx -> (head group, work rank, head) as in the pair kernel; a rank
  // is one 64-row block, longest first under a causal mask
  const int per_group = int(gridDim.x / p.h) * p.hg;
  const int grp = blockIdx.x / per_group;
  const int in_grp = blockIdx.x - grp * per_group;
  const int rank = in_grp / p.hg;
  const int head = grp * p.hg + (in_grp - rank * p.hg);
  int item, half;
  if (p.seqs == 0) {
    const int q = p.causal ? (2 * p.count - 1 - rank) : rank;
    item = p.item0 + (q >> 1);
    half = q & 1;
  } else {
    int s, q;
    if (p.causal) {
      q = 2 * p.nb - 1 - rank / p.seqs;
      s = rank % p.seqs;
    } else {
      s = rank / (2 * p.nb);
      q = rank % (2 * p.nb);
    }
    item = p.item0 + s * p.nb + (q >> 1);
    half = q & 1;
  }
  const int bidx = item / p.nb;
  const int i128 = item - bidx * p.nb;           // the 128-row block
  const int row0 = i128 * C::BKV + half * C::BQ;  // first query row in the sequence
  if (row0 >= p.N) return;                       // a ragged tail's empty half
  const int n_kv = p.causal ? i128 + 1 : p.nb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(ring_full0 + 8 * s, 1);
      mbar_init(ring_empty0 + 8 * s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 4);
    mbar_init(p_ready, 4);
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&tmem_base_sh), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;
  const int colQ = head * D, colK = p.d + head * D, colV = 2 * p.d + head * D;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&mapQ64);
      tma_prefetch_desc(&mapQKV);
      mbar_arrive_expect_tx(q_full, C::QTILE);
      tma_load_4d(smem_u32(smem + C::OFF_Q), &mapQ64, q_full, 0, row0, colQ / 64, bidx);
    }
    int armed[C::NSLOT];
    for (int s = 0; s < C::NSLOT; ++s) armed[s] = -1;
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      for (int w = 0; w < 2; ++w) {
        if (!mbar_wait_warp(ring_empty0 + 8 * slot, phase ^ 1u, abort_flag, p.err,
                            kSiteAttnProducer)) {
          ok = false;
          break;
        }
        // test hook 2: CTA 0 never loads V_0 (a lost arrive)
        const bool lost = p.fault == 2 && blockIdx.x == 0 && j == 0 && w == 1;
        if (!lost) {
          armed[slot] = static_cast<int>(phase);
          if (leader) {
            mbar_arrive_expect_tx(ring_full0 + 8 * slot, C::KTILE);
            tma_load_4d(smem_u32(smem + C::OFF_RING + slot * C::KTILE), &mapQKV,
                        ring_full0 + 8 * slot, 0, j * C::BKV, (w == 0 ? colK : colV) / 64, bidx);
          }
        }
        __syncwarp();
        if (++slot == C::NSLOT) {
          slot = 0;
          phase ^= 1u;
        }
      }
    }
    mbar_wait_drain(q_full, 0, p.err);
    for (int s = 0; s < C::NSLOT; ++s)
      if (armed[s] >= 0) mbar_wait_drain(ring_full0 + 8 * s, static_cast<uint32_t>(armed[s]), p.err);
  } else if (warp == 1) {
    // ----------------------------------------------------------- UMMA issue
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_f16_f32(C::BQ, C::BKV, false, false);
    constexpr uint32_t idesc_o = idesc_f16_f32(C::BQ, D, false, true);
    constexpr uint32_t hi = sdesc_hi(1024);
    const uint32_t q_lo = sdesc_lo(smem_u32(smem + C::OFF_Q), 16);
    const uint32_t p_lo = sdesc_lo(smem_u32(smem + C::OFF_P), 16);
    const uint32_t ring = smem_u32(smem + C::OFF_RING);
    auto slot_of = [&](int t) { return t % C::NSLOT; };
    auto phase_of = [&](int t) { return static_cast<uint32_t>((t / C::NSLOT) & 1); };
    auto commit = [&](uint32_t bar) {
      if (leader) umma_commit(bar);
      __syncwarp();
    };
    // S into TMEM columns 0..127: K-major Q (8 KB chunks) and K (16 KB chunks)
    auto issue_s = [&](int tk) {
      const uint32_t k_lo = sdesc_lo(ring + slot_of(tk) * C::KTILE, 16);
      if (leader) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          umma_ss(tmem, q_lo + (((k >> 2) * C::QCHUNK + (k & 3) * 32) >> 4), hi,
                  k_lo + (((k >> 2) * C::KCHUNK + (k & 3) * 32) >> 4), hi, idesc_s,
                  k > 0 ? 1u : 0u);
      }
      __syncwarp();
    };
    bool ok = mbar_wait_warp(q_full, 0, abort_flag, p.err, kSiteAttnMma) &&
              mbar_wait_warp(ring_full0 + 8 * slot_of(0), phase_of(0), abort_flag, p.err,
                             kSiteAttnMma);
    if (ok) {
      tc_fence_after();
      issue_s(0);
      commit(s_full);
      commit(ring_empty0 + 8 * slot_of(0));
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      const int tv = 2 * j + 1, tk = 2 * j + 2;
      // S_j+1 as soon as S_j has been read (P goes to shared memory)
      if (!mbar_wait_warp(s_read, static_cast<uint32_t>(j & 1), abort_flag, p.err, kSiteAttnMma))
        break;
      if (j + 1 < n_kv) {
        if (!mbar_wait_warp(ring_full0 + 8 * slot_of(tk), phase_of(tk), abort_flag, p.err,
                            kSiteAttnMma))
          break;
        tc_fence_after();
        issue_s(tk);
        commit(s_full);
        commit(ring_empty0 + 8 * slot_of(tk));
      }
      // PV_j once P_j is stored and V_j has landed
      if (!mbar_wait_warp(p_ready, static_cast<uint32_t>(j & 1), abort_flag, p.err,
                          kSiteAttnMma) ||
          !mbar_wait_warp(ring_full0 + 8 * slot_of(tv), phase_of(tv), abort_flag, p.err,
                          kSiteAttnMma))
        break;
      tc_fence_after();
      const uint32_t v_lo = sdesc_lo(ring + slot_of(tv) * C::KTILE, C::KCHUNK);
      if (leader) {
#pragma unroll
        for (int k = 0; k < C::BKV / 16; ++k)
          umma_ss(tmem + C::TM_O, p_lo + (((k >> 2) * C::QCHUNK + (k & 3) * 32) >> 4), hi,
                  v_lo + ((k * 2048) >> 4), hi, idesc_o, (j > 0 || k > 0) ? 1u : 0u);
      }
      __syncwarp();
      commit(pv_done);
      commit(ring_empty0 + 8 * slot_of(tv));
    }
    commit(drain);
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int e = warp & 3;            // TMEM lane quarter: rows 16 e .. 16 e + 15
    const bool own = lane < 16;        // lanes 16..31 read TMEM lanes no row uses
    const int r = e * 16 + (lane & 15);  // query row within the block
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(e * 32) << 16);
    const uint32_t tS = t_lane, tO = t_lane + C::TM_O;
    const float c = p.scale_log2;
    const bool ragged = (p.N % C::BKV) != 0;
    const int qpos = row0 + r;         // query position in the sequence
    float m_run = -INFINITY, m_true = -INFINITY, l = 0.f;
    bool o_live = false;
    uint8_t* prow = smem + C::OFF_P + r * 128;  // this row's 128-byte line in each chunk
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      if (!mbar_wait_fast(s_full, static_cast<uint32_t>(j & 1), abort_flag, p.err,
                          kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool masked = p.causal ? (j == i128) : (ragged && j == p.nb - 1);
      const int lim = !masked ? C::BKV : (p.causal ? qpos - j * C::BKV + 1 : p.N - j * C::BKV);
      // pass 1: the row maximum, 64 columns at a time (two CTAs share an SM:
      // 128 registers per thread).  max is exact, so the order of the partial
      // maxima does not matter.
      float mxp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mxp[k] = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t sr[64];
        tmem_ld_32x32b_x32(tS + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld_32x32b_x32(tS + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        if (masked) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (hh * 64 + k >= lim) sr[k] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int k = 0; k < 64; k += 16)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            mxp[q] = max3f(mxp[q], __uint_as_float(sr[k + q]), __uint_as_float(sr[k + 8 + q]));
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) mxp[k] = fmaxf(mxp[k], mxp[k + 4]);
      const float mx = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3]));
      m_true = fmaxf(m_true, mx);
      float m_new = m_run;
      bool need = false;
      if (mx > m_run) {
        need = (m_run == -INFINITY) || ((mx - m_run) * c > 8.0f);
        if (need) m_new = mx;
      }
      const float alpha =
          need ? (m_run == -INFINITY ? 0.f : ex2_approx((m_run - m_new) * c)) : 1.f;
      // PV_j-1 must be complete: P and O are reused
      if (j > 0 && !mbar_wait_fast(pv_done, static_cast<uint32_t>((j - 1) & 1), abort_flag,
                                   p.err, kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool warp_need = __any_sync(0xffffffffu, need && own) && o_live;
      if (warp_need) {
#pragma unroll 1
        for (int cc = 0; cc < D / 8; ++cc) {
          uint32_t v[8];
          tmem_ld_32x32b_x8(tO + cc * 8, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
          tmem_st_32x32b_x8(tO + cc * 8, v);
        }
        tmem_st_wait();
      }
      const float2 cc2 = make_float2(c, c);
      const float2 mref2 = make_float2(-m_new * c, -m_new * c);
      float2 sum2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
      // pass 2: exponentials, 64 columns at a time, in column order (the
      // partial sums see the columns in the order of the pair kernel)
      auto exp_half = [&](auto emu_mask, int hh) {
        constexpr uint32_t kMask = decltype(emu_mask)::value;
        uint32_t sr[64];
        tmem_ld_32x32b_x32(tS + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld_32x32b_x32(tS + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        if (hh == 1) {  // S_j is read in full: S_j+1 may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_read);
        }
        if (masked) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (hh * 64 + k >= lim) sr[k] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // 16-byte units of 8 keys
          uint32_t pk[4];
#pragma unroll
          for (int k = 0; k < 8; k += 2) {
            const int col = hh * 64 + u * 8 + k;
            float2 a = __ffma2_rn(make_float2(__uint_as_float(sr[u * 8 + k]),
                                              __uint_as_float(sr[u * 8 + k + 1])),
                                  cc2, mref2);
            float2 e2;
            if ((kMask >> (col >> 4)) & 1u) {
              e2 = exp2_poly2(a);
            } else {
              e2.x = ex2_approx(a.x);
              e2.y = ex2_approx(a.y);
            }
            sum2[(col >> 1) & 3] = __fadd2_rn(sum2[(col >> 1) & 3], e2);
            pk[k >> 1] = pack_f16x2(e2.x, e2.y);
          }
          // K-major P, 128-byte swizzle: unit u of row r in chunk hh at the
          // 16-byte slot u ^ (r % 8)
          if (own)
            *reinterpret_cast<uint4*>(prow + hh * C::QCHUNK + ((u ^ (r & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      };
      for (int hh = 0; hh < 2; ++hh) {
        if (masked || emu_group_mask(EMU) == 0u)
          exp_half(std::integral_constant<uint32_t, 0u>{}, hh);
        else
          exp_half(std::integral_constant<uint32_t, emu_group_mask(EMU)>{}, hh);
      }
      fence_proxy_async_smem();  // P is read by the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready);
      sum2[0] = __fadd2_rn(__fadd2_rn(sum2[0], sum2[1]), __fadd2_rn(sum2[2], sum2[3]));
      l = alpha * l + (sum2[0].x + sum2[0].y);
      m_run = m_new;
      o_live = true;
    }
    if (ok && mbar_wait_fast(pv_done, static_cast<uint32_t>((n_kv - 1) & 1), abort_flag, p.err,
                             kSiteAttnSoftmax)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool valid = own && qpos < p.N;
      if (p.stats != nullptr && valid) {
        const float m_s = m_true * p.scale_log2 * 0.69314718055994531f;
        const float l_s = l * ex2_approx((m_run - m_true) * p.scale_log2);
        p.stats[(static_cast<long long>(bidx) * p.h + head) * p.N + qpos] = make_float2(m_s, l_s);
      }
      const long long orow = p.o_tok ? static_cast<long long>(bidx) * p.N + qpos
                                     : static_cast<long long>(item - p.item0) * C::BKV +
                                           half * C::BQ + r;
      __half* dst = p.o + orow * p.o_ld + head * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tO + cc * 32, v);
        tmem_ld_wait();
        if (!valid) continue;
        uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_f16x2(__uint_as_float(v[q * 8 + 0]) * inv_l, __uint_as_float(v[q * 8 + 1]) * inv_l);
          w.y = pack_f16x2(__uint_as_float(v[q * 8 + 2]) * inv_l, __uint_as_float(v[q * 8 + 3]) * inv_l);
          w.z = pack_f16x2(__uint_as_float(v[q * 8 + 4]) * inv_l, __uint_as_float(v[q * 8 + 5]) * inv_l);
          w.w = pack_f16x2(__uint_as_float(v[q * 8 + 6]) * inv_l, __uint_as_float(v[q * 8 + 7]) * inv_l);
          d4[q] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace bpt
