// Block-sparse gated attention ("Block Sparse Flash Attention", sections
// "Methodology and Mechanism" and "Gating Mechanism and Threshold
// Calibration"), two query blocks per CTA, with the scores S and the
// probabilities P kept apart.
//
// The gate needs each block's exact scores: S_X(j) is computed, its block
// maximum over the tile's valid rows is compared with the threshold, and a
// pruned block contributes nothing (no exponentials, no PV, no change to the
// row statistics; its V tile is not loaded when every tile that visits the
// block prunes it).  In attn_pair_tc_kernel<..., GATE> P is written over S in
// TMEM, so the next block's scores can only be computed once the tile's
// decision is known and, for a kept block, its PV has read P: a pruned block
// still costs the whole chain (scores, maximum, exchange, hand-over, next
// scores).  Here P has its own storage (d_k = 64: TMEM columns 384..511;
// d_k = 128: shared memory, K-major, 128-byte swizzled, PV reading both
// operands from shared memory, K/V ring of three slots), so S_X(j+1) is
// issued as soon as the tile's softmax warps have read S_X(j), while they
// take its maximum and the decision.  A kept block then runs the online
// softmax of attn_pair_tc_kernel (same arithmetic: bitwise the same result
// when every block is kept); the softmax of block j+1 waits for PV_X(j) only
// before its first P store.
//
// Ring order K_0 K_1 K_2 V_0 K_3 V_1 ... V_n-1: K two blocks ahead of V, and
// V_j issued once the tiles that visit block j have decided (at once if tile
// A keeps it; completed without a load if every visiting tile prunes it).
//
// Warp roles (384 threads): 0 TMA, 1 UMMA issue, 2 TMEM owner, 3 idle,
// 4..7 softmax of tile A, 8..11 of tile B.  Every wait is bounded.
#pragma once

#include "attn_pair_tc.cuh"

namespace bpt {

template <int D>
struct AttnGateCfg {
  static constexpr int BQ = 128;
  static constexpr int BKV = 128;
  static constexpr int TILE = 128 * D * 2;    // one Q, K or V tile
  static constexpr int CHUNK = 128 * 128;     // one 64-column swizzled chunk (16 KB)
  static constexpr bool P_SMEM = D == 128;
  static constexpr int PTILE = P_SMEM ? 128 * 128 * 2 : 0;  // P of one tile, fp16
  static constexpr int NSLOT = D == 128 ? 3 : 10;
  static constexpr int OFF_QA = 0;
  static constexpr int OFF_QB = TILE;
  static constexpr int OFF_P = 2 * TILE;      // [A, B] (d_k = 128)
  static constexpr int OFF_RING = OFF_P + 2 * PTILE;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * TILE;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S_B = 128;
  static constexpr uint32_t TM_O_A = 256;
  static constexpr uint32_t TM_O_B = 256 + D;
  static constexpr uint32_t TM_P_A = 384;     // d_k = 64
  static constexpr uint32_t TM_P_B = 448;
};
static_assert(AttnGateCfg<128>::SMEM <= 232448, "d_k = 128 shared memory");
static_assert(AttnGateCfg<64>::SMEM <= 232448, "d_k = 64 shared memory");

template <int D, int EMU>
__global__ void __launch_bounds__(384, 1)
    attn_gate_tc_kernel(const __grid_constant__ CUtensorMap mapQKV, const AttnPairParams p) {
  using C = AttnGateCfg<D>;
  constexpr int kHand = fwd_handovers<D>();      // P hand-overs per 128-key tile
  constexpr int kChunksPerHand = 4 / kHand;      // 32-key chunks per hand-over
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t ring_full0 = smem_u32(bars + 1);
  const uint32_t ring_empty0 = smem_u32(bars + 1 + C::NSLOT);
  const uint32_t s_full0 = smem_u32(bars + 1 + 2 * C::NSLOT);   // [A, B]: S_X(j) landed
  const uint32_t s_read0 = smem_u32(bars + 3 + 2 * C::NSLOT);   // [A, B]: S_X(j) read (4 warps)
  const uint32_t pv_done0 = smem_u32(bars + 5 + 2 * C::NSLOT);  // [A, B]: block j finished
  // [A: hand-overs 0..3, B: 0..3]: P keys of the hand-over stored (4 warps);
  // the first also carries the tile's decision
  const uint32_t p_ready0 = smem_u32(bars + 7 + 2 * C::NSLOT);
  const uint32_t drain = smem_u32(bars + 15 + 2 * C::NSLOT);
  const uint32_t gate_x0 = smem_u32(bars + 16 + 2 * C::NSLOT);  // [A, B], count 4
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  // per tile, block parity and softmax warp: the maximum of its rows; the
  // tile's four warps exchange them on gate_x (one phase per block)
  __shared__ float gate_slot[2][2][4];
  // per tile, the decisions of the last four blocks as ((j + 1) << 1) | keep,
  // read by the producer (V loads) and the UMMA warp (PV or not)
  __shared__ int gate_dec[2][4];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int itemA, head;
  bool has_b;
  {
    const int per_group = int(gridDim.x / p.h) * p.hg;
    const int grp = blockIdx.x / per_group;
    const int in_grp = blockIdx.x - grp * per_group;
    const int rank = in_grp / p.hg;
    head = grp * p.hg + (in_grp - rank * p.hg);
    attn_pair_decode(p, rank, itemA, has_b);
  }
  const int bidx = itemA / p.nb;
  const int iA = itemA - bidx * p.nb;
  const int iB = iA + 1;
  const int nA = p.causal ? iA + 1 : p.nb;
  const int nB = has_b ? (p.causal ? iB + 1 : p.nb) : 0;
  const int n_kv = nA > nB ? nA : nB;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(ring_full0 + 8 * s, 1);
      mbar_init(ring_empty0 + 8 * s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full0 + 8 * x, 1);
      mbar_init(s_read0 + 8 * x, 4);
      mbar_init(pv_done0 + 8 * x, 1);
      for (int c = 0; c < 4; ++c) mbar_init(p_ready0 + 8 * (4 * x + c), 4);
    }
    mbar_init(drain, 1);
    mbar_init(gate_x0, 4);
    mbar_init(gate_x0 + 8, 4);
    for (int i = 0; i < 8; ++i) (&gate_dec[0][0])[i] = 0;
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
  // Ring order K_0 K_1, then per block j: K_j+2 (if any), V_j.  K runs two
  // blocks ahead, so the decision V_j waits for delays K_j+3, not the K the
  // next-but-one score product needs.  Positions of K_m and V_j:
  auto pos_k = [&](int m) { return m <= 1 ? m : 2 * m - 2; };
  auto pos_v = [&](int j) {
    return n_kv == 1 ? 1 : 2 + j + max(0, min(j + 2, n_kv - 1) - 1);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&mapQKV);
      mbar_arrive_expect_tx(q_full, C::TILE * (has_b ? 2 : 1));
      tma_load_4d(smem_u32(smem + C::OFF_QA), &mapQKV, q_full, 0, iA * C::BQ, colQ / 64, bidx);
      if (has_b)
        tma_load_4d(smem_u32(smem + C::OFF_QB), &mapQKV, q_full, 0, iB * C::BQ, colQ / 64, bidx);
    }
    int armed[C::NSLOT];
    for (int s = 0; s < C::NSLOT; ++s) armed[s] = -1;
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    // the order as a sequence: K_0, K_1, then (K_j+2,) V_j for j = 0, 1, ...
    int jv = 0;          // next V block
    int kn = 0;          // next K block
    bool k_turn = true;  // after K_0 K_1: a K_j+2 (if any) before each V_j
    for (int t = 0; t < 2 * n_kv && ok; ++t) {
      int j, w;  // key block, 0 = K / 1 = V
      if (kn < 2 && kn < n_kv) {
        j = kn++;
        w = 0;
      } else if (k_turn && kn < n_kv && kn == jv + 2) {
        j = kn++;
        w = 0;
        k_turn = false;
      } else {
        j = jv++;
        w = 1;
        k_turn = true;
      }
      if (!mbar_wait_warp(ring_empty0 + 8 * slot, phase ^ 1u, abort_flag, p.err,
                          kSiteAttnProducer)) {
        ok = false;
        break;
      }
      bool load = true;
      if (w == 1) {
        // wait (bounded) for the decisions of the tiles that visit block j
        const bool needA = j < nA, needB = j < nB;
        const int tag = (j + 1) << 1;
        bool seen = false;
        const uint64_t g0 = global_ns();
        for (uint32_t it = 0;; ++it) {
          const int da = *reinterpret_cast<volatile int*>(&gate_dec[0][j & 3]);
          const int db = *reinterpret_cast<volatile int*>(&gate_dec[1][j & 3]);
          const bool haveA = !needA || (da & ~1) == tag;
          const bool haveB = !needB || (db & ~1) == tag;
          const bool keepA = needA && da == (tag | 1);
          const bool keepB = needB && db == (tag | 1);
          if (keepA || (haveA && haveB)) {
            load = keepA || keepB;
            seen = true;
            break;
          }
          if ((it & 63u) == 63u) {
            if (*abort_flag) break;
            if (global_ns() - g0 > BPT_WAIT_LIMIT_NS) {
              record_error(p.err, kErrTimeout, kSiteAttnProducer);
              *abort_flag = 1;
              break;
            }
          }
        }
        if (!__all_sync(0xffffffffu, seen)) {
          ok = false;
          break;
        }
      }
      const uint32_t fb = ring_full0 + 8 * slot;
      armed[slot] = static_cast<int>(phase);
      if (leader) {
        if (!load) {
          mbar_arrive_expect_tx(fb, 0);  // V_j not needed: the slot completes empty
        } else {
          mbar_arrive_expect_tx(fb, C::TILE);
          tma_load_4d(smem_u32(smem + C::OFF_RING + slot * C::TILE), &mapQKV, fb, 0,
                      j * C::BKV, (w == 0 ? colK : colV) / 64, bidx);
        }
      }
      __syncwarp();
      if (++slot == C::NSLOT) {
        slot = 0;
        phase ^= 1u;
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
    const uint32_t ring = smem_u32(smem + C::OFF_RING);
    const uint32_t q_lo[2] = {sdesc_lo(smem_u32(smem + C::OFF_QA), 16),
                              sdesc_lo(smem_u32(smem + C::OFF_QB), 16)};
    auto slot_of = [&](int t) { return t % C::NSLOT; };
    auto phase_of = [&](int t) { return static_cast<uint32_t>((t / C::NSLOT) & 1); };
    auto wait_full = [&](int t) {
      return mbar_wait_warp(ring_full0 + 8 * slot_of(t), phase_of(t), abort_flag, p.err,
                            kSiteAttnMma);
    };
    auto issue_s = [&](int x, uint32_t k_lo) {
      if (leader) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::CHUNK + (k & 3) * 32) >> 4;
          umma_ss(tmem + (x == 0 ? 0u : C::TM_S_B), q_lo[x] + off, hi, k_lo + off, hi, idesc_s,
                  k > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    auto issue_pv_chunk = [&](int x, uint32_t v_lo, int c, bool first) {
      if (leader) {
        const uint32_t d_tmem = tmem + (x == 0 ? C::TM_O_A : C::TM_O_B);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int k = 2 * c + kk;
          const uint32_t acc = (!first || k > 0) ? 1u : 0u;
          if constexpr (C::P_SMEM) {
            const uint32_t p_lo =
                sdesc_lo(smem_u32(smem + C::OFF_P + x * C::PTILE), 16) +
                (((k >> 2) * C::CHUNK + (k & 3) * 32) >> 4);
            umma_ss(d_tmem, p_lo, hi, v_lo + ((k * 2048) >> 4), hi, idesc_o, acc);
          } else {
            const uint32_t tP = tmem + (x == 0 ? C::TM_P_A : C::TM_P_B);
            umma_ts(d_tmem, tP + 8 * k, v_lo + ((k * 2048) >> 4), hi, idesc_o, acc);
          }
        }
      }
      __syncwarp();
    };
    auto commit = [&](uint32_t bar) {
      if (leader) umma_commit(bar);
      __syncwarp();
    };
    const int nX[2] = {nA, nB};
    uint32_t sph[2] = {0, 0};  // s_read phases
    uint32_t pph[2] = {0, 0};  // p_ready phases
    bool o_started[2] = {false, false};  // first kept PV of a tile overwrites O
    bool ok = mbar_wait_warp(q_full, 0, abort_flag, p.err, kSiteAttnMma) && wait_full(0);
    if (ok) {
      tc_fence_after();
      const uint32_t k0_lo = sdesc_lo(ring + slot_of(0) * C::TILE, 16);
      for (int x = 0; x < 2; ++x)
        if (nX[x] > 0) {
          issue_s(x, k0_lo);
          commit(s_full0 + 8 * x);
        }
      commit(ring_empty0 + 8 * slot_of(0));
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      const int tk = pos_k(j + 1), tv = pos_v(j);
      // S_X(j+1) once tile X has read S_X(j)
      if (j + 1 < n_kv) {
        if (!wait_full(tk)) break;
        const uint32_t k_lo = sdesc_lo(ring + slot_of(tk) * C::TILE, 16);
        for (int x = 0; x < 2 && ok; ++x) {
          if (j + 1 >= nX[x]) continue;
          if (!mbar_wait_warp(s_read0 + 8 * x, sph[x], abort_flag, p.err, kSiteAttnMma)) {
            ok = false;
            break;
          }
          sph[x] ^= 1u;
          tc_fence_after();
          issue_s(x, k_lo);
          commit(s_full0 + 8 * x);
        }
        if (!ok) break;
        commit(ring_empty0 + 8 * slot_of(tk));
      }
      // PV_X(j) for a kept block as its hand-overs come; a pruned block
      // hands everything over at once (its first hand-over carries the
      // decision; the skipped phases complete regardless)
      bool v_ready = false;
      for (int x = 0; x < 2 && ok; ++x) {
        if (j >= nX[x]) continue;
        const uint32_t pr = p_ready0 + 8 * (4 * x);
        bool kept = true;
        for (int hh = 0; hh < kHand; ++hh) {
          if (hh > 0 && !kept) break;
          if (!mbar_wait_warp(pr + 8 * hh, pph[x], abort_flag, p.err, kSiteAttnMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // the decision of block j (the softmax may already be deciding
          // block j+1: S_X(j+1) went out before this hand-over)
          if (hh == 0) kept = (*reinterpret_cast<volatile int*>(&gate_dec[x][j & 3]) & 1) != 0;
          if (!kept) break;
          if (!v_ready) {
            if (!wait_full(tv)) {
              ok = false;
              break;
            }
            v_ready = true;
          }
          const uint32_t v_lo = sdesc_lo(ring + slot_of(tv) * C::TILE, C::CHUNK);
          for (int q = 0; q < kChunksPerHand; ++q)
            issue_pv_chunk(x, v_lo, hh * kChunksPerHand + q, !o_started[x]);
        }
        if (!ok) break;
        pph[x] ^= 1u;
        if (kept) o_started[x] = true;
        commit(pv_done0 + 8 * x);  // block j of tile X finished (kept or not)
      }
      if (!ok) break;
      // the slot of V_j: completed (loaded or empty) once both tiles decided
      if (!v_ready && !wait_full(tv)) break;
      commit(ring_empty0 + 8 * slot_of(tv));
    }
    commit(drain);
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int x = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const int e = warp & 3;         // TMEM lane quarter
    const int r = e * 32 + lane;    // query row within the tile
    const int nXs = x == 0 ? nA : nB;
    const int iX = x == 0 ? iA : iB;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(e * 32) << 16);
    const uint32_t tS = t_lane + (x == 0 ? 0u : C::TM_S_B);
    const uint32_t tO = t_lane + (x == 0 ? C::TM_O_A : C::TM_O_B);
    const uint32_t tP = t_lane + (x == 0 ? C::TM_P_A : C::TM_P_B);  // d_k = 64
    const uint32_t prow = smem_u32(smem + C::OFF_P + x * C::PTILE + r * 128);  // d_k = 128
    const uint32_t rsw = static_cast<uint32_t>(r & 7) << 4;
    const uint32_t s_full = s_full0 + 8 * x, s_read = s_read0 + 8 * x;
    const uint32_t pv_done = pv_done0 + 8 * x, p_ready = p_ready0 + 8 * (4 * x);
    const float c = p.scale_log2;
    const bool ragged = (p.N % C::BKV) != 0;
    const float t_thr = nXs > 0 ? p.gate_t[head * p.nb + iX] : 0.f;
    float m_run = -INFINITY, m_true = -INFINITY, l = 0.f;
    bool o_live = false;
    bool ok = nXs > 0;
    for (int j = 0; j < nXs && ok; ++j) {
      if (!mbar_wait_fast(s_full, j & 1, abort_flag, p.err, kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[C::BKV];
#pragma unroll
      for (int cc = 0; cc < C::BKV / 32; ++cc)
        tmem_ld_32x32b_x32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[cc * 32]));
      tmem_ld_wait();
      // S_X(j) is in registers: S_X(j+1) may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_read);
      const bool masked = p.causal ? (j == iX) : (ragged && j == p.nb - 1);
      if (masked) {
        const int lim = p.causal ? r + 1 : p.N - j * C::BKV;
#pragma unroll
        for (int k = 0; k < C::BKV; ++k)
          if (k >= lim) sr[k] = __float_as_uint(-INFINITY);
      }
      float mxp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mxp[k] = -INFINITY;
#pragma unroll
      for (int k = 0; k < C::BKV; k += 16)
#pragma unroll
        for (int q = 0; q < 8; ++q)
          mxp[q] = max3f(mxp[q], __uint_as_float(sr[k + q]), __uint_as_float(sr[k + 8 + q]));
#pragma unroll
      for (int k = 0; k < 4; ++k) mxp[k] = fmaxf(mxp[k], mxp[k + 4]);
      const float mx = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3]));
      // block maximum over the tile's valid query rows, in units of s: each
      // warp publishes its rows' maximum, the four meet on gate_x (a warp is
      // at most one block ahead of the others: the slots alternate by block)
      float wm = (iX * C::BQ + r < p.N) ? mx : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
      if (lane == 0) {
        gate_slot[x][j & 1][e] = wm;
        mbar_arrive(gate_x0 + 8 * x);
      }
      if (!mbar_wait_warp(gate_x0 + 8 * x, static_cast<uint32_t>(j & 1), abort_flag, p.err,
                          kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      const float bmax = fmaxf(fmaxf(gate_slot[x][j & 1][0], gate_slot[x][j & 1][1]),
                               fmaxf(gate_slot[x][j & 1][2], gate_slot[x][j & 1][3]));
      const float smax = bmax * (p.scale_log2 * 0.69314718055994531f);
      const bool keep_blk = (j == iX) || (smax >= t_thr);
      if (e == 0 && lane == 0) {
        *reinterpret_cast<volatile int*>(&gate_dec[x][j & 3]) =
            ((j + 1) << 1) | (keep_blk ? 1 : 0);
        const long long o = ((static_cast<long long>(bidx) * p.h + head) * p.nb + iX) * p.nb + j;
        if (p.gate_bmax != nullptr) p.gate_bmax[o] = smax;
        if (p.gate_kept != nullptr) p.gate_kept[o] = keep_blk ? 1 : 0;
      }
      // block j-1 finished (its PV read P, or it was pruned): P and O free
      if (j > 0 && !mbar_wait_inline(pv_done, static_cast<uint32_t>((j - 1) & 1), abort_flag,
                                     p.err, kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (!keep_blk) {
        // pruned: the hand-overs carry only the decision (written above,
        // before the first arrive)
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
          for (int hh = 0; hh < kHand; ++hh) mbar_arrive(p_ready + 8 * hh);
        continue;
      }
      m_true = fmaxf(m_true, mx);
      float m_new = m_run;
      bool need = false;
      if (mx > m_run) {
        need = (m_run == -INFINITY) || ((mx - m_run) * c > 8.0f);
        if (need) m_new = mx;
      }
      const bool warp_need = __any_sync(0xffffffffu, need) && o_live;
      const float alpha =
          need ? (m_run == -INFINITY ? 0.f : ex2_approx((m_run - m_new) * c)) : 1.f;
      if (warp_need) {
#pragma unroll 1
        for (int q = 0; q < D / 8; ++q) {
          uint32_t v[8];
          tmem_ld_32x32b_x8(tO + q * 8, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
          tmem_st_32x32b_x8(tO + q * 8, v);
        }
        tmem_st_wait();  // O is final before PV_X(j) accumulates into it
      }
      const float2 cc2 = make_float2(c, c);
      const float2 mref2 = make_float2(-m_new * c, -m_new * c);
      float2 sum2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
      auto exp_row = [&](auto emu_mask) {
        constexpr uint32_t kMask = decltype(emu_mask)::value;
#pragma unroll
        for (int cc = 0; cc < C::BKV / 32; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const int col = cc * 32 + k;
            float2 a = __ffma2_rn(
                make_float2(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])), cc2, mref2);
            float2 e2;
            if ((kMask >> (col >> 4)) & 1u) {
              e2 = exp2_poly2(a);
            } else {
              e2.x = ex2_approx(a.x);
              e2.y = ex2_approx(a.y);
            }
            sum2[(k >> 1) & 3] = __fadd2_rn(sum2[(k >> 1) & 3], e2);
            pk[k >> 1] = pack_f16x2(e2.x, e2.y);
          }
          if constexpr (C::P_SMEM) {
            // keys 32 cc .. : chunk cc / 2, 16-byte units u = 4 (cc % 2) + q at
            // their swizzled slots u ^ (r % 8)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_shared_v4(((prow + (cc >> 1) * C::CHUNK + (((cc & 1) * 4 + q) << 4)) ^ rsw),
                           pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          } else {
            tmem_st_32x32b_x16(tP + cc * 16, pk);
          }
          if ((cc + 1) % kChunksPerHand == 0) {
            if constexpr (C::P_SMEM)
              fence_proxy_async_smem();  // P is read by the tensor core
            else
              tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_ready + 8 * (cc / kChunksPerHand));
          }
        }
      };
      if (masked || emu_group_mask(EMU) == 0u)
        exp_row(std::integral_constant<uint32_t, 0u>{});
      else
        exp_row(std::integral_constant<uint32_t, emu_group_mask(EMU)>{});
      sum2[0] = __fadd2_rn(__fadd2_rn(sum2[0], sum2[1]), __fadd2_rn(sum2[2], sum2[3]));
      l = alpha * l + (sum2[0].x + sum2[0].y);
      m_run = m_new;
      o_live = true;
    }
    if (ok && mbar_wait_fast(pv_done, static_cast<uint32_t>((nXs - 1) & 1), abort_flag, p.err,
                             kSiteAttnSoftmax)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const int pos = iX * C::BQ + r;
      if (p.stats != nullptr && pos < p.N) {
        const float m_s = m_true * p.scale_log2 * 0.69314718055994531f;
        const float l_s = l * ex2_approx((m_run - m_true) * p.scale_log2);
        p.stats[(static_cast<long long>(bidx) * p.h + head) * p.N + pos] = make_float2(m_s, l_s);
      }
      long long orow;
      bool store = true;
      if (p.o_tok) {
        store = pos < p.N;
        orow = static_cast<long long>(bidx) * p.N + pos;
      } else {
        orow = static_cast<long long>(itemA + x - p.item0) * C::BQ + r;
      }
      __half* dst = p.o + orow * p.o_ld + head * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tO + cc * 32, v);
        tmem_ld_wait();
        if (!store) continue;
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
