// Attention backward on the tcgen05 tensor cores ("Blockwise Parallel
// Transformer — BPT", section "The backward pass": each block recomputes its
// scores from the saved per-row statistics (m, l) and consumes them at once).
//
// Per head, with s = q.k / sqrt(d_k), P = exp(s - m) / l, D = rowsum(dO * O):
//   dP = dO V^T,  dS = P * (dP - D),
//   dV = P^T dO,  dK = dS^T Q / sqrt(d_k),  dQ = dS K / sqrt(d_k).
// Two kernels, both deterministic (no atomics):
//   attn_bwd_dkv_tc_kernel  one CTA per (128-key block, head, sequence of
//       the wave): K, V stay in shared memory; the wave's query blocks that
//       see the key block stream through a two-slot ring (Q, dO and the
//       rows' terms a' = -(m + ln l) log2 e and -D).  Per query block:
//         S^T = K Q^T, dP^T = V dO^T     UMMA (SS), fp32 in TMEM
//         P^T, dS^T                       elementwise warps, fp16 back in TMEM
//         dV += P^T dO, dK += dS^T Q     UMMA with A from TMEM
//       The elementwise pass runs in two phases so the tensor core is never
//       left waiting for all of it: P^T (from S^T alone) while dP^T is still
//       being computed, then dS^T once dP^T is done; P^T stays in registers
//       (fp16 pairs) in between.  The UMMA warp issues
//         S_0, dP_0, then per block t: dV_t, S_t+1, dK_t, dP_t+1,
//       each gradient product 64 query columns at a time as they are handed
//       over, and S_t+1 as soon as S_t has been read.  At the end dK, dV are
//       added into the fp32 gradients (waves run in stream order, so each
//       key row is updated by one CTA at a time).
//   attn_bwd_dq_tc_kernel  one CTA per (128-query block, head): Q, dO stay
//       in shared memory, K and V stream through rings.  Per key block:
//         S = Q K^T, dP = dO V^T          UMMA (SS)
//         dS                              elementwise warps, fp16 in TMEM
//         dQ += dS K                      UMMA with A from TMEM
//       The scores are double-buffered in TMEM (S, S, dP, dQ fill the 512
//       columns at d_k = 128), so S_j+2 is computed while block j is being
//       finished; the elementwise pass keeps P in registers from S alone and
//       forms dS once dP lands.  Issue order S_0, dP_0, S_1, then per block
//       j: dQ_j, dP_j+1, S_j+2.
// A 128-row tile of Q, K, V or dO in shared memory ([d_k/64 chunks][128
// rows][64], 128-byte swizzle) is a K-major operand in one product and an
// MN-major one in another (same bytes, different descriptor).
// Warp roles (256 threads): 0 TMA, 1 UMMA issue, 2 TMEM owner, 3 idle,
// 4..7 elementwise (warp w takes TMEM lanes 32(w%4)..: a row of the 128 per
// thread).  Every wait is bounded; on expiry the kernel records a site code,
// drains and frees its tensor memory.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace bpt {

struct AttnBwdTcParams {
  int N, nb, h, d, causal, item0, count, seqs;
  const float* qs;      // [h][count][2][128]: per query block of the wave, the
                        // rows' a' = -(m + ln l) log2 e, then their -D
                        // (attn_row_terms_kernel)
  float* dq;            // [B*N, d] written (this wave's query rows)
  float* dk;            // [B*N, d] accumulated (+=)
  float* dv;            // [B*N, d] accumulated (+=)
  float scale;          // 1 / sqrt(d_k)
  uint32_t* err;
};

template <int D>
struct AttnBwdCfg {
  static constexpr int TILE = 128 * D * 2;  // one 128-row fp16 tile
  static constexpr int CHUNK = 128 * 128;   // one 64-column swizzled chunk
  static constexpr int NSLOT = 2;
  static constexpr int STATS = 2 * 128 * 4;  // a' of the 128 rows, then their -D
  // dK/dV kernel: K, V resident, ring of (Q, dO, stats)
  static constexpr int KV_SLOT = (2 * TILE + STATS + 1023) / 1024 * 1024;
  static constexpr int KV_OFF_RING = 2 * TILE;
  static constexpr int KV_OFF_BAR = KV_OFF_RING + NSLOT * KV_SLOT;
  static constexpr int KV_SMEM = KV_OFF_BAR + 256 + 1024;
  // dQ kernel: Q, dO resident; K in a three-slot ring (held until dQ_j),
  // V in a two-slot ring (held until dP_j)
  static constexpr int QK_SLOTS = 3, QV_SLOTS = 2;
  static constexpr int Q_OFF_K = 2 * TILE;
  static constexpr int Q_OFF_V = Q_OFF_K + QK_SLOTS * TILE;
  static constexpr int Q_OFF_BAR = Q_OFF_V + QV_SLOTS * TILE;
  static constexpr int Q_SMEM = Q_OFF_BAR + 512 + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_A0 = 256, TM_A1 = 256 + D;
  // dQ kernel: scores double-buffered (S_j in TQ_S + 128 (j % 2)), dQ at TQ_A
  static constexpr uint32_t TQ_S = 0, TQ_DP = 256, TQ_A = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(KV_SMEM <= 232448 && Q_SMEM <= 232448, "shared memory budget");
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBwdThreads = 256;
#ifndef BPT_BWD_HANDOVERS
#define BPT_BWD_HANDOVERS 2
#endif
// Hand-overs per 128-column tile from the elementwise warps to the UMMA warp
// (4: every 32 columns; 2: every 64).  Each costs the UMMA warp a barrier
// wait (~100 clocks even when complete), and that warp is the critical path.
constexpr int kBwdHandovers = BPT_BWD_HANDOVERS;
static_assert(kBwdHandovers == 2 || kBwdHandovers == 4, "2 or 4 hand-overs per tile");
constexpr int kBwdChunksPerHand = 4 / kBwdHandovers;

// Issue a 128 x 128 x d_k SS product: D[tmem] = A[a_lo] B[b_lo]^T, both
// K-major tiles (the k-step walks 32 B inside a 64-column chunk, then the
// next chunk).
template <int D>
__device__ __forceinline__ void bwd_issue_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                             uint32_t idesc) {
  constexpr uint32_t hi = sdesc_hi(1024);
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint32_t off = ((k >> 2) * AttnBwdCfg<D>::CHUNK + (k & 3) * 32) >> 4;
    umma_ss(d_tmem, a_lo + off, hi, b_lo + off, hi, idesc, k > 0 ? 1u : 0u);
  }
}

// TMEM column (of the 128 that held the fp32 scores) where the fp16 pairs of
// 32-column chunk cc go: the front of the chunk's own 64-column half.  The
// chunks are handled in order, so only scores already loaded are
// overwritten.
__device__ __forceinline__ constexpr int packed_col(int cc) { return (cc >> 1) * 64 + (cc & 1) * 16; }

// The two 16-deep k-steps of a TS product that cover 32 rows of B (one chunk
// of the A columns the elementwise warps hand over at a time).
template <int D>
__device__ __forceinline__ void bwd_issue_ts_chunk(uint32_t d_tmem, uint32_t a_tmem,
                                                   uint32_t b_lo, uint32_t idesc, int cc,
                                                   bool first) {
  constexpr uint32_t hi = sdesc_hi(1024);
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int k = 2 * cc + kk;
    umma_ts(d_tmem, a_tmem + packed_col(cc) + 8 * kk, b_lo + ((k * 2048) >> 4), hi, idesc,
            (!first || k > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// ----------------------------------------------------------------- dK, dV --
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap mapQKV,
                           const __grid_constant__ CUtensorMap mapDO, const AttnBwdTcParams p) {
  using C = AttnBwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int jb = blockIdx.x, head = blockIdx.y;
  const int bidx = p.seqs > 0 ? p.item0 / p.nb + static_cast<int>(blockIdx.z) : p.item0 / p.nb;
  // this wave's query blocks of sequence bidx, and those that see key block jb
  int ib_lo, ib_hi;
  if (p.seqs > 0) {
    ib_lo = 0;
    ib_hi = p.nb;
  } else {
    ib_lo = p.item0 - bidx * p.nb;
    ib_hi = ib_lo + p.count;
  }
  const int ib0 = p.causal ? max(ib_lo, jb) : ib_lo;
  const int n_q = ib_hi - ib0;
  if (n_q <= 0 || jb * 128 >= p.N) return;  // no query of this wave sees the block

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::KV_OFF_BAR);
  const uint32_t kv_full = smem_u32(bars + 0);
  const uint32_t ring_full0 = smem_u32(bars + 1);
  const uint32_t ring_empty0 = smem_u32(bars + 1 + C::NSLOT);
  const uint32_t s_full = smem_u32(bars + 1 + 2 * C::NSLOT);
  const uint32_t dp_full = smem_u32(bars + 2 + 2 * C::NSLOT);
  const uint32_t p_chunk0 = smem_u32(bars + 3 + 2 * C::NSLOT);   // [kBwdHandovers]: P^T
  const uint32_t ds_chunk0 = smem_u32(bars + 7 + 2 * C::NSLOT);  // [kBwdHandovers]: dS^T
  const uint32_t acc_done = smem_u32(bars + 11 + 2 * C::NSLOT);
  const uint32_t drain = smem_u32(bars + 12 + 2 * C::NSLOT);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(ring_full0 + 8 * s, 1);
      mbar_init(ring_empty0 + 8 * s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    for (int c = 0; c < 4; ++c) {
      mbar_init(p_chunk0 + 8 * c, 4);
      mbar_init(ds_chunk0 + 8 * c, 4);
    }
    mbar_init(acc_done, 1);
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
  const int chQ = head * D / 64, chK = (p.d + head * D) / 64, chV = (2 * p.d + head * D) / 64;
  const long long lbase = static_cast<long long>(bidx * p.nb - p.item0) * 128;  // wave row of pos 0
  // row terms of this head: [count][2][128] floats from here, by wave block
  const float* qs_head = p.qs + static_cast<long long>(head) * p.count * 256;
  const int lblk0 = bidx * p.nb - p.item0;  // wave block of this sequence's block 0

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = lane == 0;
    int armed[C::NSLOT];
    for (int s = 0; s < C::NSLOT; ++s) armed[s] = -1;
    if (leader) {
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
      tma_load_4d(smem_u32(smem), &mapQKV, kv_full, 0, jb * 128, chK, bidx);
      tma_load_4d(smem_u32(smem + C::TILE), &mapQKV, kv_full, 0, jb * 128, chV, bidx);
    }
    for (int t = 0; t < n_q; ++t) {
      const int slot = t % C::NSLOT;
      const uint32_t phase = static_cast<uint32_t>((t / C::NSLOT) & 1);
      if (!mbar_wait_warp(ring_empty0 + 8 * slot, phase ^ 1u, abort_flag, p.err,
                          kSiteAttnProducer))
        break;
      const int ib = ib0 + t;
      uint8_t* sl = smem + C::KV_OFF_RING + slot * C::KV_SLOT;
      if (leader) {
        armed[slot] = static_cast<int>(phase);
        mbar_arrive_expect_tx(ring_full0 + 8 * slot, 2 * C::TILE + C::STATS);
        bulk_load(smem_u32(sl + 2 * C::TILE), qs_head + (lblk0 + ib) * 256LL, C::STATS,
                  ring_full0 + 8 * slot);
        tma_load_4d(smem_u32(sl), &mapQKV, ring_full0 + 8 * slot, 0, ib * 128, chQ, bidx);
        tma_load_3d(smem_u32(sl + C::TILE), &mapDO, ring_full0 + 8 * slot, 0,
                    static_cast<int>(lbase + ib * 128), head * D / 64);
      }
      __syncwarp();
    }
    mbar_wait_drain(kv_full, 0, p.err);
    for (int s = 0; s < C::NSLOT; ++s)
      if (armed[s] >= 0) mbar_wait_drain(ring_full0 + 8 * s, static_cast<uint32_t>(armed[s]), p.err);
  } else if (warp == 1) {
    // ---------------------------------------------------------- UMMA issue
    const bool leader = lane == 0;
    constexpr uint32_t idesc_s = idesc_f16_f32(128, 128, false, false);
    constexpr uint32_t idesc_o = idesc_f16_f32(128, D, false, true);
    const uint32_t k_lo = sdesc_lo(smem_u32(smem), 16);
    const uint32_t v_lo = sdesc_lo(smem_u32(smem + C::TILE), 16);
    auto commit = [&](uint32_t bar) {
      if (leader) umma_commit(bar);
      __syncwarp();
    };
    auto slot_of = [&](int t) {
      return smem_u32(smem + C::KV_OFF_RING + (t % C::NSLOT) * C::KV_SLOT);
    };
    // S^T_t = K Q_t^T once Q_t has landed
    auto issue_s = [&](int t) -> bool {
      if (!mbar_wait_warp(ring_full0 + 8 * (t % C::NSLOT),
                          static_cast<uint32_t>((t / C::NSLOT) & 1), abort_flag, p.err,
                          kSiteAttnMma))
        return false;
      tc_fence_after();
      if (leader) bwd_issue_ss<D>(tmem + C::TM_S, k_lo, sdesc_lo(slot_of(t), 16), idesc_s);
      __syncwarp();
      commit(s_full);
      return true;
    };
    // dP^T_t = V dO_t^T (slot already waited by issue_s)
    auto issue_dp = [&](int t) {
      if (leader)
        bwd_issue_ss<D>(tmem + C::TM_DP, v_lo, sdesc_lo(slot_of(t) + C::TILE, 16), idesc_s);
      __syncwarp();
      commit(dp_full);
    };
    // one gradient product, 128 / kBwdHandovers query columns at a time as
    // the elementwise warps hand them over on barriers cb[0 .. kBwdHandovers)
    auto issue_grad = [&](int t, uint32_t cb, uint32_t acc, uint32_t a_tm, uint32_t b_lo) {
      for (int hh = 0; hh < kBwdHandovers; ++hh) {
        if (!mbar_wait_warp(cb + 8 * hh, static_cast<uint32_t>(t & 1), abort_flag, p.err,
                            kSiteAttnMma))
          return false;
        tc_fence_after();
        if (leader)
          for (int q = 0; q < kBwdChunksPerHand; ++q)
            bwd_issue_ts_chunk<D>(acc, a_tm, b_lo, idesc_o, hh * kBwdChunksPerHand + q, t == 0);
        __syncwarp();
      }
      return true;
    };
    bool ok = mbar_wait_warp(kv_full, 0, abort_flag, p.err, kSiteAttnMma) && issue_s(0);
    if (ok) issue_dp(0);
    for (int t = 0; t < n_q && ok; ++t) {
      const uint32_t sl = slot_of(t);
      // dV += P^T dO_t
      if (!(ok = issue_grad(t, p_chunk0, tmem + C::TM_A0, tmem + C::TM_S,
                            sdesc_lo(sl + C::TILE, C::CHUNK))))
        break;
      // S^T_t has been read in full: the next block's scores can go there
      if (t + 1 < n_q && !(ok = issue_s(t + 1))) break;
      // dK += dS^T Q_t
      if (!(ok = issue_grad(t, ds_chunk0, tmem + C::TM_A1, tmem + C::TM_DP,
                            sdesc_lo(sl, C::CHUNK))))
        break;
      commit(ring_empty0 + 8 * (t % C::NSLOT));
      if (t + 1 < n_q) issue_dp(t + 1);
    }
    commit(acc_done);
    commit(drain);
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // --------------------------------------------------------- elementwise
    const int e = warp & 3;
    const int kr = e * 32 + lane;  // key row of the block
    const int kp = jb * 128 + kr;
    const bool key_ok = kp < p.N;
    const bool key_blk_full = jb * 128 + 128 <= p.N;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(e * 32) << 16);
    const float2 c2 = make_float2(p.scale * kLog2e, p.scale * kLog2e);
    bool ok = true;
    for (int t = 0; t < n_q && ok; ++t) {
      const int slot = t % C::NSLOT;
      // The slot's row terms arrive by bulk copy on its full barrier: acquire
      // it (long complete by now; the slot is released only after this
      // warp's last dS^T hand-over of block t).
      if (!mbar_wait_warp(ring_full0 + 8 * slot, static_cast<uint32_t>((t / C::NSLOT) & 1),
                          abort_flag, p.err, kSiteAttnSoftmax) ||
          !mbar_wait_warp(s_full, static_cast<uint32_t>(t & 1), abort_flag, p.err,
                          kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* st = reinterpret_cast<const float*>(smem + C::KV_OFF_RING + slot * C::KV_SLOT +
                                                       2 * C::TILE);
      const int ib = ib0 + t;
      // masking only on the diagonal block and a ragged last key block
      const bool diag = p.causal && ib == jb;
      const bool masked = diag || !key_blk_full;
      uint32_t pp[64];  // P^T of this key row, fp16 pairs, kept for the dS^T phase
      // ---- phase 1: P^T = 2^(S^T c + a'), per query column
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sr[32];
        tmem_ld_32x32b_x32(t_lane + C::TM_S + cc * 32, sr);
        tmem_ld_wait();
        auto tile = [&](auto mask) {
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const int q = cc * 32 + k;
            const float2 a = *reinterpret_cast<const float2*>(st + q);  // broadcast
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])), c2, a);
            float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if constexpr (decltype(mask)::value) {
              if (!key_ok || (diag && kr > q)) pr.x = 0.f;
              if (!key_ok || (diag && kr > q + 1)) pr.y = 0.f;
            }
            pp[cc * 16 + (k >> 1)] = pack_f16x2(pr.x, pr.y);
          }
        };
        if (masked)
          tile(std::true_type{});
        else
          tile(std::false_type{});
        tmem_st16(t_lane + C::TM_S + packed_col(cc), pp + cc * 16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && (cc + 1) % kBwdChunksPerHand == 0)
          mbar_arrive(p_chunk0 + 8 * (cc / kBwdChunksPerHand));
      }
      // ---- phase 2: dS^T = P^T (dP^T - D)
      if (!mbar_wait_warp(dp_full, static_cast<uint32_t>(t & 1), abort_flag, p.err,
                          kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t dr[32], ds[16];
        tmem_ld_32x32b_x32(t_lane + C::TM_DP + cc * 32, dr);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const float2 nd = *reinterpret_cast<const float2*>(st + 128 + cc * 32 + k);
          const float2 pr = __half22float2(*reinterpret_cast<const __half2*>(&pp[cc * 16 + (k >> 1)]));
          const float2 v = __fmul2_rn(
              pr, __fadd2_rn(make_float2(__uint_as_float(dr[k]), __uint_as_float(dr[k + 1])), nd));
          ds[k >> 1] = pack_f16x2(v.x, v.y);
        }
        tmem_st16(t_lane + C::TM_DP + packed_col(cc), ds);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && (cc + 1) % kBwdChunksPerHand == 0)
          mbar_arrive(ds_chunk0 + 8 * (cc / kBwdChunksPerHand));
      }
    }
    if (ok && mbar_wait_warp(acc_done, 0, abort_flag, p.err, kSiteAttnSoftmax)) {
      tc_fence_after();
      const long long g = static_cast<long long>(bidx) * p.N + kp;
      float* dvr = p.dv + g * p.d + head * D;
      float* dkr = p.dk + g * p.d + head * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t a[32], b[32];  // warp-collective loads: every lane takes them
        tmem_ld_32x32b_x32(t_lane + C::TM_A0 + cc * 32, a);
        tmem_ld_32x32b_x32(t_lane + C::TM_A1 + cc * 32, b);
        tmem_ld_wait();
        if (key_ok) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            dvr[cc * 32 + k] += __uint_as_float(a[k]);
            dkr[cc * 32 + k] += __uint_as_float(b[k]) * p.scale;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------- dQ --
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap mapQKV,
                          const __grid_constant__ CUtensorMap mapDO, const AttnBwdTcParams p) {
  using C = AttnBwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int qb = blockIdx.x, head = blockIdx.y;
  const int item = p.item0 + qb;
  const int bidx = item / p.nb, ib = item - (item / p.nb) * p.nb;
  const int n_kv = p.causal ? ib + 1 : p.nb;
  const long long lrow = static_cast<long long>(qb) * 128;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::Q_OFF_BAR);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t k_full0 = smem_u32(bars + 1);   // [3]
  const uint32_t k_empty0 = smem_u32(bars + 4);  // [3]
  const uint32_t v_full0 = smem_u32(bars + 7);   // [2]
  const uint32_t v_empty0 = smem_u32(bars + 9);  // [2]
  const uint32_t s_full0 = smem_u32(bars + 11);  // [2]: S_j landed in buffer j % 2
  const uint32_t s_free0 = smem_u32(bars + 13);  // [2]: buffer j % 2 read by every warp
  const uint32_t dp_full = smem_u32(bars + 15);
  const uint32_t ds_chunk0 = smem_u32(bars + 16);  // [kBwdHandovers]: dS column groups
  const uint32_t acc_done = smem_u32(bars + 20);
  const uint32_t drain = smem_u32(bars + 21);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::QK_SLOTS; ++s) {
      mbar_init(k_full0 + 8 * s, 1);
      mbar_init(k_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < C::QV_SLOTS; ++s) {
      mbar_init(v_full0 + 8 * s, 1);
      mbar_init(v_empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full0 + 8 * b, 1);
      mbar_init(s_free0 + 8 * b, 4);
    }
    mbar_init(dp_full, 1);
    for (int c = 0; c < 4; ++c) mbar_init(ds_chunk0 + 8 * c, 4);
    mbar_init(acc_done, 1);
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
  const int chQ = head * D / 64, chK = (p.d + head * D) / 64, chV = (2 * p.d + head * D) / 64;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = lane == 0;
    int k_armed[C::QK_SLOTS], v_armed[C::QV_SLOTS];
    for (int s = 0; s < C::QK_SLOTS; ++s) k_armed[s] = -1;
    for (int s = 0; s < C::QV_SLOTS; ++s) v_armed[s] = -1;
    if (leader) {
      mbar_arrive_expect_tx(q_full, 2 * C::TILE);
      tma_load_4d(smem_u32(smem), &mapQKV, q_full, 0, ib * 128, chQ, bidx);
      tma_load_3d(smem_u32(smem + C::TILE), &mapDO, q_full, 0, static_cast<int>(lrow),
                  head * D / 64);
    }
    for (int j = 0; j < n_kv; ++j) {
      const int ks = j % C::QK_SLOTS, vs = j % C::QV_SLOTS;
      const uint32_t kph = static_cast<uint32_t>((j / C::QK_SLOTS) & 1);
      const uint32_t vph = static_cast<uint32_t>((j / C::QV_SLOTS) & 1);
      if (!mbar_wait_warp(k_empty0 + 8 * ks, kph ^ 1u, abort_flag, p.err, kSiteAttnProducer))
        break;
      if (leader) {
        k_armed[ks] = static_cast<int>(kph);
        mbar_arrive_expect_tx(k_full0 + 8 * ks, C::TILE);
        tma_load_4d(smem_u32(smem + C::Q_OFF_K + ks * C::TILE), &mapQKV, k_full0 + 8 * ks, 0,
                    j * 128, chK, bidx);
      }
      __syncwarp();
      if (!mbar_wait_warp(v_empty0 + 8 * vs, vph ^ 1u, abort_flag, p.err, kSiteAttnProducer))
        break;
      if (leader) {
        v_armed[vs] = static_cast<int>(vph);
        mbar_arrive_expect_tx(v_full0 + 8 * vs, C::TILE);
        tma_load_4d(smem_u32(smem + C::Q_OFF_V + vs * C::TILE), &mapQKV, v_full0 + 8 * vs, 0,
                    j * 128, chV, bidx);
      }
      __syncwarp();
    }
    mbar_wait_drain(q_full, 0, p.err);
    for (int s = 0; s < C::QK_SLOTS; ++s)
      if (k_armed[s] >= 0) mbar_wait_drain(k_full0 + 8 * s, static_cast<uint32_t>(k_armed[s]), p.err);
    for (int s = 0; s < C::QV_SLOTS; ++s)
      if (v_armed[s] >= 0) mbar_wait_drain(v_full0 + 8 * s, static_cast<uint32_t>(v_armed[s]), p.err);
  } else if (warp == 1) {
    // ---------------------------------------------------------- UMMA issue
    const bool leader = lane == 0;
    constexpr uint32_t idesc_s = idesc_f16_f32(128, 128, false, false);
    constexpr uint32_t idesc_o = idesc_f16_f32(128, D, false, true);
    const uint32_t q_lo = sdesc_lo(smem_u32(smem), 16);
    const uint32_t do_lo = sdesc_lo(smem_u32(smem + C::TILE), 16);
    auto commit = [&](uint32_t bar) {
      if (leader) umma_commit(bar);
      __syncwarp();
    };
    auto k_slot = [&](int j) { return smem_u32(smem + C::Q_OFF_K + (j % C::QK_SLOTS) * C::TILE); };
    auto v_slot = [&](int j) { return smem_u32(smem + C::Q_OFF_V + (j % C::QV_SLOTS) * C::TILE); };
    // S_j = Q K_j^T into buffer j % 2, once K_j has landed
    auto issue_s = [&](int j) -> bool {
      if (!mbar_wait_warp(k_full0 + 8 * (j % C::QK_SLOTS),
                          static_cast<uint32_t>((j / C::QK_SLOTS) & 1), abort_flag, p.err,
                          kSiteAttnMma))
        return false;
      tc_fence_after();
      if (leader)
        bwd_issue_ss<D>(tmem + C::TQ_S + 128u * static_cast<uint32_t>(j & 1), q_lo,
                        sdesc_lo(k_slot(j), 16), idesc_s);
      __syncwarp();
      commit(s_full0 + 8 * (j & 1));
      return true;
    };
    // dP_j = dO V_j^T, once V_j has landed; V_j's slot is free once it is done
    auto issue_dp = [&](int j) -> bool {
      if (!mbar_wait_warp(v_full0 + 8 * (j % C::QV_SLOTS),
                          static_cast<uint32_t>((j / C::QV_SLOTS) & 1), abort_flag, p.err,
                          kSiteAttnMma))
        return false;
      tc_fence_after();
      if (leader) bwd_issue_ss<D>(tmem + C::TQ_DP, do_lo, sdesc_lo(v_slot(j), 16), idesc_s);
      __syncwarp();
      commit(dp_full);
      commit(v_empty0 + 8 * (j % C::QV_SLOTS));
      return true;
    };
    bool ok = mbar_wait_warp(q_full, 0, abort_flag, p.err, kSiteAttnMma) && issue_s(0) &&
              issue_dp(0) && (n_kv < 2 || issue_s(1));
    for (int j = 0; j < n_kv && ok; ++j) {
      // dQ += dS_j K_j, 128 / kBwdHandovers key columns at a time as handed over
      for (int hh = 0; hh < kBwdHandovers; ++hh) {
        if (!mbar_wait_warp(ds_chunk0 + 8 * hh, static_cast<uint32_t>(j & 1), abort_flag, p.err,
                            kSiteAttnMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader)
          for (int q = 0; q < kBwdChunksPerHand; ++q)
            bwd_issue_ts_chunk<D>(tmem + C::TQ_A, tmem + C::TQ_DP, sdesc_lo(k_slot(j), C::CHUNK),
                                  idesc_o, hh * kBwdChunksPerHand + q, j == 0);
        __syncwarp();
      }
      if (!ok) break;
      commit(k_empty0 + 8 * (j % C::QK_SLOTS));
      // dP_j+1 overwrites dP_j / dS_j: after dQ_j (in order) and after every
      // warp's last dS hand-over (all of dP_j has been read)
      if (j + 1 < n_kv && !(ok = issue_dp(j + 1))) break;
      // S_j+2 reuses S_j's buffer once every warp has read S_j
      if (j + 2 < n_kv) {
        if (!mbar_wait_warp(s_free0 + 8 * (j & 1), static_cast<uint32_t>((j >> 1) & 1),
                            abort_flag, p.err, kSiteAttnMma) ||
            !issue_s(j + 2)) {
          ok = false;
          break;
        }
      }
    }
    commit(acc_done);
    commit(drain);
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // --------------------------------------------------------- elementwise
    const int e = warp & 3;
    const int qr = e * 32 + lane;  // query row of the block
    const int qp = ib * 128 + qr;
    const bool q_ok = qp < p.N;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(e * 32) << 16);
    const float2 c2 = make_float2(p.scale * kLog2e, p.scale * kLog2e);
    const float* rt = p.qs + (static_cast<long long>(head) * p.count + qb) * 256;
    const float2 a2 = make_float2(rt[qr], rt[qr]);               // a': -inf past the sequence
    const float2 nd2 = make_float2(rt[128 + qr], rt[128 + qr]);  // -D
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      if (!mbar_wait_warp(s_full0 + 8 * (j & 1), static_cast<uint32_t>((j >> 1) & 1), abort_flag,
                          p.err, kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = p.causal && j == ib;
      const int klim = p.N - j * 128;  // keys >= klim are past the sequence
      const bool masked = diag || klim < 128;
      const uint32_t tS = t_lane + C::TQ_S + 128u * static_cast<uint32_t>(j & 1);
      uint32_t pp[64];  // P of this query row, fp16 pairs, kept for the dS phase
      // ---- phase 1: P = 2^(S c + a') from S alone
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sr[32];
        tmem_ld_32x32b_x32(tS + cc * 32, sr);
        tmem_ld_wait();
        if (cc == 3) {
          // every score of buffer j % 2 is in registers: S_j+2 may go there
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free0 + 8 * (j & 1));
        }
        auto tile = [&](auto mask) {
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const int kc = cc * 32 + k;
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])), c2, a2);
            float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if constexpr (decltype(mask)::value) {
              if (kc >= klim || (diag && kc > qr)) pr.x = 0.f;
              if (kc + 1 >= klim || (diag && kc + 1 > qr)) pr.y = 0.f;
            }
            pp[cc * 16 + (k >> 1)] = pack_f16x2(pr.x, pr.y);
          }
        };
        if (masked)
          tile(std::true_type{});
        else
          tile(std::false_type{});
      }
      // ---- phase 2: dS = P (dP - D)
      if (!mbar_wait_warp(dp_full, static_cast<uint32_t>(j & 1), abort_flag, p.err,
                          kSiteAttnSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t dr[32], ds16[16];
        tmem_ld_32x32b_x32(t_lane + C::TQ_DP + cc * 32, dr);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const float2 pr =
              __half22float2(*reinterpret_cast<const __half2*>(&pp[cc * 16 + (k >> 1)]));
          const float2 v = __fmul2_rn(
              pr, __fadd2_rn(make_float2(__uint_as_float(dr[k]), __uint_as_float(dr[k + 1])), nd2));
          ds16[k >> 1] = pack_f16x2(v.x, v.y);
        }
        tmem_st16(t_lane + C::TQ_DP + packed_col(cc), ds16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && (cc + 1) % kBwdChunksPerHand == 0)
          mbar_arrive(ds_chunk0 + 8 * (cc / kBwdChunksPerHand));
      }
    }
    if (ok && mbar_wait_warp(acc_done, 0, abort_flag, p.err, kSiteAttnSoftmax)) {
      tc_fence_after();
      float* dst = p.dq + (static_cast<long long>(bidx) * p.N + qp) * p.d + head * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + C::TQ_A + cc * 32, v);
        tmem_ld_wait();
        if (q_ok) {
#pragma unroll
          for (int k = 0; k < 32; ++k) dst[cc * 32 + k] = __uint_as_float(v[k]) * p.scale;
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
