// The per-query-block layer body after attention, fused into one persistent
// kernel on CTA pairs ("Blockwise Parallel Transformer — BPT", section "The
// fused blockwise algorithm": inside the outer loop over query blocks, after
// the block's attention output o_i, the body forms y_i = x_i + o_i W_O, then
// LN2, the FFN hidden of the block and Z_i = y_i + FFN(LN2(y_i)); section
// "Memory accounting: what actually shrinks": the FFN hidden becomes a
// [b, 4d]-shaped transient instead of an [N, 4d] tensor).
//
// A work item is two query blocks (256 rows); CTA rank r of a pair owns the
// item's block r (128 rows, the tensor-memory lanes of its SM) and the pair
// multiplies with tcgen05.mma.cta_group::2 (M = 256), each CTA loading its
// own 128 rows of A and half of each 256-column slab of B, as in the GEMM of
// gemm_tc.cuh.  Per item, in this order:
//
//   B  y   = x + o W_O        N-tiles of 256 over d,    K = d     -> out (fp32)
//   C  v   = LN2(y)           the epilogue warps, one warp per row -> v scratch
//   D  H_c = GELU(v W_1[:, c] + b_1[c])   c = 256-column chunks of d_ff
//                                                        K = d     -> H scratch
//   E  Z   = y + H W_2 + b_2  N-tiles of 512 (256 if d % 512 != 0) over d,
//                                                        K = d_ff  -> out (fp32)
//
// o is read from the Q columns of the QKV buffer (the attention kernel wrote
// each block's output over the block's own queries).  v [256, d] and
// H [256, d_ff] (fp16) are the pair's private scratch in global memory: the
// accumulator of a [128, d] product does not fit one SM's tensor memory
// (512 columns) for d > 512, so the hidden goes through L2, chunk by chunk,
// and lives only while its item is in flight.  The workspace is therefore
// pairs x 256 x (2d + 2 d_ff) bytes, independent of N.
//
// Hand-offs inside a CTA (all bounded mbarrier waits):
//   ep_sync  the eight epilogue warps, after their last y tile: LN2 reads
//            whole rows that other warps wrote;
//   v_ready  LN2 done (v written, made visible to the async proxy): the
//            producer may load v as the A operand of D;
//   h_ready  every H chunk of the item written (likewise): the producer may
//            load H as the A operand of E.
// The producer issues each stage's B (weight) load before it waits for a
// hand-off, so the weights stream in while the epilogue finishes.
//
// Items are dealt round-robin over the pairs.  When R whole rounds leave L
// items over (0 < L <= pairs / 2), the last round would keep L pairs busy for
// a whole item while the others idle; instead each left-over item is shared
// by two pairs (q and q + L), each computing half of its y tiles, all of its
// LN2, half of its H chunks and half of its Z tiles (by columns).  LN2 needs
// the other pair's y columns, and a Z tile (K = d_ff) needs the other pair's
// H columns, read from that pair's scratch; two counters per CTA in global
// memory (written with release, polled with acquire, bounded) carry these
// two hand-overs.  Every output element still comes from the same products
// in the same K order, so sharing changes no bit of the result.
//
// Arithmetic per element is that of the wave path (same UMMA shapes and
// K order, same epilogues, LN2 with the summation order of ln_rows_kernel),
// so the two schedules give bitwise the same output.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "rows.cuh"

namespace bpt {

struct TailParams {
  int blocks;    // query block items (batch * nb)
  int items;     // pair items = ceil(blocks / 2)
  int nb, N;     // query blocks per sequence, tokens per sequence
  int d, d_ff;
  float* out;                      // [B*N, d] fp32: y, then Z
  const __nv_bfloat16* x;          // [B*N, d] residual input
  const __nv_bfloat16* ln2;        // [2, d] gamma; beta
  const __nv_bfloat16* b1;         // [d_ff]
  const __nv_bfloat16* b2;         // [d]
  __half* v_scr;                   // [pairs*256, d]
  __half* h_scr;                   // [pairs*256, d_ff]
  uint32_t* err;
  uint32_t* flags;  // shared items: [2][kTailMaxPairs][2] arrival counters, zero at launch
  int split;        // share the left-over items (needs d % 1024 == 0, d_ff % 512 == 0)
  int fault;  // test hook: 3 = pair 0's leader never loads its first A tile
};

constexpr int kTailEpi = 8;  // epilogue warps (two per TMEM lane quarter)
constexpr int kTailThreads = 32 * (4 + kTailEpi);
// CTA pairs the workspace is sized for (148 SMs); launches use at most this.
constexpr int kTailMaxPairs = 74;

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Counter of a CTA's hand-over to the partner pair: kind 0 = its y columns
// of the shared item are stored, 1 = its H columns are.  Each of the CTA's
// epilogue warps adds one.
__device__ __forceinline__ int tail_flag(int kind, int pair, uint32_t rank) {
  return (kind * kTailMaxPairs + pair) * 2 + static_cast<int>(rank);
}

// A pair's items: j = 0 .. J-1, whole items pair + j * npairs, then (when
// half >= 0) its half of the shared item hitem, computed with `partner`.
struct TailPlan {
  int J, Jfull, hitem, half, partner;
  int first, stride;
  __host__ __device__ __forceinline__ int item(int j) const {
    return j < Jfull ? first + j * stride : hitem;
  }
  __host__ __device__ __forceinline__ int half_of(int j) const { return j < Jfull ? -1 : half; }
};

// Whether the launch shares the left-over items: L = items mod pairs with
// 0 < L <= pairs / 2, and every half a whole number of tiles (y tiles and H
// chunks of 256 columns, Z tiles of 512).
__host__ __device__ __forceinline__ bool tail_shares(int items, int pairs, int d, int d_ff) {
  const int left = items % pairs;
  return left > 0 && 2 * left <= pairs && d % 1024 == 0 && d_ff % 512 == 0;
}

// Also compiled for the host, where bpt_layer_tail_plan reports it.
__host__ __device__ __forceinline__ TailPlan tail_plan(const TailParams& p, int pair, int npairs) {
  TailPlan pl{};
  pl.first = pair;
  pl.stride = npairs;
  pl.half = -1;
  pl.hitem = 0;
  pl.partner = pair;
  const int R = p.items / npairs, L = p.items - R * npairs;
  if (p.split && L > 0 && 2 * L <= npairs) {
    pl.Jfull = R;
    pl.J = R;
    if (pair < 2 * L) {
      pl.half = pair >= L ? 1 : 0;
      pl.hitem = R * npairs + pair - pl.half * L;
      pl.partner = pl.half ? pair - L : pair + L;
      pl.J = R + 1;
    }
  } else {
    pl.Jfull = pl.J = pair < p.items ? (p.items - pair + npairs - 1) / npairs : 0;
  }
  return pl;
}

// Tiles [n0, n1) of a segment of `tiles` tiles: all of them, or half h.
__device__ __forceinline__ void tail_range(int tiles, int h, int& n0, int& n1) {
  if (h < 0) {
    n0 = 0;
    n1 = tiles;
  } else {
    n0 = h * (tiles / 2);
    n1 = n0 + tiles / 2;
  }
}

// LN2 of the CTA's 128 rows of an item, one warp per row (rows w, w + 8, ..),
// reading y from `out` three times (sum, squared deviations, normalise) in
// the summation order of ln_rows_kernel (lane l sums its 8-element chunks
// (l + 32 q) * 8 in q order, then a warp sum).  Rows without a token (ragged
// last block, absent second block) get zeros.  It runs while the tensor
// cores work on the previous item's W_2 tiles (see the item order below).
__device__ __forceinline__ void tail_ln2(const TailParams& p, const RowMap& map, int m_valid,
                                         int s_base, long long v_row0, int w, int lane) {
  const int d = p.d;
#pragma unroll 1
  for (int q = w; q < 128; q += kTailEpi) {
    const int s = s_base + q;
    const long long g = s < m_valid ? map.map(s) : -1;
    __half* vrow = p.v_scr + (v_row0 + q) * d;
    bool bad = false;
    if (g < 0) {
      const float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int c = lane * 8; c < d; c += 256) store8(vrow + c, z, bad);
      continue;
    }
    const float* yrow = p.out + g * d;
    float sum = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      float v[8];
      load8(yrow + c, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) sum += v[e];
    }
    const float mean = warp_sum(sum) / static_cast<float>(d);
    float sq = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      float v[8];
      load8(yrow + c, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float t = v[e] - mean;
        sq += t * t;
      }
    }
    const float var = warp_sum(sq) / static_cast<float>(d);
    const float rstd = 1.0f / sqrtf(var + kLnEps);
    for (int c = lane * 8; c < d; c += 256) {
      float v[8], gm[8], bt[8], o[8];
      load8(yrow + c, v);
      load8(p.ln2 + c, gm);
      load8(p.ln2 + d + c, bt);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = (v[e] - mean) * rstd * gm[e] + bt[e];
      store8(vrow + c, o, bad);
    }
    if (bad) record_error(p.err, kErrRange, kSiteRangeLN);
  }
}

// The tiles of one item.  y tiles and H chunks are 256 columns wide (K = d,
// 128-deep stages); Z tiles are 512 columns wide when e512 (d % 512 == 0; K =
// d_ff in 64-deep stages; the two 256-column halves share every H load, which
// halves the re-reads of the hidden), else 256.  The epilogue sees a
// 512-column tile as two consecutive 256-column accumulator slots.
struct TailShape {
  int nB, nD, nE, kbD, kbF, kbF64;  // tiles per phase; K blocks over d, d_ff (128 / 64 deep)
  bool e512;
  __device__ __forceinline__ int kblocks(int phase) const {
    return phase == 2 ? (e512 ? kbF64 : kbF) : kbD;
  }
};

// Segment order of a pair's J items (B = y tiles, D = H chunks, E = Z tiles):
//   B0 D0 | B1 E0 D1 | B2 E1 D2 | ... | B(J-1) E(J-2) D(J-1) | E(J-1)
// Item j's LN2 runs in the epilogue between B(j) and E(j-1), so the tensor
// cores compute E(j-1) meanwhile; and E(j) waits for the whole hidden of item
// j behind B(j+1).  One H buffer suffices: UMMA work issued by one thread
// completes in order, so every load of E(j) has landed before any D(j+1)
// epilogue store.
__device__ __forceinline__ void tail_segment(int s, int J, int& phase, int& j) {
  if (s < 2) {
    phase = s == 0 ? 0 : 1;
    j = 0;
    return;
  }
  const int t = s - 2;
  if (t == 3 * (J - 1)) {
    phase = 2;
    j = J - 1;
    return;
  }
  const int q = t / 3 + 1, r = t % 3;
  phase = r == 0 ? 0 : (r == 1 ? 2 : 1);
  j = r == 1 ? q - 1 : q;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTailThreads, 1)
    tail_pair_kernel(const __grid_constant__ CUtensorMap mapO,
                     const __grid_constant__ CUtensorMap mapWo,
                     const __grid_constant__ CUtensorMap mapV,
                     const __grid_constant__ CUtensorMap mapW1,
                     const __grid_constant__ CUtensorMap mapH,
                     const __grid_constant__ CUtensorMap mapW2,
                     const __grid_constant__ CUtensorMap mapH1,
                     const __grid_constant__ CUtensorMap mapW2e, const TailParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPairStages * kPairABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  const uint32_t full0 = smem_u32(bars + 0);
  const uint32_t empty0 = smem_u32(bars + kPairStages);
  const uint32_t accf0 = smem_u32(bars + 2 * kPairStages);
  const uint32_t acce0 = smem_u32(bars + 2 * kPairStages + 2);
  const uint32_t drain = smem_u32(bars + 2 * kPairStages + 4);
  const uint32_t ep_sync = smem_u32(bars + 2 * kPairStages + 5);
  const uint32_t v_ready = smem_u32(bars + 2 * kPairStages + 6);
  const uint32_t h_ready = smem_u32(bars + 2 * kPairStages + 7);
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(nclusters_x());
  const TailPlan pl = tail_plan(p, pair, npairs);
  const int J = pl.J;
  const int n_seg = 3 * J;
  TailShape sh;
  sh.e512 = p.d % 512 == 0;
  sh.nB = (p.d + kGemmBN - 1) / kGemmBN;
  sh.nD = (p.d_ff + kGemmBN - 1) / kGemmBN;
  sh.nE = sh.e512 ? p.d / 512 : sh.nB;
  sh.kbD = (p.d + kGemmBK - 1) / kGemmBK;
  sh.kbF = (p.d_ff + kGemmBK - 1) / kGemmBK;
  sh.kbF64 = (p.d_ff + 63) / 64;

  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < kPairStages; ++s2) {
      mbar_init(full0 + 8 * s2, 1);
      mbar_init(empty0 + 8 * s2, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 2 * kTailEpi);
    }
    mbar_init(drain, 1);
    mbar_init(ep_sync, kTailEpi);
    mbar_init(v_ready, kTailEpi);
    mbar_init(h_ready, kTailEpi);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(&tmem_base_sh), kGemmTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&mapO);
      tma_prefetch_desc(&mapWo);
      tma_prefetch_desc(&mapV);
      tma_prefetch_desc(&mapW1);
      tma_prefetch_desc(&mapH);
      tma_prefetch_desc(&mapW2);
      tma_prefetch_desc(&mapH1);
      tma_prefetch_desc(&mapW2e);
    }
    int armed[kPairStages];
    for (int s2 = 0; s2 < kPairStages; ++s2) armed[s2] = -1;
    int stage = 0;
    uint32_t phase_bit = 0;
    bool ok = true;
    const int scr_row = pair * 256 + static_cast<int>(rank) * 128;
    const int scr_row_partner = pl.partner * 256 + static_cast<int>(rank) * 128;
    for (int sg = 0; sg < n_seg && ok; ++sg) {
      int ph, j;
      tail_segment(sg, J, ph, j);
      const int item = pl.item(j);
      const int hf = pl.half_of(j);
      // token row of this CTA's block (an absent second block reads block 0's
      // rows: its results are never stored)
      int blk = 2 * item + static_cast<int>(rank);
      if (blk >= p.blocks) blk = 0;
      const int bseq = blk / p.nb;
      const int tok_row = bseq * p.N + (blk - bseq * p.nb) * 128;
      // a 512-column Z tile: A in 64-deep single-chunk boxes (mapH1), B as
      // this CTA's contiguous 256-column slab, 64 K rows (mapW2e)
      const bool wide = ph == 2 && sh.e512;
      const CUtensorMap* ma = ph == 0 ? &mapO : (ph == 1 ? &mapV : (wide ? &mapH1 : &mapH));
      const CUtensorMap* mb = ph == 0 ? &mapWo : (ph == 1 ? &mapW1 : (wide ? &mapW2e : &mapW2));
      const int a_row = ph == 0 ? tok_row : scr_row;
      const int kbs = sh.kblocks(ph);
      const int tiles = ph == 0 ? sh.nB : (ph == 1 ? sh.nD : sh.nE);
      const uint32_t stage_bytes =
          wide ? 2u * (kPairABytes / 2 + kPairBBytes) : 2u * kPairStageBytes;
      int n0, n1;
      tail_range(tiles, hf, n0, n1);
      for (int n = n0; n < n1 && ok; ++n) {
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait_warp(empty0 + 8 * stage, phase_bit ^ 1u, abort_flag, p.err,
                              kSiteGemmProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb_leader = map_to_rank(full0 + 8 * stage, 0);
          if (rank == 0) armed[stage] = static_cast<int>(phase_bit);
          if (leader) {
            if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * stage, stage_bytes);
            if (wide)
              tma_load_3d_pair(smem_u32(sB + stage * kPairBBytes), mb, fb_leader, 0, kb * 64,
                               n * 8 + static_cast<int>(rank) * 4);
            else
              tma_load_3d_pair(smem_u32(sB + stage * kPairBBytes), mb, fb_leader, 0,
                               kb * kGemmBK, n * 4 + static_cast<int>(rank) * 2);
          }
          __syncwarp();
          // A of item j's first H chunk / Z tile waits for its LN2 / whole
          // hidden (of a shared item: also the partner's half of the hidden)
          if (kb == 0 && n == n0 && ph > 0) {
            if (!mbar_wait_warp(ph == 1 ? v_ready : h_ready, static_cast<uint32_t>(j & 1),
                                abort_flag, p.err, kSiteGemmProducer)) {
              ok = false;
              break;
            }
            if (ph == 2 && hf >= 0) {
              if (!flag_wait_warp(p.flags + tail_flag(1, pl.partner, rank), kTailEpi,
                                  abort_flag, p.err, kSiteTailPartner)) {
                ok = false;
                break;
              }
              fence_proxy_async_global();
            }
          }
          // K blocks of a shared item's Z tile in the partner's half of d_ff
          // read the partner's hidden rows
          const bool theirs = ph == 2 && hf >= 0 && (kb >= kbs / 2 ? 1 : 0) != hf;
          const bool lost = p.fault == 3 && pair == 0 && rank == 0 && sg == 0 && n == 0 &&
                            kb == 0;
          if (leader && !lost)
            tma_load_3d_pair(smem_u32(sA + stage * kPairABytes), ma, fb_leader, 0,
                             theirs ? scr_row_partner : a_row, wide ? kb : kb * 2);
          __syncwarp();
          if (++stage == kPairStages) {
            stage = 0;
            phase_bit ^= 1u;
          }
        }
      }
    }
    const bool aborted = !ok;
    // Drain (as in the pair GEMM): the leader waits for every phase it armed;
    // after an abort the peer gives its loads a bounded 200 us.  A stage whose
    // A load was skipped by an abort never completes: its drain wait runs out
    // (bounded) and records the drain site.
    if (rank == 0) {
      for (int s2 = 0; s2 < kPairStages; ++s2)
        if (armed[s2] >= 0) mbar_wait_drain(full0 + 8 * s2, static_cast<uint32_t>(armed[s2]), p.err);
    } else if (aborted || *abort_flag) {
      const uint64_t t0 = global_ns();
      while (global_ns() - t0 < 200000ull) {
      }
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------ UMMA issue (leader)
    const bool leader = elect_one();
    constexpr uint32_t idesc = idesc_f16_f32(kPairBM, kGemmBN, false, true);
    int stage = 0;
    uint32_t phase_bit = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    auto next_slot = [&]() {
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    };
    for (int sg = 0; sg < n_seg && ok; ++sg) {
      int ph, j;
      tail_segment(sg, J, ph, j);
      const bool wide = ph == 2 && sh.e512;
      const int kbs = sh.kblocks(ph);
      const int tiles = ph == 0 ? sh.nB : (ph == 1 ? sh.nD : sh.nE);
      int n0, n1;
      tail_range(tiles, pl.half_of(j), n0, n1);
      for (int n = n0; n < n1 && ok; ++n) {
        // accumulator slots: one, or two consecutive for a 512-column tile
        const int s0 = acc;
        const uint32_t p0 = acc_phase;
        next_slot();
        const int s1 = acc;
        const uint32_t p1 = acc_phase;
        if (wide) next_slot();
        if (!mbar_wait_warp(acce0 + 8 * s0, p0 ^ 1u, abort_flag, p.err, kSiteGemmMma) ||
            (wide && !mbar_wait_warp(acce0 + 8 * s1, p1 ^ 1u, abort_flag, p.err, kSiteGemmMma))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem + static_cast<uint32_t>(s0 * kGemmBN);
        const uint32_t d1 = tmem + static_cast<uint32_t>(s1 * kGemmBN);
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait_warp(full0 + 8 * stage, phase_bit, abort_flag, p.err, kSiteGemmMma)) {
            ok = false;
            break;
          }
          const uint32_t a_lo = sdesc_lo(smem_u32(sA + stage * kPairABytes), 16);
          constexpr uint32_t hi = sdesc_hi(1024);
          if (leader) {
            if (wide) {
              // A: one 64-column chunk (four 16-deep k-steps of 32 bytes); B:
              // [4 chunks][64 K rows][64], instruction i on chunks 2i, 2i+1
              const uint32_t b0 = sdesc_lo(smem_u32(sB + stage * kPairBBytes), 8192);
              const uint32_t b1 = sdesc_lo(smem_u32(sB + stage * kPairBBytes + 16384), 8192);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
                umma_ss_pair(d0, a_lo + 2u * k, hi, b0 + 128u * k, hi, idesc, accum);
                umma_ss_pair(d1, a_lo + 2u * k, hi, b1 + 128u * k, hi, idesc, accum);
              }
            } else {
              const uint32_t b_lo =
                  sdesc_lo(smem_u32(sB + stage * kPairBBytes), kPairBBytes / 2);
#pragma unroll
              for (int k = 0; k < kGemmBK / 16; ++k)
                umma_ss_pair(d0, a_lo + (k >> 2) * ((kPairABytes / 2) >> 4) + 2u * (k & 3), hi,
                             b_lo + 128u * k, hi, idesc, (kb | k) != 0 ? 1u : 0u);
            }
            umma_commit_pair_mc(empty0 + 8 * stage, 0x3);
          }
          __syncwarp();
          if (++stage == kPairStages) {
            stage = 0;
            phase_bit ^= 1u;
          }
        }
        if (!ok) break;
        if (leader) {
          umma_commit_pair_mc(accf0 + 8 * s0, 0x3);
          if (wide) umma_commit_pair_mc(accf0 + 8 * s1, 0x3);
        }
        __syncwarp();
      }
    }
    if (leader) umma_commit_pair(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // ------------------------------------------- epilogue (both CTAs)
    const int ew = warp - 4;                       // 0..7
    const int e = warp & 3;                        // TMEM lane quarter
    constexpr int kCols = kGemmBN * 4 / kTailEpi;  // 128 columns per warp
    const int part = ew >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    const int s_base = static_cast<int>(rank) * 128;
    const long long v_row0 = static_cast<long long>(pair) * 256 + s_base;
    bool ok = true;
    for (int sg = 0; sg < n_seg && ok; ++sg) {
      int ph, j;
      tail_segment(sg, J, ph, j);
      const int item = pl.item(j);
      const int hf = pl.half_of(j);
      const int m_valid = 2 * item + 1 < p.blocks ? 256 : 128;
      const RowMap map{2 * item, p.nb, p.N, 128, 0};
      GemmParams gp{};
      gp.err = p.err;
      if (ph == 1) {
        gp.epi = kEpiGeluBias;
        gp.M = 0x7fffffff;
        gp.N = p.d_ff;
        gp.out_h = p.h_scr;
        gp.ld_out = p.d_ff;
        gp.bias = p.b1;
      } else {
        gp.epi = ph == 0 ? kEpiResidX : kEpiBiasAccum;
        gp.M = m_valid;
        gp.N = p.d;
        gp.out_f32 = p.out;
        gp.ld_f32 = p.d;
        gp.resid = p.x;
        gp.ld_resid = p.d;
        gp.bias = p.b2;
        gp.map = map;
      }
      // logical 256-column tiles of the segment
      const int tiles = ph == 0 ? sh.nB : (ph == 1 ? sh.nD : (sh.e512 ? 2 * sh.nE : sh.nE));
      int n0, n1;
      tail_range(tiles, hf, n0, n1);
      for (int n = n0; n < n1 && ok; ++n) {
        int col;
        if (ph == 2 && sh.e512)
          // Z tile T = n / 2: CTA r loaded columns 512T + 256r .. +255 as B, and
          // instruction i = n % 2 took 128 of them from each CTA (TMEM columns
          // 0..127 from CTA 0, 128..255 from CTA 1): part j holds 512T + 256j + 128i
          col = (n >> 1) * 512 + part * 256 + (n & 1) * 128;
        else
          col = n * kGemmBN + part * kCols;
        if (!mbar_wait_fast(accf0 + 8 * acc, acc_phase, abort_flag, p.err, kSiteGemmEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after();
        long long row = s_base + e * 32 + lane;  // item-local row (mapped), or scratch row
        if (ph == 1) row += static_cast<long long>(pair) * 256;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(e * 32) << 16) +
                               static_cast<uint32_t>(acc * kGemmBN + part * kCols);
        gemm_epilogue_row(gp, t_row, row, col, kCols);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(map_to_rank(acce0 + 8 * acc, 0));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) break;
      if (ph == 0) {
        // every y tile of item j is stored: LN2 of the CTA's rows (of a
        // shared item, once the partner's y columns are stored too)
        if (hf >= 0) {
          __threadfence();
          __syncwarp();
          if (lane == 0) red_release_gpu_add(p.flags + tail_flag(0, pair, rank), 1u);
        }
        if (lane == 0) mbar_arrive(ep_sync);
        if (!mbar_wait_fast(ep_sync, static_cast<uint32_t>(j & 1), abort_flag, p.err,
                            kSiteGemmEpilogue)) {
          ok = false;
          break;
        }
        if (hf >= 0 && !flag_wait_warp(p.flags + tail_flag(0, pl.partner, rank), kTailEpi,
                                       abort_flag, p.err, kSiteTailPartner)) {
          ok = false;
          break;
        }
        tail_ln2(p, map, m_valid, s_base, v_row0, ew, lane);
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) mbar_arrive(v_ready);
      } else if (ph == 1) {
        // every H chunk of item j is stored (of a shared item: also for the
        // partner, whose Z tiles read this half of the hidden)
        fence_proxy_async_global();
        if (hf >= 0) __threadfence();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(h_ready);
          if (hf >= 0) red_release_gpu_add(p.flags + tail_flag(1, pair, rank), 1u);
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem, kGemmTmemCols);
}

}  // namespace bpt
