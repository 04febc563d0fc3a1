// Blockwise attention, two query blocks per CTA (the BPT inner loop on the
// tcgen05 tensor cores).
//
// A CTA owns one head t and two consecutive query blocks of one sequence, tile
// A = block iA and tile B = block iA + 1 (B may be absent at the end of a
// sequence or of a wave).  Both tiles walk the same key/value blocks, so each
// K_j / V_j tile is loaded once into shared memory and used by both.  Per key
// block j and tile X the CTA keeps the online-softmax state of every query row
// (reference max m, running sum l, accumulator o):
//
//   S_X = Q_X K_j^T                        UMMA, fp32 in tensor memory
//   P_X = exp2(S_X * log2(e)/sqrt(d_k) - m), l = alpha l + rowsum(P_X)
//                                           softmax warpgroup X, P_X in fp16
//                                           written back over S_X in TMEM
//   O_X = alpha O_X + P_X V_j               UMMA with A = P_X from TMEM
//
// Causal: tile X visits blocks j <= iX only (blocks above the diagonal are
// never loaded or scored) and masks keys after the query on its diagonal
// block.  Non-causal: a ragged last key block masks keys >= N.
// The reference max moves only when a row's maximum grows by more than 2^8 in
// exp2 units; then O_X is rescaled by alpha = exp2(m_old - m_new).  Smaller
// growth keeps the old reference (exact: o / l does not depend on it; P stays
// <= 2^8).
//
// Ping-pong: the UMMA warp issues PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), ...
// so the tensor core works on one tile while the other tile's softmax runs.
// tcgen05.mma issued by one thread executes in order, so S_X(j+1) overwriting
// the TMEM that P_X(j) occupies is ordered after PV_X(j) has read it.
//
// exp2: most elements use the MUFU ex2 instruction; on blocks with no masked
// key, EMU of the eight 16-column groups of each row use a cubic on the FMA
// pipe instead, so MUFU and FMA share the work: 2^x = 2^n * 2^f with
// n = round(x) (the 1.5 * 2^23 addition trick, no conversion instruction),
// f = x - n in [-1/2, 1/2], 2^f from a fitted cubic (relative error 7.5e-5,
// below the fp16 resolution of P), and n added to the exponent field.

// Shared memory: Q_A, Q_B and a ring of NSLOT K/V tiles (loaded K_0, V_0,
// K_1, V_1, ...), all 128 rows x d_k fp16 in 64-column chunks with the
// 128-byte swizzle.  Tensor memory: S_A 0..127, S_B 128..255, O_A 256..,
// O_B 256+d_k...
//
// Warp roles (384 threads): 0 TMA, 1 UMMA issue, 2 TMEM owner, 3 idle,
// 4..7 softmax of tile A, 8..11 softmax of tile B (thread = query row).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace bpt {

struct AttnPairParams {
  int N;       // tokens per sequence
  int nb;      // query blocks per sequence
  int h;       // heads
  int d;       // model width (row stride of Q, K and V is 3d)
  int causal;
  int item0;   // first flattened block item (batch * nb + block) of the wave
  int count;   // block items in the wave
  int seqs;    // >0: the wave is `seqs` whole sequences; 0: part of one sequence
  int hg;      // heads per group (divides h): CTAs run group by group, so the
               // K/V that concurrent CTAs sweep is that of hg heads only
  __half* o;         // output, fp16: o_tok = 0: [count * 128, o_ld] block
                     // scratch in wave order; o_tok = 1: [B*N, o_ld] token
                     // rows (the Q columns of the QKV buffer: each block's
                     // output replaces its own queries; rows past N are not
                     // written)
  long long o_ld;    // row stride of o (elements)
  int o_tok;
  float scale_log2;  // log2(e) / sqrt(d_k)
  float2* stats;     // nullable: per-row softmax statistics [B][h][N] (m, l)
  uint32_t* err;
  int fault;         // test hook: 2 = CTA 0 never loads V_0 (a lost arrive)
  int qpc;           // query blocks per CTA: 2 (a pair, 256 query rows sharing
                     // each K/V tile) or 1 (one 128-row block)
  // Sequence shard (kernel instantiated with SHARD only).  The sequence of
  // N_kv tokens is cut into 2G chunks of kv_cb query/key blocks; this rank
  // owns chunks q_c0 and q_c1 (its local blocks 0..kv_cb-1 and kv_cb..2kv_cb-1).
  // Q, o and the block indices above are local; keys come from the all-gathered
  // K | V of every rank, [G][B][N / G][2d], where chunk c is held by rank
  // c < G ? c : 2G-1-c as its local chunk c < G ? 0 : 1.
  int kv_cb, q_c0, q_c1, kv_G, N_kv;
  // Block gating (attn_gate_tc_kernel only):
  const float* gate_t;  // [h][nb] thresholds T in units of s = q.k / sqrt(d_k)
  float* gate_bmax;     // nullable [B][h][nb][nb]: s_max of each visited pair
  uint8_t* gate_kept;   // nullable [B][h][nb][nb]: 1 processed, 0 pruned
};


#ifndef BPT_FWD_HANDOVERS_DK128
#define BPT_FWD_HANDOVERS_DK128 2
#endif
#ifndef BPT_FWD_HANDOVERS_DK64
#define BPT_FWD_HANDOVERS_DK64 4
#endif
// P hand-overs per 128-key tile from a softmax warpgroup to the UMMA warp
// (4: every 32 keys; 2: every 64).  Measured: every 64 keys is faster at
// d_k = 128 (each wait costs the UMMA warp ~100 clocks), every 32 at d_k =
// 64 (shorter PV products, earlier overlap matters more).
template <int D>
constexpr int fwd_handovers() {
  return D == 128 ? BPT_FWD_HANDOVERS_DK128 : BPT_FWD_HANDOVERS_DK64;
}
static_assert(BPT_FWD_HANDOVERS_DK128 == 2 || BPT_FWD_HANDOVERS_DK128 == 4, "2 or 4");
static_assert(BPT_FWD_HANDOVERS_DK64 == 2 || BPT_FWD_HANDOVERS_DK64 == 4, "2 or 4");

template <int D, int EMU>
struct AttnPairCfg {
  static constexpr int BQ = 128;
  static constexpr int BKV = 128;
  static constexpr int TILE = 128 * D * 2;   // one Q, K or V tile
  static constexpr int CHUNK = 128 * 128;    // one 64-column swizzled chunk (16 KB)
  static constexpr int NSLOT = (D == 128) ? 5 : 10;
  static constexpr int OFF_QA = 0;
  static constexpr int OFF_QB = TILE;
  static constexpr int OFF_RING = 2 * TILE;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * TILE;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S_B = 128;
  static constexpr uint32_t TM_O_A = 256;
  static constexpr uint32_t TM_O_B = 256 + D;
  static constexpr int THREADS = 384;
};

// Work rank -> first block item of the CTA's query blocks (qpc of them) and
// whether its second block exists.  Causal work is handed out longest first
// (descending query block).
__device__ __forceinline__ void attn_pair_decode(const AttnPairParams& p, int rank, int& itemA,
                                                 bool& has_b) {
  const int w = p.qpc;
  if (p.seqs == 0) {
    const int nunits = (p.count + w - 1) / w;
    const int q = p.causal ? (nunits - 1 - rank) : rank;
    itemA = p.item0 + w * q;
    has_b = w == 2 && 2 * q + 1 < p.count;
  } else {
    const int pp = (p.nb + w - 1) / w;  // units per sequence
    int s, q;
    if (p.causal) {
      q = pp - 1 - rank / p.seqs;
      s = rank % p.seqs;
    } else {
      s = rank / pp;
      q = rank % pp;
    }
    itemA = p.item0 + s * p.nb + w * q;
    has_b = w == 2 && 2 * q + 1 < p.nb;
  }
}

// XP: work rank -> the first block item of the cluster's four query blocks
// and how many of them exist (1..4).  Longest first, as attn_pair_decode.
__device__ __forceinline__ void attn_quad_decode(const AttnPairParams& p, int rank, int& item0q,
                                                 int& nq) {
  if (p.seqs == 0) {
    const int nunits = (p.count + 3) / 4;
    const int q = p.causal ? (nunits - 1 - rank) : rank;
    item0q = p.item0 + 4 * q;
    nq = min(4, p.count - 4 * q);
  } else {
    const int pp = (p.nb + 3) / 4;  // units per sequence
    int s, q;
    if (p.causal) {
      q = pp - 1 - rank / p.seqs;
      s = rank % p.seqs;
    } else {
      s = rank / pp;
      q = rank % pp;
    }
    item0q = p.item0 + s * p.nb + 4 * q;
    nq = min(4, p.nb - 4 * q);
  }
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 16-column groups (of eight per 128-key row) whose exp2 runs on the FMA
// pipe, as a bit mask, spread over the row.
__host__ __device__ constexpr uint32_t emu_group_mask(int emu) {
  return emu <= 0 ? 0x00u : emu == 1 ? 0x80u : emu == 2 ? 0x88u : emu == 3 ? 0xA8u
       : emu == 4 ? 0xAAu : emu == 5 ? 0xBAu : emu == 6 ? 0xEEu : emu == 7 ? 0xFEu : 0xFFu;
}

__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// 32 lanes x 8 columns (the O rescale: few registers, since the scores are
// still live when it runs).
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Global block of local query block i on a sequence shard.
__device__ __forceinline__ int shard_global_block(const AttnPairParams& p, int i) {
  return (i < p.kv_cb ? p.q_c0 : p.q_c1) * p.kv_cb + (i % p.kv_cb);
}

// XP: b = 512.  A cluster of two CTAs takes four consecutive query blocks
// (two per CTA) and shares every K/V tile: each CTA TMA-loads one 64-key half
// of each tile from L2 (mapKV: 64-row boxes of QKV) and copies it into the
// partner's ring slot over DSMEM (a shared-to-shared bulk copy; no multicast
// load), so each K/V byte fetched from L2 serves 512 query rows.  The
// products stay per CTA (same arithmetic as b = 256).  Ring barriers then
// count both CTAs: a slot is full when the own half has landed (the copier
// warp's arrive) and the partner's copy has (its bytes), and empty when both
// CTAs' UMMA warps have released it (multicast commit).  Both CTAs walk the
// key blocks of all four query blocks.
template <int D, int EMU, bool SHARD = false, bool XP = false>
__global__ void __launch_bounds__(384, 1)
    attn_pair_tc_kernel(const __grid_constant__ CUtensorMap mapQKV,
                        const __grid_constant__ CUtensorMap mapKV, const AttnPairParams p) {
  static_assert(!(XP && SHARD), "the b = 512 pair is unsharded");
  using C = AttnPairCfg<D, EMU>;
  constexpr int kFwdHandovers = fwd_handovers<D>();
  constexpr int kFwdChunksPerHand = 4 / kFwdHandovers;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t ring_full0 = smem_u32(bars + 1);
  const uint32_t ring_empty0 = smem_u32(bars + 1 + C::NSLOT);
  const uint32_t s_full0 = smem_u32(bars + 1 + 2 * C::NSLOT);   // [A, B]
  // [A: chunks 0..3, B: chunks 0..3]: P columns 32c.. of the tile handed over
  const uint32_t p_chunk0 = smem_u32(bars + 3 + 2 * C::NSLOT);
  const uint32_t o_done0 = smem_u32(bars + 11 + 2 * C::NSLOT);  // [A, B]
  const uint32_t drain = smem_u32(bars + 13 + 2 * C::NSLOT);
  const uint32_t half0 = smem_u32(bars + 14 + 2 * C::NSLOT);  // XP: own half landed
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx -> (head group, work rank, head): within a group, consecutive
  // CTAs (XP: clusters) take the group's heads for one rank, longest ranks
  // first.
  int itemA, head;
  bool has_b;
  int xr = 0;         // XP: rank in the cluster
  bool has_a = true;  // XP: the CTA has query blocks
  int last_item = 0;  // XP: the last block item of the cluster's four
  if constexpr (XP) {
    xr = int(blockIdx.x & 1);
    const int cl = int(blockIdx.x >> 1);
    const int per_group = int(gridDim.x / 2 / p.h) * p.hg;
    const int grp = cl / per_group;
    const int in_grp = cl - grp * per_group;
    const int rank = in_grp / p.hg;
    head = grp * p.hg + (in_grp - rank * p.hg);
    int item0q, nq;
    attn_quad_decode(p, rank, item0q, nq);
    has_a = 2 * xr < nq;
    has_b = 2 * xr + 1 < nq;
    itemA = has_a ? item0q + 2 * xr : item0q;
    last_item = item0q + nq - 1;
  } else {
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
  // global block positions (for the causal range and the diagonal) and the
  // key blocks of the whole sequence
  const int gA = SHARD ? shard_global_block(p, iA) : iA;
  const int gB = SHARD ? shard_global_block(p, iB) : iB;
  const int nb_kv = SHARD ? p.N_kv / C::BKV : p.nb;
  const int nA = XP && !has_a ? 0 : (p.causal ? gA + 1 : nb_kv);
  const int nB = has_b ? (p.causal ? gB + 1 : nb_kv) : 0;
  // key blocks the ring carries: this CTA's, or (XP) the cluster's
  int n_kv = nA > nB ? nA : nB;
  if constexpr (XP) n_kv = p.causal ? last_item - bidx * p.nb + 1 : nb_kv;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(ring_full0 + 8 * s, XP ? 2 : 1);
      mbar_init(ring_empty0 + 8 * s, XP ? 2 : 1);
      if constexpr (XP) mbar_init(half0 + 8 * s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full0 + 8 * x, 1);
      for (int c = 0; c < 4; ++c) mbar_init(p_chunk0 + 8 * (4 * x + c), 4);
      mbar_init(o_done0 + 8 * x, 1);
    }
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
  if constexpr (XP) cluster_sync();  // the partner's barriers exist before any copy
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;
  const int colQ = head * D, colK = p.d + head * D, colV = 2 * p.d + head * D;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the role (warp-uniform coordinates); the elected
    // lane issues the TMA loads.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&mapQKV);
      if constexpr (SHARD) tma_prefetch_desc(&mapKV);
    }
    int armed[C::NSLOT];
    for (int s = 0; s < C::NSLOT; ++s) armed[s] = -1;
    if (leader) {
      if constexpr (XP) {
        mbar_arrive_expect_tx(q_full, C::TILE * ((has_a ? 1 : 0) + (has_b ? 1 : 0)));
        if (has_a)
          tma_load_4d(smem_u32(smem + C::OFF_QA), &mapQKV, q_full, 0, iA * C::BQ, colQ / 64,
                      bidx);
      } else {
        mbar_arrive_expect_tx(q_full, C::TILE * (has_b ? 2 : 1));
        tma_load_4d(smem_u32(smem + C::OFF_QA), &mapQKV, q_full, 0, iA * C::BQ, colQ / 64, bidx);
      }
      if (has_b)
        tma_load_4d(smem_u32(smem + C::OFF_QB), &mapQKV, q_full, 0, iB * C::BQ, colQ / 64, bidx);
    }
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    if constexpr (XP) {
      // this CTA's 64-key half of every K/V tile: one 8 KB box per 64-column
      // chunk (rows 64 xr .. of the chunk); the partner's half arrives by copy
      int armed_h[C::NSLOT];
      for (int s = 0; s < C::NSLOT; ++s) armed_h[s] = -1;
      for (int t = 0; t < 2 * n_kv && ok; ++t) {
        const int j = t >> 1, w = t & 1;
        if (!mbar_wait_warp(ring_empty0 + 8 * slot, phase ^ 1u, abort_flag, p.err,
                            kSiteAttnProducer)) {
          ok = false;
          break;
        }
        armed[slot] = static_cast<int>(phase);
        armed_h[slot] = static_cast<int>(phase);
        if (leader) {
          mbar_arrive_expect_tx(ring_full0 + 8 * slot, C::TILE / 2);  // the partner's half
          mbar_arrive_expect_tx(half0 + 8 * slot, C::TILE / 2);
          const int col = w == 0 ? colK : colV;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(smem_u32(smem + C::OFF_RING + slot * C::TILE + c * C::CHUNK + xr * 8192),
                        &mapKV, half0 + 8 * slot, 0, j * C::BKV + xr * 64, col / 64 + c, bidx);
        }
        __syncwarp();
        if (++slot == C::NSLOT) {
          slot = 0;
          phase ^= 1u;
        }
      }
      for (int s = 0; s < C::NSLOT; ++s)
        if (armed_h[s] >= 0) mbar_wait_drain(half0 + 8 * s, static_cast<uint32_t>(armed_h[s]), p.err);
    } else {
      // ring order K_0 V_0 K_1 V_1 ...
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int w = 0; w < 2; ++w) {
          if (!mbar_wait_warp(ring_empty0 + 8 * slot, phase ^ 1u, abort_flag, p.err,
                              kSiteAttnProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb = ring_full0 + 8 * slot;
          const bool lost = p.fault == 2 && blockIdx.x == 0 && j == 0 && w == 1;
          if (!lost) {
            armed[slot] = static_cast<int>(phase);
            if (leader) {
              mbar_arrive_expect_tx(fb, C::TILE);
              if constexpr (SHARD) {
                // key block j of the sequence: its owner rank and local block
                const int c = j / p.kv_cb;
                const int owner = c < p.kv_G ? c : 2 * p.kv_G - 1 - c;
                const int lb = (c < p.kv_G ? 0 : p.kv_cb) + (j - c * p.kv_cb);
                const int col = w == 0 ? head * D : p.d + head * D;  // in K | V
                tma_load_5d(smem_u32(smem + C::OFF_RING + slot * C::TILE), &mapKV, fb, 0,
                            lb * C::BKV, col / 64, bidx, owner);
              } else {
                const int col = w == 0 ? colK : colV;
                tma_load_4d(smem_u32(smem + C::OFF_RING + slot * C::TILE), &mapQKV, fb, 0,
                            j * C::BKV, col / 64, bidx);
              }
            }
          }
          if (++slot == C::NSLOT) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
    }
    mbar_wait_drain(q_full, 0, p.err);
    for (int s = 0; s < C::NSLOT; ++s)
      if (armed[s] >= 0) mbar_wait_drain(ring_full0 + 8 * s, static_cast<uint32_t>(armed[s]), p.err);
  } else if (XP && warp == 3) {
    // ------------------------------------------- XP: copy own halves across
    const bool leader = elect_one();
    const uint32_t peer = static_cast<uint32_t>(xr ^ 1);
    int slot = 0;
    uint32_t phase = 0;
    for (int t = 0; t < 2 * n_kv; ++t) {
      if (!mbar_wait_warp(half0 + 8 * slot, phase, abort_flag, p.err, kSiteAttnProducer)) break;
      if (leader) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const uint32_t off = C::OFF_RING + slot * C::TILE + c * C::CHUNK + xr * 8192;
          bulk_copy_to_peer(map_to_rank(smem_u32(smem + off), peer), smem_u32(smem + off), 8192,
                            map_to_rank(ring_full0 + 8 * slot, peer));
        }
        mbar_arrive(ring_full0 + 8 * slot);  // own half landed
      }
      __syncwarp();
      if (++slot == C::NSLOT) {
        slot = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- UMMA issue
    // The whole warp runs the role so that descriptors stay warp-uniform; the
    // elected lane issues each MMA and commit (issuing from one lane with
    // per-lane descriptors cost ~100 clocks per MMA, above the 64 of an
    // M128 N128 K16 MMA).
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_f16_f32(C::BQ, C::BKV, false, false);
    constexpr uint32_t idesc_o = idesc_f16_f32(C::BQ, D, false, true);
    const uint32_t sQA = smem_u32(smem + C::OFF_QA);
    const uint32_t sQB = smem_u32(smem + C::OFF_QB);
    const uint32_t ring = smem_u32(smem + C::OFF_RING);
    auto slot_of = [&](int t) { return t % C::NSLOT; };
    auto phase_of = [&](int t) { return static_cast<uint32_t>((t / C::NSLOT) & 1); };
    // Descriptor words: Q_A, Q_B fixed; K/V per ring slot.  A k-step adds a
    // constant to the low word (start address >> 4).
    constexpr uint32_t hi = sdesc_hi(1024);
    const uint32_t qa_lo = sdesc_lo(sQA, 16), qb_lo = sdesc_lo(sQB, 16);
    auto issue_s = [&](uint32_t q_lo, uint32_t k_lo, uint32_t d_tmem) {
      if (leader) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::CHUNK + (k & 3) * 32) >> 4;
          umma_ss(d_tmem, q_lo + off, hi, k_lo + off, hi, idesc_s, k > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    // the two 16-key k-steps of PV for keys 32c..32c+31 (P packed: 16
    // columns per 32 keys); `first` = O not yet written by this tile
    auto issue_pv_chunk = [&](uint32_t tP, uint32_t v_lo, uint32_t d_tmem, int c, bool first) {
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int k = 2 * c + kk;
          umma_ts(d_tmem, tP + 8 * k, v_lo + ((k * 2048) >> 4), hi, idesc_o,
                  (!first || k > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    auto commit = [&](uint32_t bar) {
      if (leader) umma_commit(bar);
      __syncwarp();
    };
    // a ring slot is released to both CTAs of an XP cluster
    auto release = [&](uint32_t bar) {
      if (leader) {
        if constexpr (XP)
          umma_commit_mc(bar, 0x3);
        else
          umma_commit(bar);
      }
      __syncwarp();
    };
    uint32_t pph[2] = {0, 0};
    bool o_started[2] = {false, false};  // first PV of a tile overwrites O
    bool ok = mbar_wait_warp(q_full, 0, abort_flag, p.err, kSiteAttnMma);
    if (ok)
      ok = mbar_wait_warp(ring_full0 + 8 * slot_of(0), phase_of(0), abort_flag, p.err,
                          kSiteAttnMma);
    if (ok) {
      tc_fence_after();
      const uint32_t k0_lo = sdesc_lo(ring + slot_of(0) * C::TILE, 16);
      if (nA > 0) {
        issue_s(qa_lo, k0_lo, tmem);
        commit(s_full0);
      }
      if (nB > 0) {
        issue_s(qb_lo, k0_lo, tmem + C::TM_S_B);
        commit(s_full0 + 8);
      }
      release(ring_empty0 + 8 * slot_of(0));
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      // ring positions of K_j+1 and V_j (see the producer's order)
      const int tk = 2 * (j + 1);
      const int tv = 2 * j + 1;
      bool k_ready = false;
      if (!mbar_wait_warp(ring_full0 + 8 * slot_of(tv), phase_of(tv), abort_flag, p.err,
                          kSiteAttnMma))
        break;
      const uint32_t v_lo = sdesc_lo(ring + slot_of(tv) * C::TILE, C::CHUNK);
      const uint32_t k_lo = sdesc_lo(ring + slot_of(tk) * C::TILE, 16);
      for (int x = 0; x < 2 && ok; ++x) {
        const int nX = x == 0 ? nA : nB;
        if (j >= nX) continue;
        const uint32_t tS = tmem + (x == 0 ? 0u : C::TM_S_B);
        const uint32_t tO = tmem + (x == 0 ? C::TM_O_A : C::TM_O_B);
        // PV_X(j) as the P hand-overs come (each 128 / kFwdHandovers keys)
        for (int hh = 0; hh < kFwdHandovers; ++hh) {
          if (!mbar_wait_warp(p_chunk0 + 8 * (4 * x + hh), pph[x], abort_flag, p.err,
                              kSiteAttnMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int q = 0; q < kFwdChunksPerHand; ++q)
            issue_pv_chunk(tS, v_lo, tO, hh * kFwdChunksPerHand + q, !o_started[x]);
        }
        if (!ok) break;
        pph[x] ^= 1u;
        o_started[x] = true;
        if (j + 1 < nX) {
          if (!k_ready) {
            if (!mbar_wait_warp(ring_full0 + 8 * slot_of(tk), phase_of(tk), abort_flag, p.err,
                                kSiteAttnMma)) {
              ok = false;
              break;
            }
            // (TMA data: ordered by the mbarrier wait itself)
            k_ready = true;
          }
          issue_s(x == 0 ? qa_lo : qb_lo, k_lo, tS);
          commit(s_full0 + 8 * x);
        } else {
          commit(o_done0 + 8 * x);
        }
      }
      if (!ok) break;
      if (XP && !k_ready && j + 1 < n_kv) {
        // the cluster's ring goes on past this CTA's blocks: consume K_j+1
        if (!mbar_wait_warp(ring_full0 + 8 * slot_of(tk), phase_of(tk), abort_flag, p.err,
                            kSiteAttnMma))
          break;
        k_ready = true;
      }
      release(ring_empty0 + 8 * slot_of(tv));
      if (k_ready) release(ring_empty0 + 8 * slot_of(tk));
    }
    commit(drain);
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int x = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const int e = warp & 3;         // TMEM lane quarter
    const int r = e * 32 + lane;    // query row within the tile
    const int nX = x == 0 ? nA : nB;
    const int iX = x == 0 ? iA : iB;
    const int gX = x == 0 ? gA : gB;  // global block (the diagonal)
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(e * 32) << 16);
    const uint32_t tS = t_lane + (x == 0 ? 0u : C::TM_S_B);
    const uint32_t tO = t_lane + (x == 0 ? C::TM_O_A : C::TM_O_B);
    const uint32_t s_full = s_full0 + 8 * x, o_done = o_done0 + 8 * x;
    const uint32_t p_chunk = p_chunk0 + 8 * (4 * x);  // [4]
    const float c = p.scale_log2;
    const bool ragged = !SHARD && (p.N % C::BKV) != 0;
    float m_run = -INFINITY;  // reference maximum (moves only by > 2^8 in exp2 units)
    float m_true = -INFINITY;  // exact running row maximum, for the statistics
    float l = 0.f;
    bool o_live = false;       // O holds a PV product
    bool ok = nX > 0;
    for (int j = 0; j < nX && ok; ++j) {
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
      const bool masked = p.causal ? (j == gX) : (ragged && j == p.nb - 1);
      if (masked) {
        const int lim = p.causal ? r + 1 : p.N - j * C::BKV;
#pragma unroll
        for (int k = 0; k < C::BKV; ++k)
          if (k >= lim) sr[k] = __float_as_uint(-INFINITY);
      }
      // Row max as eight independent partial maxima (short dependency chains),
      // three-input max over columns k + q and k + 8 + q.
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
      // Rescale O first: the PV of this block starts with its first P
      // chunk (PV_X(j-1) is complete: S_X(j), issued after it, has landed).
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
      }
      const float2 cc2 = make_float2(c, c);
      const float2 mref2 = make_float2(-m_new * c, -m_new * c);
      float2 sum2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
      // One unrolled loop per tile kind, so the MUFU / FMA choice of each
      // 16-column group is fixed at compile time (no per-element branch).
      // Each 32-key chunk of P is handed over as soon as it is stored.
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
          tmem_st_32x32b_x16(tS + cc * 16, pk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && (cc + 1) % kFwdChunksPerHand == 0)
            mbar_arrive(p_chunk + 8 * (cc / kFwdChunksPerHand));
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
    if (ok && mbar_wait_fast(o_done, 0, abort_flag, p.err, kSiteAttnSoftmax)) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      if (p.stats != nullptr) {
        // (m, l) of the row in the units of s = q.k / sqrt(d_k): m the exact
        // maximum over its allowed keys, l = sum exp(s - m) (l was kept
        // relative to the reference maximum m_run <= m_true).
        const int pos = iX * C::BQ + r;
        if (pos < p.N) {
          const float m_s = m_true * p.scale_log2 * 0.69314718055994531f;
          const float l_s = l * ex2_approx((m_run - m_true) * p.scale_log2);
          p.stats[(static_cast<long long>(bidx) * p.h + head) * p.N + pos] = make_float2(m_s, l_s);
        }
      }
      long long orow;
      bool store = true;
      if (p.o_tok) {
        const int pos = iX * C::BQ + r;
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
  if constexpr (XP) cluster_sync();  // no copy into a CTA that has left
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace bpt
