// Persistent tcgen05 GEMM with fused epilogues: C[M, N] = A[M, K] * B[K, N],
// on CTA pairs (tcgen05.mma.cta_group::2, 256 x 256 output tiles).
//
//   A: fp16 [M, K] row-major (K contiguous) -> K-major UMMA operand, 128-byte
//      swizzle.  Viewed by its tensor map as [K/64][M][64] so that one TMA
//      box brings 128 rows x 128 K (two 64-column chunks, 32 KB).
//   B: fp16 [K, N] row-major (N contiguous; weights are [d_in, d_out]) ->
//      MN-major UMMA operand, no transpose.  Viewed as [N/64][K][64]: one box
//      brings 128 K rows x 128 N (two 64-column chunks, 32 KB).  B may be the
//      column concatenation of up to three matrices with the same number of
//      columns each (W_Q | W_K | W_V); when that number is not a multiple of
//      128 a CTA's 128 columns can straddle two of them, and it loads one
//      chunk per box instead.
//   One TMA box costs a CTA ~400 clocks whatever its size (measured), so
//   boxes are 32 KB: 16 KB boxes delivered ~40 B/clk per SM, 32 KB ~75.
//   Accumulator: fp32 256 x 256 tile (128 rows per CTA) in tensor memory,
//      double buffered, so the epilogue of one tile overlaps the main loop of
//      the next.
//
// Warp roles (32 x (4 + EPI) threads per CTA): warp 0 issues TMA loads,
// warp 1 issues UMMA (leader CTA), warp 2 owns the tensor-memory allocation,
// warps 4.. run the epilogue.  With EPI = 4 warp w reads TMEM lanes
// 32(w%4)..+31 (accumulator rows of this CTA's 128) and all 256 columns; with
// EPI = 8 two warps share each lane quarter, 128 columns each.  The GELU and
// residual epilogues (W_1, W_O) use 8: their per-element work would otherwise
// outlast the next tile's main loop; the light ones use 4, whose fewer warps
// leave the TMA and UMMA warps more issue slots.
//
// Epilogues (all in fp32 before the final rounding):
//   kEpiStoreF16    out_h[row, col]  = acc                       (QKV, fp16; with
//                   split_col > 0 columns >= split_col go to out_h2, which is
//                   how a sequence shard stores Q apart from its K | V)
//   kEpiResidX      out_f32[g, col]  = x[g, col] + acc           (y = x + o W_O)
//   kEpiGeluBias    out_h[row, col]  = GELU(acc + bias[col])     (FFN hidden, fp16)
//   kEpiBiasAccum   out_f32[g, col] += acc + bias[col]           (Z = y + h W_2 + b_2)
// where g = map(row) is the residual-stream row of a scratch row; x and the
// biases are the caller's bf16 tensors.  An fp16 store of a value beyond the
// fp16 range (or NaN) is reported in the device error word.
#pragma once

#include "common.cuh"

namespace bpt {

enum GemmEpi : int {
  kEpiStoreF16 = 0,
  kEpiResidX = 1,
  kEpiGeluBias = 2,
  kEpiBiasAccum = 3,
  kEpiAccumF32 = 4,      // out_f32[row, col] += acc                      (weight gradients)
  kEpiStoreF32 = 5,      // out_f32[row, col]  = acc                      (data gradients)
  kEpiGeluGrad = 6,      // out_h[row, col]    = acc * GELU'(out_h[row, col])  (in place)
  kEpiGeluBiasKeep = 7,  // out_h2 = acc + bias[col]; out_h = GELU(out_h2)  (fp16 both)
};

// Operand layouts (K = the reduction axis):
//   kLayAkBn  A [M, K] K-contiguous, B [K, N] N-contiguous   (forward: X W)
//   kLayAnBn  A [K, M] M-contiguous, B [K, N] N-contiguous   (X^T dY: weight gradients)
//   kLayAkBk  A [M, K] K-contiguous, B [N, K] K-contiguous   (dY W^T: data gradients)
enum GemmLayout : int { kLayAkBn = 0, kLayAnBn = 1, kLayAkBk = 2 };

struct GemmParams {
  int M, N, K;     // problem size (N, K multiples of 64)
  int n_sub;       // columns of each concatenated B matrix
  int n_maps;      // B matrices in use (1..3)
  int b_chunks;    // 64-column chunks per B box: 2, or 1 if n_sub % 128 != 0
  int epi;
  __half* out_h;
  __half* out_h2;  // kEpiGeluBiasKeep: pre-activation copy (same ld as out_h);
                   // kEpiStoreF16 with split_col > 0: columns >= split_col
  long long ld_out;
  int split_col;       // kEpiStoreF16: 0, or the first column stored to out_h2
  long long ld_out2;   // row stride of out_h2 for the split store
  float* out_f32;
  long long ld_f32;
  const __nv_bfloat16* resid;
  long long ld_resid;
  const __nv_bfloat16* bias;
  RowMap map;
  uint32_t* err;
  int fault;  // test hook: 1 = CTA 0 never loads its first stage (a lost arrive)
};

constexpr int kGemmBN = 256;  // output columns per tile
constexpr int kGemmBK = 128;  // K depth of one pipeline stage
constexpr int kGemmBarrierBytes = 256;
template <int EPI>
constexpr int gemm_threads() {
  return 32 * (4 + EPI);
}
constexpr uint32_t kGemmTmemCols = 512;

// Epilogue of one accumulator row (this thread's TMEM lane): ncols columns
// starting at global column col_base, read in 32-column chunks.  Every lane of
// the warp must call it (tcgen05.ld is warp-collective).
__device__ __forceinline__ void gemm_epilogue_row(const GemmParams& p, uint32_t t_row,
                                                  long long row, int col_base, int ncols) {
  long long g = -1;
  bool row_ok;
  if (p.epi != kEpiResidX && p.epi != kEpiBiasAccum) {
    row_ok = row < p.M;
  } else {
    g = row < p.M ? p.map.map(row) : -1;
    row_ok = g >= 0;
  }
  bool bad = false;
#pragma unroll 1
  for (int ch = 0; ch < ncols / 32; ++ch) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(t_row + ch * 32, r);
    tmem_ld_wait();
    const int col0 = col_base + ch * 32;
    if (!row_ok || col0 >= p.N) continue;
    float v[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
    if (p.epi == kEpiAccumF32 || p.epi == kEpiStoreF32) {
      float4* dst = reinterpret_cast<float4*>(p.out_f32 + row * p.ld_f32 + col0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 w = make_float4(v[q * 4 + 0], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
        if (p.epi == kEpiAccumF32) {
          const float4 o = dst[q];
          w.x += o.x;
          w.y += o.y;
          w.z += o.z;
          w.w += o.w;
        }
        dst[q] = w;
      }
      continue;
    }
    if (p.epi == kEpiGeluGrad) {
      uint4* io = reinterpret_cast<uint4*>(p.out_h + row * p.ld_out + col0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 zz = io[q];
        const __half* zh = reinterpret_cast<const __half*>(&zz);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[q * 8 + k] *= gelu_erf_grad(__half2float(zh[k]));
        uint4 w;
        w.x = pack_f16x2(v[q * 8 + 0], v[q * 8 + 1], bad);
        w.y = pack_f16x2(v[q * 8 + 2], v[q * 8 + 3], bad);
        w.z = pack_f16x2(v[q * 8 + 4], v[q * 8 + 5], bad);
        w.w = pack_f16x2(v[q * 8 + 6], v[q * 8 + 7], bad);
        io[q] = w;
      }
      continue;
    }
    if (p.epi == kEpiStoreF16 || p.epi == kEpiGeluBias || p.epi == kEpiGeluBiasKeep) {
      if (p.epi == kEpiGeluBias || p.epi == kEpiGeluBiasKeep) {
        const uint4* bp = reinterpret_cast<const uint4*>(p.bias + col0);
        uint4* keep = reinterpret_cast<uint4*>(p.out_h2 + row * p.ld_out + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 bb = __ldg(bp + q);
          const __nv_bfloat16* bh = reinterpret_cast<const __nv_bfloat16*>(&bb);
#pragma unroll
          for (int k = 0; k < 8; ++k) v[q * 8 + k] += __bfloat162float(bh[k]);
          if (p.epi == kEpiGeluBiasKeep) {
            uint4 w;
            w.x = pack_f16x2(v[q * 8 + 0], v[q * 8 + 1], bad);
            w.y = pack_f16x2(v[q * 8 + 2], v[q * 8 + 3], bad);
            w.z = pack_f16x2(v[q * 8 + 4], v[q * 8 + 5], bad);
            w.w = pack_f16x2(v[q * 8 + 6], v[q * 8 + 7], bad);
            keep[q] = w;
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) v[q * 8 + k] = gelu_erf(v[q * 8 + k]);
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(p.out_h + row * p.ld_out + col0);
      if (p.epi == kEpiStoreF16 && p.split_col > 0 && col0 >= p.split_col)
        dst = reinterpret_cast<uint4*>(p.out_h2 + row * p.ld_out2 + (col0 - p.split_col));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_f16x2(v[q * 8 + 0], v[q * 8 + 1], bad);
        w.y = pack_f16x2(v[q * 8 + 2], v[q * 8 + 3], bad);
        w.z = pack_f16x2(v[q * 8 + 4], v[q * 8 + 5], bad);
        w.w = pack_f16x2(v[q * 8 + 6], v[q * 8 + 7], bad);
        dst[q] = w;
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(p.out_f32 + g * p.ld_f32 + col0);
      if (p.epi == kEpiResidX) {
        const uint4* xp = reinterpret_cast<const uint4*>(p.resid + g * p.ld_resid + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 xx = __ldg(xp + q);
          const __nv_bfloat16* xh = reinterpret_cast<const __nv_bfloat16*>(&xx);
#pragma unroll
          for (int k = 0; k < 8; ++k) v[q * 8 + k] += __bfloat162float(xh[k]);
        }
      } else {
        const uint4* bp = reinterpret_cast<const uint4*>(p.bias + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 bb = __ldg(bp + q);
          const __nv_bfloat16* bh = reinterpret_cast<const __nv_bfloat16*>(&bb);
#pragma unroll
          for (int k = 0; k < 8; ++k) v[q * 8 + k] += __bfloat162float(bh[k]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 y = dst[q];
          v[q * 4 + 0] += y.x;
          v[q * 4 + 1] += y.y;
          v[q * 4 + 2] += y.z;
          v[q * 4 + 3] += y.w;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        dst[q] = make_float4(v[q * 4 + 0], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
    }
  }
  if (bad)
    record_error(p.err, kErrRange,
                 (p.epi == kEpiGeluBias || p.epi == kEpiGeluBiasKeep || p.epi == kEpiGeluGrad)
                     ? kSiteRangeHidden
                     : kSiteRangeQKV);
}

// ---------------------------------------------------------------------------
// A cluster of two CTAs on two SMs computes one 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256).  Each CTA loads its own 128 rows of A
// and its half (128 columns) of the 256-column B slab: a 128-deep stage is
// 64 KB per CTA (one 32 KB box of A, one of B), three stages.  Each CTA's
// tensor memory holds its own 128 accumulator rows (two 256-column buffers),
// read by its own epilogue.
//
// Protocol (CTA rank 0 = leader, rank 1 = peer):
//   full[s]   leader only; the leader's producer arms it with the bytes of
//             both CTAs; both CTAs' TMA loads complete on it.
//   empty[s]  both CTAs; the leader's UMMA commit arrives on both (multicast).
//   accf[b]   both CTAs; the leader's UMMA commit arrives on both (multicast).
//   acce[b]   leader only, 2 x EPI arrivals: the epilogue warps of both CTAs.
// No TMA load uses cluster multicast.  The pair starts and ends with a
// cluster barrier, so neither CTA frees memory the other may still signal.
constexpr int kPairStages = 3;
constexpr int kPairABytes = 128 * kGemmBK * 2;  // 32 KB: this CTA's 128 rows, [2][128][64]
constexpr int kPairBBytes = kGemmBK * 128 * 2;  // 32 KB: this CTA's 128 columns, [2][128][64]
constexpr int kPairStageBytes = kPairABytes + kPairBBytes;
constexpr int kPairSmem = kPairStages * kPairStageBytes + kGemmBarrierBytes + 1024;
constexpr int kPairBM = 256;
constexpr int kPairGroupM = 8;  // 256-row blocks per rasterisation group

template <int EPI, int LAYOUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm_threads<EPI>(), 1)
    gemm_f16_pair_kernel(const __grid_constant__ CUtensorMap mapA,
                         const __grid_constant__ CUtensorMap mapB0,
                         const __grid_constant__ CUtensorMap mapB1,
                         const __grid_constant__ CUtensorMap mapB2, const GemmParams p) {
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
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(nclusters_x());
  const int m_blocks = (p.M + kPairBM - 1) / kPairBM;
  const int n_blocks = (p.N + kGemmBN - 1) / kGemmBN;
  const int k_blocks = (p.K + kGemmBK - 1) / kGemmBK;  // a half-empty last stage reads zeros
  const int tiles = m_blocks * n_blocks;

  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < kPairStages; ++s2) {
      mbar_init(full0 + 8 * s2, 1);
      mbar_init(empty0 + 8 * s2, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 2 * EPI);
    }
    mbar_init(drain, 1);
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
  bool aborted = false;

  auto coords = [&](int tile, int& mb, int& nb) {
    const int per_group = kPairGroupM * n_blocks;
    const int group = tile / per_group;
    const int first_m = group * kPairGroupM;
    const int gm = min(kPairGroupM, m_blocks - first_m);
    const int in = tile - group * per_group;
    mb = first_m + in % gm;
    nb = in / gm;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Whole warp (warp-uniform coordinates); the elected lane issues.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB0);
      if (p.n_maps > 1) tma_prefetch_desc(&mapB1);
      if (p.n_maps > 2) tma_prefetch_desc(&mapB2);
    }
    int armed[kPairStages];
    for (int s2 = 0; s2 < kPairStages; ++s2) armed[s2] = -1;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = pair; tile < tiles && ok; tile += npairs) {
      int mb, nb;
      coords(tile, mb, nb);
      // This CTA's two 64-column B chunks: which weight map, and the chunk in it.
      const CUtensorMap* bmap[2];
      int bchunk[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int c = nb * kGemmBN + static_cast<int>(rank) * 128 + q * 64;
        int which = c / p.n_sub;
        if (which > p.n_maps - 1) which = p.n_maps - 1;  // past the end: TMA zero-fills
        bmap[q] = which == 0 ? &mapB0 : (which == 1 ? &mapB1 : &mapB2);
        bchunk[q] = (c - which * p.n_sub) >> 6;
      }
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_warp(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.err, kSiteGemmProducer)) {
          ok = false;
          break;
        }
        const uint32_t fb_leader = map_to_rank(full0 + 8 * stage, 0);
        const bool lost = p.fault == 1 && pair == 0 && rank == 0 && tile == pair && kb == 0;
        if (!lost) {
          if (rank == 0) armed[stage] = static_cast<int>(phase);
          if (leader) {
            if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * stage, 2 * kPairStageBytes);
            const int m0 = mb * kPairBM + static_cast<int>(rank) * 128;
            if (LAYOUT == kLayAnBn)  // A viewed [M/64][K][64]: 128 K rows x two M chunks
              tma_load_3d_pair(smem_u32(sA + stage * kPairABytes), &mapA, fb_leader, 0,
                               kb * kGemmBK, m0 >> 6);
            else                     // A viewed [K/64][M][64]: 128 M rows x two K chunks
              tma_load_3d_pair(smem_u32(sA + stage * kPairABytes), &mapA, fb_leader, 0, m0,
                               kb * 2);
            if (LAYOUT == kLayAkBk) {  // B viewed [K/64][N][64]: 128 N rows x two K chunks
              tma_load_3d_pair(smem_u32(sB + stage * kPairBBytes), &mapB0, fb_leader, 0,
                               nb * kGemmBN + static_cast<int>(rank) * 128, kb * 2);
            } else if (p.b_chunks == 2) {
              tma_load_3d_pair(smem_u32(sB + stage * kPairBBytes), bmap[0], fb_leader, 0,
                               kb * kGemmBK, bchunk[0]);
            } else {
#pragma unroll
              for (int q = 0; q < 2; ++q)
                tma_load_3d_pair(smem_u32(sB + stage * kPairBBytes + q * (kPairBBytes / 2)),
                                 bmap[q], fb_leader, 0, kb * kGemmBK, bchunk[q]);
            }
          }
        }
        if (++stage == kPairStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    aborted = !ok;
    // Drain.  The leader waits for every phase it armed (they count the
    // peer's bytes too).  The peer cannot observe its own loads; after a
    // normal run the leader consumed them all, after an abort it waits a
    // bounded 200 us for any still in flight before the final cluster barrier.
    if (rank == 0) {
      for (int s2 = 0; s2 < kPairStages; ++s2)
        if (armed[s2] >= 0)
          mbar_wait_drain(full0 + 8 * s2, static_cast<uint32_t>(armed[s2]), p.err);
    } else if (aborted || *abort_flag) {
      const uint64_t t0 = global_ns();
      while (global_ns() - t0 < 200000ull) {
      }
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------ UMMA issue (leader)
    // Whole warp (warp-uniform descriptors); the elected lane issues.
    const bool leader = elect_one();
    constexpr bool a_mn = LAYOUT == kLayAnBn, b_mn = LAYOUT != kLayAkBk;
    constexpr uint32_t idesc = idesc_f16_f32(kPairBM, kGemmBN, a_mn, b_mn);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = pair; tile < tiles && ok; tile += npairs) {
      if (!mbar_wait_warp(acce0 + 8 * acc, acc_phase ^ 1u, abort_flag, p.err, kSiteGemmMma)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kGemmBN);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_warp(full0 + 8 * stage, phase, abort_flag, p.err, kSiteGemmMma)) {
          ok = false;
          break;
        }
        // K-major operand: two 64-K chunks 16 KB apart, a 16-deep k-step
        // moves 32 B (and the next chunk after four).  MN-major operand:
        // LBO = the 16 KB between its two 64-element chunks, a k-step moves
        // 16 rows (2 KB).
        const uint32_t a_lo =
            sdesc_lo(smem_u32(sA + stage * kPairABytes), a_mn ? kPairABytes / 2 : 16);
        const uint32_t b_lo =
            sdesc_lo(smem_u32(sB + stage * kPairBBytes), b_mn ? kPairBBytes / 2 : 16);
        constexpr uint32_t hi = sdesc_hi(1024);
        auto kstep = [](bool mn, int k) -> uint32_t {
          return mn ? 128u * k : (k >> 2) * ((kPairABytes / 2) >> 4) + 2u * (k & 3);
        };
        if (leader) {
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k)
            umma_ss_pair(d_tmem, a_lo + kstep(a_mn, k), hi, b_lo + kstep(b_mn, k), hi, idesc,
                         (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair_mc(empty0 + 8 * stage, 0x3);
        }
        __syncwarp();
        if (++stage == kPairStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (leader) umma_commit_pair_mc(accf0 + 8 * acc, 0x3);
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (leader) umma_commit_pair(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0, p.err);
  } else if (warp >= 4) {
    // ------------------------------------------- epilogue (both CTAs)
    const int e = warp & 3;                        // TMEM lane quarter
    constexpr int kCols = kGemmBN * 4 / EPI;       // columns per epilogue warp
    const int part = (warp - 4) >> 2;              // which kCols-column part
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < tiles; tile += npairs) {
      int mb, nb;
      coords(tile, mb, nb);
      if (!mbar_wait_fast(accf0 + 8 * acc, acc_phase, abort_flag, p.err, kSiteGemmEpilogue)) break;
      tc_fence_after();
      const long long row =
          static_cast<long long>(mb) * kPairBM + static_cast<long long>(rank) * 128 + e * 32 + lane;
      const uint32_t t_row = tmem + (static_cast<uint32_t>(e * 32) << 16) +
                             static_cast<uint32_t>(acc * kGemmBN + part * kCols);
      gemm_epilogue_row(p, t_row, row, nb * kGemmBN + part * kCols, kCols);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(acce0 + 8 * acc, 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem, kGemmTmemCols);
}

}  // namespace bpt
