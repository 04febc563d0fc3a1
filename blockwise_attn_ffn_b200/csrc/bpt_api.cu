// libbpt host side: argument validation, workspace layout, TMA descriptors and
// the launch sequence of one BPT layer forward.
//
// Schedule ("Blockwise Parallel Transformer — BPT", sections "The fused
// blockwise algorithm" and "Why parallel is in the name"): the outer loop over
// query blocks is embarrassingly parallel, and P concurrent blocks cost
// P x O(b d) of transient memory.  Before the loop: the bf16 -> fp16 weight
// copy, LN1 (into out, reused as scratch) and the QKV GEMM.  Then, for bf16
// layers (the fused schedule, default):
//   attention (online softmax over K/V blocks) -> o over each block's Q rows
//   tail kernel: per query block, W_O + x, LN2, W_1 + b_1 + GELU chunk by
//   chunk, W_2 + b_2 + y  (tail_tc.cuh; scratch per CTA pair)
// or (the waves schedule, and fp32 layers) waves of up to BPT_WAVE_BLOCKS
// query blocks, each running five stream-ordered kernels whose
// intermediates are wave-shaped:
//   attention                                   -> o      [P b, d]
//   W_O GEMM, epilogue + x                      -> y      (into out rows)
//   LN2                                         -> v      [P b, d]
//   W_1 GEMM, epilogue + b_1, GELU              -> H      [P b, d_ff]
//   W_2 GEMM, epilogue + b_2 + y                -> Z      (into out rows)
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "bpt.h"
#include "attn_bwd_tc.cuh"
#include "attn_pair_tc.cuh"
#include "attn_b64_tc.cuh"
#include "attn_gate_tc.cuh"
#include "backward.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "rows.cuh"
#include "simt_f32.cuh"
#include "tail_tc.cuh"
#include "backward_f32.cuh"

namespace {

using bpt::RowMap;

constexpr int64_t kMaxWave = BPT_WAVE_BLOCKS;
static_assert(BPT_TAIL_MAX_PAIRS == bpt::kTailMaxPairs, "tail pairs");

// Per-call options (bpt_options), validated, defaults filled in.
struct Opts {
  int fused = 1;             // bf16 forward: fused tail (1) or waves (0)
  int qpc = 2;               // 128-row query blocks per attention CTA (b / 128)
  int b64 = 0;               // b = 64: one 64-row query block per CTA
  int64_t max_wave = kMaxWave;
  int fault = 0;             // test hook
};

bpt_status read_opts(const bpt_options* o, Opts* r) {
  *r = Opts{};
  if (o == nullptr) return BPT_OK;
  if (o->reserved != 0) return BPT_ERR_INVALID_ARG;
  if (o->schedule != BPT_SCHEDULE_FUSED && o->schedule != BPT_SCHEDULE_WAVES)
    return BPT_ERR_INVALID_ARG;
  if (o->attn_block != 0 && o->attn_block != 64 && o->attn_block != 128 &&
      o->attn_block != 256 && o->attn_block != 512)
    return BPT_ERR_INVALID_ARG;
  if (o->max_wave < 0 || o->max_wave > kMaxWave) return BPT_ERR_INVALID_ARG;
  if (o->fault < 0 || o->fault > 3) return BPT_ERR_INVALID_ARG;
  r->fused = o->schedule == BPT_SCHEDULE_FUSED ? 1 : 0;
  const int b = o->attn_block == 0 ? 256 : o->attn_block;
  r->b64 = b == 64 ? 1 : 0;
  r->qpc = b == 64 ? 1 : b / 128;
  r->max_wave = o->max_wave == 0 ? kMaxWave : o->max_wave;
  r->fault = o->fault;
  return BPT_OK;
}
// 16-column groups (of eight per 128-key row) whose exp2 runs on the FMA
// pipe instead of MUFU (compile-time tuning knobs; 2 of 8 measured fastest).
#ifndef BPT_EMU_DK128
#define BPT_EMU_DK128 2
#endif
#ifndef BPT_EMU_DK64
#define BPT_EMU_DK64 2
#endif
// Attention CTAs run head group by head group; a group is the largest
// divisor of h whose K/V (all keys of the wave) fits this many bytes, half of
// the 126 MB L2, so concurrent CTAs re-read K/V from L2 rather than HBM.
#ifndef BPT_ATTN_KV_BUDGET_MB
#define BPT_ATTN_KV_BUDGET_MB 64
#endif
// 1: the fused layer body shares the items left over after its last whole
// round between two CTA pairs (tail_tc.cuh); 0: one pair per item.
#ifndef BPT_TAIL_SHARE_ITEMS
#define BPT_TAIL_SHARE_ITEMS 1
#endif
constexpr int kEmu128 = BPT_EMU_DK128;
constexpr int kEmu64 = BPT_EMU_DK64;
// Workspace header: the device error word at offset 0; from kTailFlagOffset
// the fused layer body's hand-over counters for shared items ([2][pairs][2]
// uint32, zeroed before each launch that shares items).
constexpr size_t kTailFlagOffset = 256;
constexpr size_t kTailFlagBytes = size_t(2 * bpt::kTailMaxPairs * 2) * sizeof(uint32_t);
constexpr size_t kHeaderBytes = kTailFlagOffset + kTailFlagBytes;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Wave {
  int64_t item0, count, seqs;
};

struct Plan {
  int64_t B, N, d, h, d_ff, dk;
  int causal;
  bpt_dtype dtype;
  int64_t blk, nb, items;
  int64_t cps;   // >0: each sequence is split into cps waves
  int64_t G;     // >0: each wave holds G whole sequences
  int64_t n_waves, P;
  size_t esize;
  Opts opt;
  bool fused;          // bf16 layer on the fused schedule
  int64_t tail_pairs;  // fused: CTA pairs the scratch is sized for
  size_t off_w16, off_qkv, off_o, off_v, off_h, off_tv, off_th, total;

  Wave wave(int64_t w) const {
    Wave r;
    if (cps > 0) {
      const int64_t csize = (nb + cps - 1) / cps;
      const int64_t b = w / cps, c = w % cps;
      const int64_t i0 = c * csize, i1 = std::min(nb, i0 + csize);
      r.item0 = b * nb + i0;
      r.count = i1 - i0;
      r.seqs = 0;
    } else {
      const int64_t b0 = w * G;
      const int64_t g = std::min(G, B - b0);
      r.item0 = b0 * nb;
      r.count = g * nb;
      r.seqs = g;
    }
    return r;
  }
};

bpt_status check_shape(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff, int causal,
                       bpt_dtype dtype) {
  (void)causal;
  if (B < 0 || N < 0 || d <= 0 || h <= 0 || d_ff <= 0) return BPT_ERR_INVALID_ARG;
  if (dtype != BPT_F32 && dtype != BPT_BF16) return BPT_ERR_INVALID_ARG;
  if (d % h != 0) return BPT_ERR_INVALID_ARG;
  const int64_t dk = d / h;
  if (d % 8 != 0) return BPT_ERR_UNSUPPORTED;
  if (dtype == BPT_BF16) {
    if (dk != 64 && dk != 128) return BPT_ERR_UNSUPPORTED;
    if (d % 64 != 0 || d_ff % 64 != 0) return BPT_ERR_UNSUPPORTED;
  } else {
    if (dk > bpt::kF32AttnMaxDk || d_ff % 4 != 0) return BPT_ERR_UNSUPPORTED;
  }
  if (d > 8192 || d_ff > 65536) return BPT_ERR_UNSUPPORTED;
  // Rows and TMA coordinates are 32-bit; element offsets are 64-bit.  The
  // largest buffers are QKV [B*N, 3d] and the wave scratch (bounded by the
  // wave size), so only B*N is limited.
  if (B > 0 && N > 0 && B * N > (int64_t(1) << 30)) return BPT_ERR_UNSUPPORTED;
  return BPT_OK;
}

// The waves layout (wave scratch o / v / H) serves the waves schedule, the
// fp32 path and the backward; the fused schedule uses tail scratch instead.
Plan make_plan(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff, int causal,
               bpt_dtype dtype, const Opts& opt = Opts{}, bool forward = true) {
  Plan p{};
  p.opt = opt;
  p.B = B; p.N = N; p.d = d; p.h = h; p.d_ff = d_ff; p.dk = d / h;
  p.causal = causal ? 1 : 0;
  p.dtype = dtype;
  p.blk = dtype == BPT_BF16 ? 128 : bpt::kF32AttnRows;
  p.esize = dtype == BPT_BF16 ? 2 : 4;
  p.nb = (N + p.blk - 1) / p.blk;
  p.items = B * p.nb;
  if (p.items == 0) {
    p.n_waves = 0;
    p.P = 0;
  } else if (p.nb > opt.max_wave) {
    const int64_t mw = opt.max_wave;
    p.cps = (p.nb + mw - 1) / mw;
    p.G = 0;
    p.n_waves = B * p.cps;
    p.P = (p.nb + p.cps - 1) / p.cps;
  } else {
    p.cps = 0;
    p.G = std::max<int64_t>(1, std::min<int64_t>(B, opt.max_wave / p.nb));
    p.n_waves = (B + p.G - 1) / p.G;
    p.P = p.G * p.nb;
  }
  p.fused = forward && dtype == BPT_BF16 && opt.fused != 0 && p.items > 0;
  p.tail_pairs = p.fused ? std::min<int64_t>(bpt::kTailMaxPairs, (p.items + 1) / 2) : 0;
  size_t off = align_up(kHeaderBytes, 1024);
  p.off_w16 = off;
  if (dtype == BPT_BF16)  // fp16 copies of W_Q, W_K, W_V, W_O, W_1, W_2
    off = align_up(off + (size_t(4 * d * d) + size_t(2 * d * d_ff)) * 2, 1024);
  p.off_qkv = off;
  off = align_up(off + size_t(B * N) * size_t(3 * d) * p.esize, 1024);
  if (p.fused) {
    // per CTA pair: LN2(y) [256, d] and the FFN hidden [256, d_ff], fp16
    const size_t rows = size_t(p.tail_pairs) * 256;
    p.off_o = p.off_v = p.off_h = 0;
    p.off_tv = off;
    off = align_up(off + rows * size_t(d) * 2, 1024);
    p.off_th = off;
    off = align_up(off + rows * size_t(d_ff) * 2, 1024);
  } else {
    const size_t rows = size_t(p.P * p.blk);
    p.off_tv = p.off_th = 0;
    p.off_o = off;
    off = align_up(off + rows * size_t(d) * p.esize, 1024);
    p.off_v = off;
    off = align_up(off + rows * size_t(d) * p.esize, 1024);
    p.off_h = off;
    off = align_up(off + rows * size_t(d_ff) * p.esize, 1024);
  }
  p.total = off;
  return p;
}


// ------------------------------------------------------------ device info --
// True on failure (so that calls chain with ||).
template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
         cudaSuccess;
}

struct DeviceInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  int pair_clusters = 0;  // co-resident CTA pairs of the pair GEMM
};
std::mutex g_mu;
DeviceInfo g_dev[64];

bpt_status device_info(int* sms, int* pair_clusters = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BPT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.init) {
    int major = 0, minor = 0, n = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BPT_ERR_CUDA;
    di.ok = (major == 10 && minor == 0);
    di.sms = n;
    if (di.ok) {
      if (set_smem(bpt::attn_pair_tc_kernel<64, kEmu64>, bpt::AttnPairCfg<64, kEmu64>::SMEM) ||
          set_smem(bpt::attn_pair_tc_kernel<128, kEmu128>, bpt::AttnPairCfg<128, kEmu128>::SMEM) ||
          set_smem(bpt::attn_gate_tc_kernel<64, kEmu64>, bpt::AttnGateCfg<64>::SMEM) ||
          set_smem(bpt::attn_gate_tc_kernel<128, kEmu128>, bpt::AttnGateCfg<128>::SMEM) ||
          // b = 512 cluster pair (SHARD = false, XP = true) and sequence shard
          set_smem(bpt::attn_pair_tc_kernel<64, kEmu64, false, true>,
                   bpt::AttnPairCfg<64, kEmu64>::SMEM) ||
          set_smem(bpt::attn_pair_tc_kernel<128, kEmu128, false, true>,
                   bpt::AttnPairCfg<128, kEmu128>::SMEM) ||
          set_smem(bpt::attn_pair_tc_kernel<64, kEmu64, true>,
                   bpt::AttnPairCfg<64, kEmu64>::SMEM) ||
          set_smem(bpt::attn_pair_tc_kernel<128, kEmu128, true>,
                   bpt::AttnPairCfg<128, kEmu128>::SMEM) ||
          set_smem(bpt::gemm_f16_pair_kernel<4, bpt::kLayAkBn>, bpt::kPairSmem) ||
          set_smem(bpt::gemm_f16_pair_kernel<8, bpt::kLayAkBn>, bpt::kPairSmem) ||
          set_smem(bpt::gemm_f16_pair_kernel<4, bpt::kLayAnBn>, bpt::kPairSmem) ||
          set_smem(bpt::gemm_f16_pair_kernel<4, bpt::kLayAkBk>, bpt::kPairSmem) ||
          set_smem(bpt::gemm_f16_pair_kernel<8, bpt::kLayAkBk>, bpt::kPairSmem) ||
          set_smem(bpt::attn_bwd_dq_tc_kernel<128>, bpt::AttnBwdCfg<128>::Q_SMEM) ||
          set_smem(bpt::attn_bwd_dkv_tc_kernel<128>, bpt::AttnBwdCfg<128>::KV_SMEM) ||
          set_smem(bpt::attn_bwd_dq_tc_kernel<64>, bpt::AttnBwdCfg<64>::Q_SMEM) ||
          set_smem(bpt::attn_bwd_dkv_tc_kernel<64>, bpt::AttnBwdCfg<64>::KV_SMEM) ||
          set_smem(bpt::tail_pair_kernel, bpt::kPairSmem) ||
          set_smem(bpt::attn_b64_tc_kernel<128, kEmu128>, bpt::AttnB64Cfg<128>::SMEM) ||
          set_smem(bpt::attn_b64_tc_kernel<64, kEmu64>, bpt::AttnB64Cfg<64>::SMEM) ||
          cudaFuncSetAttribute(bpt::attn_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (3 * 64 * 128 + 64 * 65) * 4) != cudaSuccess)
        return BPT_ERR_CUDA;
      // How many CTA pairs of the pair GEMM fit on the device at once (the
      // shared memory, not the thread count, limits it to one CTA per SM).
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(unsigned(2 * (n / 2)));
      cfg.blockDim = dim3(bpt::gemm_threads<8>());
      cfg.dynamicSmemBytes = bpt::kPairSmem;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, bpt::gemm_f16_pair_kernel<8, bpt::kLayAkBn>,
                                         &cfg) !=
              cudaSuccess ||
          clusters <= 0) {
        cudaGetLastError();
        clusters = n / 2;
      }
      di.pair_clusters = clusters;
    }
    di.init = true;
  }
  if (!di.ok) return BPT_ERR_UNSUPPORTED;
  *sms = di.sms;
  if (pair_clusters) *pair_clusters = di.pair_clusters;
  return BPT_OK;
}

// ------------------------------------------------------------ tensor maps --
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bpt_status get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return BPT_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return BPT_ERR_CUDA;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return BPT_OK;
}

// fp16 tiles with the 128-byte swizzle; dims/strides innermost first.
bool encode_f16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                const uint64_t* strides_bytes, const uint32_t* box) {
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5] = {1, 1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(base),
                              gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// GEMM operand, K-contiguous: [rows, K] with row stride ld (elements), viewed
// as [K/64][rows][64]; a box is 128 rows x two 64-column chunks (32 KB,
// chunk-major in shared memory).  The A operand of the forward, and the B
// operand [N, K] of the data-gradient GEMMs.
bool map_a(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int64_t ld = 0,
           int chunks = 2) {
  const uint64_t dims[3] = {64, uint64_t(rows), uint64_t(K / 64)};
  const uint64_t st[2] = {uint64_t(ld > 0 ? ld : K) * 2, 128};
  const uint32_t box[3] = {64, 128, uint32_t(chunks)};
  return encode_f16(m, base, 3, dims, st, box);
}
// GEMM operand, row-contiguous along the output axis: [K, cols] with row
// stride ld, viewed as [cols/64][K][64]; a box is 128 K rows x `chunks`
// 64-column chunks.  The B operand of the forward (weights), and the A
// operand [K, M] of the weight-gradient GEMMs.
bool map_b(CUtensorMap* m, const void* base, int64_t K, int64_t cols, int chunks,
           int64_t ld = 0, int box_rows = 128) {
  const uint64_t dims[3] = {64, uint64_t(K), uint64_t(cols / 64)};
  const uint64_t st[2] = {uint64_t(ld > 0 ? ld : cols) * 2, 128};
  const uint32_t box[3] = {64, uint32_t(box_rows), uint32_t(chunks)};
  return encode_f16(m, base, 3, dims, st, box);
}
// QKV [B][N][3d] viewed as [B][3d/64][N][64]: a box is 128 tokens x the
// d_k/64 chunks of one head's Q, K or V (32 KB at d_k = 128), chunk-major in
// shared memory.
bool map_qkv(CUtensorMap* m, const void* base, int64_t B, int64_t N, int64_t d, int64_t dk) {
  const uint64_t dims[4] = {64, uint64_t(N), uint64_t(3 * d / 64), uint64_t(B)};
  const uint64_t st[3] = {uint64_t(3 * d) * 2, 128, uint64_t(N) * uint64_t(3 * d) * 2};
  const uint32_t box[4] = {64, 128, uint32_t(dk / 64), 1};
  return encode_f16(m, base, 4, dims, st, box);
}

// QKV viewed as map_qkv, 64-token boxes of one 64-column chunk (8 KB): the
// half tiles a b = 512 attention cluster loads, one per CTA.
bool map_qkv_half(CUtensorMap* m, const void* base, int64_t B, int64_t N, int64_t d) {
  const uint64_t dims[4] = {64, uint64_t(N), uint64_t(3 * d / 64), uint64_t(B)};
  const uint64_t st[3] = {uint64_t(3 * d) * 2, 128, uint64_t(N) * uint64_t(3 * d) * 2};
  const uint32_t box[4] = {64, 64, 1, 1};
  return encode_f16(m, base, 4, dims, st, box);
}

// QKV viewed as map_qkv, 64-token boxes of one head's d_k / 64 chunks: the
// Q tile of a b = 64 attention CTA.
bool map_q64(CUtensorMap* m, const void* base, int64_t B, int64_t N, int64_t d, int64_t dk) {
  const uint64_t dims[4] = {64, uint64_t(N), uint64_t(3 * d / 64), uint64_t(B)};
  const uint64_t st[3] = {uint64_t(3 * d) * 2, 128, uint64_t(N) * uint64_t(3 * d) * 2};
  const uint32_t box[4] = {64, 64, uint32_t(dk / 64), 1};
  return encode_f16(m, base, 4, dims, st, box);
}

// All-gathered K | V of a sequence shard, [G][B][n_loc][2d], viewed as
// [G][B][2d/64][n_loc][64]: a box is 128 tokens x the d_k/64 chunks of one
// head's K or V of one rank's batch element.
bool map_kv_shards(CUtensorMap* m, const void* base, int64_t G, int64_t B, int64_t n_loc,
                   int64_t d, int64_t dk) {
  const uint64_t row = uint64_t(2 * d) * 2;
  const uint64_t dims[5] = {64, uint64_t(n_loc), uint64_t(2 * d / 64), uint64_t(B), uint64_t(G)};
  const uint64_t st[4] = {row, 128, uint64_t(n_loc) * row, uint64_t(B * n_loc) * row};
  const uint32_t box[5] = {64, 128, uint32_t(dk / 64), 1, 1};
  return encode_f16(m, base, 5, dims, st, box);
}

// -------------------------------------------------------------- profiling --
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct LaunchScope {
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  LaunchScope(int k, cudaStream_t st) : kind(k), s(st) {
    if (g_prof_on) {
      a = pool_event();
      cudaEventRecord(a, s);
    }
  }
  ~LaunchScope() {
    if (g_prof_on && a) {
      cudaEvent_t b = pool_event();
      cudaEventRecord(b, s);
      g_prof.push_back({kind, a, b});
    }
  }
};

// ----------------------------------------------------------------- launches --
template <typename TIn, typename TOut, typename TP>
cudaError_t launch_ln(const TIn* in, const TP* ln, TOut* out, int64_t rows, int64_t d, RowMap map,
                      uint32_t* err, cudaStream_t s) {
  const int nv = int((d + 255) / 256);
  const dim3 grid(unsigned((rows + bpt::kLnWarps - 1) / bpt::kLnWarps));
  const dim3 block(bpt::kLnWarps * 32);
#define BPT_LN_CASE(NV)                                                                    \
  if (nv <= NV) {                                                                          \
    bpt::ln_rows_kernel<NV, TIn, TOut, TP><<<grid, block, 0, s>>>(in, ln, out, rows, int(d), \
                                                                  map, err);               \
    return cudaGetLastError();                                                             \
  }
  BPT_LN_CASE(1)
  BPT_LN_CASE(2)
  BPT_LN_CASE(3)
  BPT_LN_CASE(4)
  BPT_LN_CASE(6)
  BPT_LN_CASE(8)
  BPT_LN_CASE(12)
  BPT_LN_CASE(16)
  BPT_LN_CASE(32)
#undef BPT_LN_CASE
  return cudaErrorInvalidValue;
}

// layout: bpt::kLayAkBn (forward), kLayAnBn (X^T dY), kLayAkBk (dY W^T).
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& b2, const bpt::GemmParams& gp, int sms,
                        cudaStream_t s, int layout = bpt::kLayAkBn) {
  int dummy = 0, pairs_max = 0;
  if (device_info(&dummy, &pairs_max) != BPT_OK) return cudaErrorInvalidDevice;
  const int64_t tiles = int64_t((gp.M + bpt::kPairBM - 1) / bpt::kPairBM) *
                        int64_t((gp.N + bpt::kGemmBN - 1) / bpt::kGemmBN);
  const unsigned pairs = unsigned(std::max<int64_t>(1, std::min<int64_t>(tiles, pairs_max)));
  // Eight epilogue warps for the per-element-heavy epilogues, four otherwise.
  const bool heavy = gp.epi == bpt::kEpiGeluBias || gp.epi == bpt::kEpiResidX ||
                     gp.epi == bpt::kEpiGeluBiasKeep || gp.epi == bpt::kEpiGeluGrad;
  const unsigned grid = 2 * pairs;
  if (layout == bpt::kLayAnBn)
    bpt::gemm_f16_pair_kernel<4, bpt::kLayAnBn>
        <<<grid, bpt::gemm_threads<4>(), bpt::kPairSmem, s>>>(a, b0, b1, b2, gp);
  else if (layout == bpt::kLayAkBk && heavy)
    bpt::gemm_f16_pair_kernel<8, bpt::kLayAkBk>
        <<<grid, bpt::gemm_threads<8>(), bpt::kPairSmem, s>>>(a, b0, b1, b2, gp);
  else if (layout == bpt::kLayAkBk)
    bpt::gemm_f16_pair_kernel<4, bpt::kLayAkBk>
        <<<grid, bpt::gemm_threads<4>(), bpt::kPairSmem, s>>>(a, b0, b1, b2, gp);
  else if (heavy)
    bpt::gemm_f16_pair_kernel<8, bpt::kLayAkBn>
        <<<grid, bpt::gemm_threads<8>(), bpt::kPairSmem, s>>>(a, b0, b1, b2, gp);
  else
    bpt::gemm_f16_pair_kernel<4, bpt::kLayAkBn>
        <<<grid, bpt::gemm_threads<4>(), bpt::kPairSmem, s>>>(a, b0, b1, b2, gp);
  return cudaGetLastError();
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Block gating of the attention (bpt_layer_forward_bsfa).
struct AttnGate {
  const float* t;   // [h][nb] thresholds
  float* bmax;      // nullable [B][h][nb][nb]
  uint8_t* kept;    // nullable [B][h][nb][nb]
};

// Sequence shard of the attention: keys and values of the whole sequence in
// the all-gathered buffer (5-D tensor map), zig-zag chunk ownership.
struct AttnShard {
  const CUtensorMap* mKV;  // [G][B][N / G][2d] viewed as [G][B][2d/64][N/G][64]
  int cb, c0, c1, G;       // blocks per chunk, this rank's chunks, ranks
  int64_t N_kv;            // tokens of the whole sequence
};

// One wave of the tensor-core attention: o (fp16 block rows) and, if stats is
// non-null, the per-row (m, l); gated when gate is non-null.
// o_tok: o is the Q columns of the QKV buffer, token rows (fused schedule);
// otherwise wave scratch rows [count * 128, d].  shard: o_tok over the
// shard's own Q buffer [rows, d] (mQKV maps it), keys from shard->mKV.
cudaError_t launch_attn(const Plan& P, const Wave& wv_, const CUtensorMap& mQKV, __half* so,
                        float* stats, uint32_t* err, int fault, cudaStream_t s,
                        const AttnGate* gate = nullptr, bool o_tok = false,
                        const AttnShard* shard = nullptr, const CUtensorMap* xp_map = nullptr,
                        int64_t o_ld = 0) {
  bpt::AttnPairParams ap{};
  ap.N = int(P.N); ap.nb = int(P.nb); ap.h = int(P.h); ap.d = int(P.d);
  ap.causal = P.causal; ap.item0 = int(wv_.item0); ap.count = int(wv_.count);
  ap.seqs = int(wv_.seqs); ap.o = so; ap.err = err;
  ap.o_tok = o_tok ? 1 : 0;
  ap.o_ld = o_ld != 0 ? o_ld : (o_tok ? 3 * P.d : P.d);
  ap.scale_log2 = float(1.4426950408889634 / std::sqrt(double(P.dk)));
  ap.stats = reinterpret_cast<float2*>(stats);
  if (shard) {
    ap.kv_cb = shard->cb;
    ap.q_c0 = shard->c0;
    ap.q_c1 = shard->c1;
    ap.kv_G = shard->G;
    ap.N_kv = int(shard->N_kv);
  }
  const int64_t kv_head =
      (wv_.seqs > 0 ? wv_.seqs : 1) * (shard ? shard->N_kv : P.N) * P.dk * 2 * 2;
  ap.hg = 1;
  for (int g = int(P.h); g > 1; --g)
    if (P.h % g == 0 && g * kv_head <= (int64_t(BPT_ATTN_KV_BUDGET_MB) << 20)) {
      ap.hg = g;
      break;
    }
  ap.fault = fault;
  ap.qpc = P.opt.qpc;
  if (P.opt.b64) {
    // b = 64: one CTA per 64-row query block and head, two CTAs per SM
    if (gate != nullptr || shard != nullptr || xp_map == nullptr) return cudaErrorInvalidValue;
    const int64_t units64 = 2 * (wv_.seqs == 0 ? wv_.count : wv_.seqs * P.nb);
    const unsigned grid64 = unsigned(units64 * P.h);
    if (P.dk == 128)
      bpt::attn_b64_tc_kernel<128, kEmu128>
          <<<grid64, 256, bpt::AttnB64Cfg<128>::SMEM, s>>>(*xp_map, mQKV, ap);
    else
      bpt::attn_b64_tc_kernel<64, kEmu64>
          <<<grid64, 256, bpt::AttnB64Cfg<64>::SMEM, s>>>(*xp_map, mQKV, ap);
    return cudaGetLastError();
  }
  const int64_t units = wv_.seqs == 0 ? (wv_.count + ap.qpc - 1) / ap.qpc
                                      : wv_.seqs * ((P.nb + ap.qpc - 1) / ap.qpc);
  const unsigned grid = unsigned(units * P.h);
  const CUtensorMap& mKV = shard ? *shard->mKV : mQKV;
  if (ap.qpc == 4) {
    // b = 512: clusters of two CTAs, each with two query blocks, sharing K/V
    if (gate != nullptr || shard != nullptr || xp_map == nullptr) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * grid);
    cfg.blockDim = dim3(384);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (P.dk == 128) {
      cfg.dynamicSmemBytes = bpt::AttnPairCfg<128, kEmu128>::SMEM;
      return cudaLaunchKernelEx(&cfg, bpt::attn_pair_tc_kernel<128, kEmu128, false, true>,
                                mQKV, *xp_map, ap);
    }
    cfg.dynamicSmemBytes = bpt::AttnPairCfg<64, kEmu64>::SMEM;
    return cudaLaunchKernelEx(&cfg, bpt::attn_pair_tc_kernel<64, kEmu64, false, true>,
                              mQKV, *xp_map, ap);
  }
  if (gate != nullptr) {
    ap.gate_t = gate->t;
    ap.gate_bmax = gate->bmax;
    ap.gate_kept = gate->kept;
    if (P.dk == 128)
      bpt::attn_gate_tc_kernel<128, kEmu128>
          <<<grid, 384, bpt::AttnGateCfg<128>::SMEM, s>>>(mQKV, ap);
    else
      bpt::attn_gate_tc_kernel<64, kEmu64><<<grid, 384, bpt::AttnGateCfg<64>::SMEM, s>>>(mQKV, ap);
  } else if (shard != nullptr) {
    if (P.dk == 128)
      bpt::attn_pair_tc_kernel<128, kEmu128, true>
          <<<grid, 384, bpt::AttnPairCfg<128, kEmu128>::SMEM, s>>>(mQKV, mKV, ap);
    else
      bpt::attn_pair_tc_kernel<64, kEmu64, true>
          <<<grid, 384, bpt::AttnPairCfg<64, kEmu64>::SMEM, s>>>(mQKV, mKV, ap);
  } else if (P.dk == 128) {
    bpt::attn_pair_tc_kernel<128, kEmu128>
        <<<grid, 384, bpt::AttnPairCfg<128, kEmu128>::SMEM, s>>>(mQKV, mKV, ap);
  } else {
    bpt::attn_pair_tc_kernel<64, kEmu64>
        <<<grid, 384, bpt::AttnPairCfg<64, kEmu64>::SMEM, s>>>(mQKV, mKV, ap);
  }
  return cudaGetLastError();
}

// One rank's part of a sequence-sharded forward (bpt_layer_shard_*): the
// plan is that of the rank's own n_loc = N / G rows; phase 1 writes its K | V
// to kv_loc, phase 2 attends against every rank's K | V in kv_all.
struct ShardSpec {
  int phase;          // 1: projection, 2: attention + layer body
  int G, rank;
  int64_t N;          // tokens of the whole sequence
  __half* kv_loc;     // phase 1: [B, n_loc, 2d]
  const void* kv_all; // phase 2: [G, B, n_loc, 2d]
};

bpt_status forward_bf16(const Plan& P, const void* x, const void* ln1, const void* W_Q,
                        const void* W_K, const void* W_V, const void* W_O, const void* ln2,
                        const void* W_1, const void* b_1, const void* W_2, const void* b_2,
                        float* out, float* stats, uint8_t* ws, cudaStream_t s, int sms,
                        const AttnGate* gate, const ShardSpec* shard = nullptr,
                        __half* o_keep = nullptr) {
  using bf = __nv_bfloat16;
  using hf = __half;
  const int64_t M = P.B * P.N, d = P.d, d_ff = P.d_ff;
  const int fault = P.opt.fault;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  // Tensor-core operands are fp16: the bf16 weights are copied to fp16 once
  // per call (exact in the fp16 normal range), activations are stored fp16.
  hf* w16 = reinterpret_cast<hf*>(ws + P.off_w16);
  hf* wq = w16;
  hf* wk = wq + d * d;
  hf* wv = wk + d * d;
  hf* wo = wv + d * d;
  hf* w1 = wo + d * d;
  hf* w2 = w1 + d * d_ff;
  hf* xn = reinterpret_cast<hf*>(out);  // LN1(x) lives in `out` until the waves start
  hf* qkv = reinterpret_cast<hf*>(ws + P.off_qkv);
  hf* so = reinterpret_cast<hf*>(ws + P.off_o);
  hf* sv = reinterpret_cast<hf*>(ws + P.off_v);
  hf* sh = reinterpret_cast<hf*>(ws + P.off_h);
  const int64_t R = P.P * P.blk;  // scratch rows

  CUtensorMap mXn, mWq, mWk, mWv, mQKV, mO, mWo, mV, mW1, mH, mW2, mH1, mW2e;
  // A CTA's 128 B columns stay inside one of W_Q | W_K | W_V when d is a
  // multiple of 128 (one two-chunk box); otherwise it loads one chunk per box.
  const int qkv_chunks = (d % 128 == 0) ? 2 : 1;
  bool ok = map_a(&mXn, xn, M, d) && map_b(&mWq, wq, d, d, qkv_chunks) &&
            map_b(&mWk, wk, d, d, qkv_chunks) && map_b(&mWv, wv, d, d, qkv_chunks) &&
            map_qkv(&mQKV, qkv, P.B, P.N, d, P.dk) && map_b(&mWo, wo, d, d, 2) &&
            map_b(&mW1, w1, d, d_ff, 2) && map_b(&mW2, w2, d_ff, d, 2);
  if (P.fused) {
    // tail A operands: o = the Q columns of QKV (token rows, row stride 3d),
    // and the per-pair scratch rows of LN2(y) and the hidden
    const int64_t trows = P.tail_pairs * 256;
    // (o_keep: the attention writes o there instead, [B*N, d])
    ok = ok && (o_keep != nullptr ? map_a(&mO, o_keep, M, d) : map_a(&mO, qkv, M, d, 3 * d)) &&
         map_a(&mV, ws + P.off_tv, trows, d) && map_a(&mH, ws + P.off_th, trows, d_ff) &&
         // 512-column W_2 tiles: H in 64-deep single-chunk boxes, W_2 as
         // 64 K rows x four 64-column chunks
         map_a(&mH1, ws + P.off_th, trows, d_ff, 0, 1) && map_b(&mW2e, w2, d_ff, d, 4, 0, 64);
  } else {
    ok = ok && map_a(&mO, so, R, d) && map_a(&mV, sv, R, d) && map_a(&mH, sh, R, d_ff);
  }
  CUtensorMap mKV, mQKVh;
  if (shard != nullptr && shard->phase == 2)
    ok = ok && map_kv_shards(&mKV, shard->kv_all, shard->G, P.B, P.N, d, P.dk);
  if (P.opt.qpc == 4) ok = ok && map_qkv_half(&mQKVh, qkv, P.B, P.N, d);
  if (P.opt.b64) ok = ok && map_q64(&mQKVh, qkv, P.B, P.N, d, P.dk);
  if (!ok) return BPT_ERR_CUDA;

  RowMap ident{0, 1, 1, 1, 1};
  if (shard == nullptr || shard->phase == 1) {
  {
    bpt::CvtSegments cs{};
    const void* src[6] = {W_Q, W_K, W_V, W_O, W_1, W_2};
    hf* dst[6] = {wq, wk, wv, wo, w1, w2};
    const int64_t n[6] = {d * d, d * d, d * d, d * d, d * d_ff, d_ff * d};
    long long acc = 0;
    for (int k = 0; k < 6; ++k) {
      cs.src[k] = static_cast<const bf*>(src[k]);
      cs.dst[k] = dst[k];
      acc += n[k] / 8;
      cs.n8_end[k] = acc;
    }
    cs.count = 6;
    const unsigned grid = unsigned(std::min<long long>((acc + 255) / 256, int64_t(sms) * 8));
    LaunchScope ls(BPT_KIND_CVT, s);
    bpt::cvt_bf16_to_f16_kernel<<<grid, 256, 0, s>>>(cs, err);
    if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
  }
  {
    LaunchScope ls(BPT_KIND_LN1, s);
    if (launch_ln<bf, hf, bf>(static_cast<const bf*>(x), static_cast<const bf*>(ln1), xn, M, d,
                              ident, err, s) != cudaSuccess)
      return BPT_ERR_CUDA;
  }
  {
    bpt::GemmParams g{};
    g.M = int(M); g.N = int(3 * d); g.K = int(d);
    g.n_sub = int(d); g.n_maps = 3; g.b_chunks = qkv_chunks;
    g.epi = bpt::kEpiStoreF16;
    g.out_h = qkv; g.ld_out = 3 * d;
    if (shard != nullptr) {  // K | V of the shard's rows go to kv_loc
      g.split_col = int(d);
      g.out_h2 = shard->kv_loc;
      g.ld_out2 = 2 * d;
    }
    g.map = ident;
    g.err = err;
    g.fault = fault == 1 ? 1 : 0;
    LaunchScope ls(BPT_KIND_QKV, s);
    if (launch_gemm(mXn, mWq, mWk, mWv, g, sms, s) != cudaSuccess) return BPT_ERR_CUDA;
  }
  }  // projection
  if (shard != nullptr && shard->phase == 1) return BPT_OK;
  if (P.fused) {
    // attention over every query block, o over each block's Q rows
    const Wave all{0, P.items, P.B};
    AttnShard as{};
    if (shard != nullptr) {
      as.mKV = &mKV;
      as.G = shard->G;
      as.cb = int(P.N / 2 / 128);
      as.c0 = shard->rank;
      as.c1 = 2 * shard->G - 1 - shard->rank;
      as.N_kv = shard->N;
    }
    {
      LaunchScope ls(BPT_KIND_ATTN, s);
      if (launch_attn(P, all, mQKV, o_keep != nullptr ? o_keep : qkv, stats, err,
                      fault == 2 ? 2 : 0, s, gate, true, shard != nullptr ? &as : nullptr, &mQKVh,
                      o_keep != nullptr ? d : 0) != cudaSuccess)
        return BPT_ERR_CUDA;
    }
    int dummy = 0, pairs_max = 0;
    if (device_info(&dummy, &pairs_max) != BPT_OK) return BPT_ERR_CUDA;
    bpt::TailParams tp{};
    tp.blocks = int(P.items);
    tp.items = int((P.items + 1) / 2);
    tp.nb = int(P.nb);
    tp.N = int(P.N);
    tp.d = int(d);
    tp.d_ff = int(d_ff);
    tp.out = out;
    tp.x = static_cast<const bf*>(x);
    tp.ln2 = static_cast<const bf*>(ln2);
    tp.b1 = static_cast<const bf*>(b_1);
    tp.b2 = static_cast<const bf*>(b_2);
    tp.v_scr = reinterpret_cast<hf*>(ws + P.off_tv);
    tp.h_scr = reinterpret_cast<hf*>(ws + P.off_th);
    tp.err = err;
    tp.fault = fault == 3 ? 3 : 0;
    const int64_t pairs = std::max<int64_t>(1, std::min<int64_t>(P.tail_pairs, pairs_max));
    // Share the items left over after the whole rounds between two pairs
    // each when at most half of the pairs would otherwise work in the last
    // round and every half is a whole number of tiles (y tiles and H chunks
    // of 256 columns, Z tiles of 512).
    tp.split = (BPT_TAIL_SHARE_ITEMS && bpt::tail_shares(tp.items, int(pairs), int(d), int(d_ff)))
                   ? 1 : 0;
    tp.flags = reinterpret_cast<uint32_t*>(ws + kTailFlagOffset);
    if (tp.split) {
      // Under stream capture (a CUDA graph being recorded) the body runs
      // unshared with a plain launch, which graphs always accept.
      cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return BPT_ERR_CUDA;
      if (cap != cudaStreamCaptureStatusNone) tp.split = 0;
    }
    LaunchScope ls(BPT_KIND_TAIL, s);
    if (tp.split) {
      // A pair waits for its partner's hand-overs, so all pairs must be
      // resident at once: a cooperative launch guarantees it (or fails, and
      // the layer body runs without sharing).
      if (cudaMemsetAsync(tp.flags, 0, kTailFlagBytes, s) != cudaSuccess) return BPT_ERR_CUDA;
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(unsigned(2 * pairs));
      cfg.blockDim = dim3(bpt::kTailThreads);
      cfg.dynamicSmemBytes = bpt::kPairSmem;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeCooperative;
      attr[0].val.cooperative = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, bpt::tail_pair_kernel, mO, mWo, mV, mW1, mH, mW2, mH1, mW2e,
                             tp) == cudaSuccess)
        return BPT_OK;
      (void)cudaGetLastError();
      tp.split = 0;
    }
    bpt::tail_pair_kernel<<<unsigned(2 * pairs), bpt::kTailThreads, bpt::kPairSmem, s>>>(
        mO, mWo, mV, mW1, mH, mW2, mH1, mW2e, tp);
    if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
    return BPT_OK;
  }
  for (int64_t w = 0; w < P.n_waves; ++w) {
    const Wave wv_ = P.wave(w);
    const int64_t rows = wv_.count * P.blk;
    RowMap map{int(wv_.item0), int(P.nb), int(P.N), int(P.blk), 0};
    {
      LaunchScope ls(BPT_KIND_ATTN, s);
      if (launch_attn(P, wv_, mQKV, so, stats, err, (fault == 2 && w == 0) ? 2 : 0, s, gate,
                      false, nullptr, &mQKVh) !=
          cudaSuccess)
        return BPT_ERR_CUDA;
      if (o_keep != nullptr) {  // the wave's o rows to their token rows
        bpt::rows_copy_f16_kernel<<<unsigned(std::min<int64_t>((rows * d / 8 + 255) / 256,
                                                               int64_t(sms) * 16)),
                                    256, 0, s>>>(so, d, o_keep, d, rows, int(d), map, 1);
        if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
      }
    }
    {
      bpt::GemmParams g{};
      g.M = int(rows); g.N = int(d); g.K = int(d);
      g.n_sub = int(d); g.n_maps = 1; g.b_chunks = 2;
      g.epi = bpt::kEpiResidX;
      g.out_f32 = out; g.ld_f32 = d;
      g.resid = static_cast<const bf*>(x); g.ld_resid = d;
      g.map = map; g.err = err;
      LaunchScope ls(BPT_KIND_WO, s);
      if (launch_gemm(mO, mWo, mWo, mWo, g, sms, s) != cudaSuccess) return BPT_ERR_CUDA;
    }
    {
      LaunchScope ls(BPT_KIND_LN2, s);
      if (launch_ln<float, hf, bf>(out, static_cast<const bf*>(ln2), sv, rows, d, map, err, s) !=
          cudaSuccess)
        return BPT_ERR_CUDA;
    }
    {
      bpt::GemmParams g{};
      g.M = int(rows); g.N = int(d_ff); g.K = int(d);
      g.n_sub = int(d_ff); g.n_maps = 1; g.b_chunks = 2;
      g.epi = bpt::kEpiGeluBias;
      g.out_h = sh; g.ld_out = d_ff;
      g.bias = static_cast<const bf*>(b_1);
      g.map = ident; g.err = err;
      LaunchScope ls(BPT_KIND_W1, s);
      if (launch_gemm(mV, mW1, mW1, mW1, g, sms, s) != cudaSuccess) return BPT_ERR_CUDA;
    }
    {
      bpt::GemmParams g{};
      g.M = int(rows); g.N = int(d); g.K = int(d_ff);
      g.n_sub = int(d); g.n_maps = 1; g.b_chunks = 2;
      g.epi = bpt::kEpiBiasAccum;
      g.out_f32 = out; g.ld_f32 = d;
      g.bias = static_cast<const bf*>(b_2);
      g.map = map; g.err = err;
      LaunchScope ls(BPT_KIND_W2, s);
      if (launch_gemm(mH, mW2, mW2, mW2, g, sms, s) != cudaSuccess) return BPT_ERR_CUDA;
    }
  }
  return BPT_OK;
}

bpt_status forward_f32(const Plan& P, const float* x, const float* ln1, const float* W_Q,
                       const float* W_K, const float* W_V, const float* W_O, const float* ln2,
                       const float* W_1, const float* b_1, const float* W_2, const float* b_2,
                       float* out, float* stats, uint8_t* ws, cudaStream_t s) {
  const int64_t M = P.B * P.N, d = P.d, d_ff = P.d_ff;
  float* qkv = reinterpret_cast<float*>(ws + P.off_qkv);
  float* so = reinterpret_cast<float*>(ws + P.off_o);
  float* sv = reinterpret_cast<float*>(ws + P.off_v);
  float* sh = reinterpret_cast<float*>(ws + P.off_h);
  float* xn = out;  // LN1(x) lives in `out` until the waves start
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  RowMap ident{0, 1, 1, 1, 1};
  auto gemm = [&](int kind, const float* A, int64_t Mr, int64_t Nc, int64_t K, const float* B0,
                  const float* B1, const float* B2, int64_t n_sub, int epi, float* o,
                  int64_t ld_out, const float* resid, const float* bias, RowMap map) -> bool {
    bpt::GemmF32Params g{};
    g.M = int(Mr); g.N = int(Nc); g.K = int(K); g.n_sub = int(n_sub);
    g.A = A; g.B[0] = B0; g.B[1] = B1; g.B[2] = B2;
    g.epi = epi; g.out = o; g.ld_out = ld_out; g.resid = resid; g.ld_resid = d;
    g.bias = bias; g.map = map;
    const dim3 grid(unsigned((Nc + bpt::kF32Tile - 1) / bpt::kF32Tile),
                    unsigned((Mr + bpt::kF32Tile - 1) / bpt::kF32Tile));
    LaunchScope ls(kind, s);
    bpt::gemm_f32_kernel<<<grid, 256, 0, s>>>(g);
    return cudaGetLastError() == cudaSuccess;
  };
  {
    LaunchScope ls(BPT_KIND_LN1, s);
    if (launch_ln<float, float, float>(x, ln1, xn, M, d, ident, err, s) != cudaSuccess)
      return BPT_ERR_CUDA;
  }
  if (!gemm(BPT_KIND_QKV, xn, M, 3 * d, d, W_Q, W_K, W_V, d, bpt::kEpiStoreF16, qkv, 3 * d,
            nullptr, nullptr, ident))
    return BPT_ERR_CUDA;
  for (int64_t w = 0; w < P.n_waves; ++w) {
    const Wave wv = P.wave(w);
    const int64_t rows = wv.count * P.blk;
    RowMap map{int(wv.item0), int(P.nb), int(P.N), int(P.blk), 0};
    {
      bpt::AttnF32Params ap{};
      ap.qkv = qkv; ap.o = so; ap.N = int(P.N); ap.nb = int(P.nb); ap.h = int(P.h);
      ap.d = int(d); ap.causal = P.causal; ap.item0 = int(wv.item0); ap.blk = int(P.blk);
      ap.scale = float(1.0 / std::sqrt(double(P.dk)));
      ap.stats = stats;
      const size_t smem = size_t(3 * 64 * P.dk + 64 * 65) * 4;
      LaunchScope ls(BPT_KIND_ATTN, s);
      bpt::attn_f32_kernel<<<unsigned(wv.count * P.h), 256, smem, s>>>(ap);
      if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
    }
    if (!gemm(BPT_KIND_WO, so, rows, d, d, W_O, W_O, W_O, d, bpt::kEpiResidX, out, d, x, nullptr,
              map))
      return BPT_ERR_CUDA;
    {
      LaunchScope ls(BPT_KIND_LN2, s);
      if (launch_ln<float, float, float>(out, ln2, sv, rows, d, map, err, s) != cudaSuccess)
        return BPT_ERR_CUDA;
    }
    if (!gemm(BPT_KIND_W1, sv, rows, d_ff, d, W_1, W_1, W_1, d_ff, bpt::kEpiGeluBias, sh, d_ff,
              nullptr, b_1, ident))
      return BPT_ERR_CUDA;
    if (!gemm(BPT_KIND_W2, sh, rows, d, d_ff, W_2, W_2, W_2, d, bpt::kEpiBiasAccum, out, d,
              nullptr, b_2, map))
      return BPT_ERR_CUDA;
  }
  return BPT_OK;
}

}  // namespace

// ----------------------------------------------------------- backward --
// Workspace of bpt_layer_backward: the forward's layout (header, fp16
// weights, QKV, wave scratch o / LN2(y) / H), then the backward's buffers.
constexpr int kColChunks = 256;  // row chunks of the deterministic column sums

struct BwdLayout {
  size_t off_hpre, off_dz16, off_dvn, off_dy16, off_do16, off_D, off_rowstat, off_y, off_u16,
      off_dq, off_dk, off_dv, off_dqkv16, off_du, off_part, total;
  int64_t part_cols;
};

BwdLayout make_bwd_layout(const Plan& P) {
  BwdLayout L{};
  const size_t R = size_t(P.P * P.blk), M = size_t(P.B * P.N), d = size_t(P.d),
               dff = size_t(P.d_ff), h = size_t(P.h);
  size_t off = align_up(P.total, 1024);
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L.off_hpre = take(R * dff * 2);
  L.off_dz16 = take(R * d * 2);
  L.off_dvn = take(R * d * 4);
  L.off_dy16 = take(R * d * 2);
  L.off_do16 = take(R * d * 2);
  L.off_D = take(R * h * 8);
  L.off_rowstat = take(std::max(R, M) * 8);
  L.off_y = take(M * d * 4);
  L.off_u16 = take(M * d * 2);
  L.off_dq = take(M * d * 4);
  L.off_dk = take(M * d * 4);
  L.off_dv = take(M * d * 4);
  L.off_dqkv16 = take(M * 3 * d * 2);
  L.off_du = take(M * d * 4);
  L.part_cols = int64_t(std::max(d, dff));
  L.off_part = take(2 * size_t(kColChunks) * size_t(L.part_cols) * 4);
  L.total = off;
  return L;
}

// out[c] (+)= column sums of A (and of A * xh if X) over `rows` rows.
template <typename TA, typename TX>
cudaError_t launch_colsum(const TA* A, int a_global, const TX* X, const float2* rowstat,
                          int64_t rows, int64_t d, RowMap map, float* part_a, float* part_b,
                          float* out_a, float* out_b, cudaStream_t s) {
  // a wave map: one chunk per query block (at most BPT_WAVE_BLOCKS of them);
  // the identity map: kColChunks runs of rows
  const int rpc = map.identity ? int((rows + kColChunks - 1) / kColChunks) : map.blk;
  const int chunks = int((rows + rpc - 1) / rpc);
  if (chunks > kColChunks || d % 4 != 0) return cudaErrorInvalidValue;
  bpt::colsum_partial_kernel<TA, TX><<<dim3(unsigned((d / 4 + 255) / 256), unsigned(chunks)), 256,
                                        0, s>>>(A, a_global, X, rowstat, part_a, part_b, rows,
                                                int(d), rpc, map);
  bpt::colsum_reduce_kernel<<<unsigned((d + 255) / 256), 256, 0, s>>>(part_a, chunks, int(d),
                                                                     out_a);
  if (X) bpt::colsum_reduce_kernel<<<unsigned((d + 255) / 256), 256, 0, s>>>(part_b, chunks,
                                                                            int(d), out_b);
  return cudaGetLastError();
}

// Workspace of the fp32 backward (after the forward plan's regions; fp32
// throughout): FFN pre-activation and its gradient, wave copies of dZ, dY
// and dO, dVn, the attention row terms, LN row statistics, y, LN1(x), dQ,
// dK, dV, dU and the column-sum partials.
struct BwdLayoutF32 {
  size_t off_hpre, off_dh, off_dzw, off_dvn, off_dyw, off_dow, off_rt, off_rowstat, off_y, off_u,
      off_dq, off_dk, off_dv, off_du, off_part, total;
  int64_t part_cols;
};

BwdLayoutF32 make_bwd_layout_f32(const Plan& P) {
  BwdLayoutF32 L{};
  const size_t R = size_t(P.P * P.blk), M = size_t(P.B * P.N), d = size_t(P.d),
               dff = size_t(P.d_ff), h = size_t(P.h);
  size_t off = align_up(P.total, 1024);
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L.off_hpre = take(R * dff * 4);
  L.off_dh = take(R * dff * 4);
  L.off_dzw = take(R * d * 4);
  L.off_dvn = take(R * d * 4);
  L.off_dyw = take(R * d * 4);
  L.off_dow = take(R * d * 4);
  L.off_rt = take(R * h * 8);
  L.off_rowstat = take(std::max(R, M) * 8);
  L.off_y = take(M * d * 4);
  L.off_u = take(M * d * 4);
  L.off_dq = take(M * d * 4);
  L.off_dk = take(M * d * 4);
  L.off_dv = take(M * d * 4);
  L.off_du = take(M * d * 4);
  L.part_cols = int64_t(std::max(d, dff));
  L.off_part = take(2 * size_t(kColChunks) * size_t(L.part_cols) * 4);
  L.total = off;
  return L;
}

// fp32 backward on the CUDA cores: the bf16 schedule (waves recomputed from
// x and (m, l), gradients accumulated wave by wave, no atomics), fp32 SIMT
// kernels (backward_f32.cuh) for the products.
bpt_status backward_f32(const Plan& P, const BwdLayoutF32& L, const float* x, const float* ln1,
                        const float* W_Q, const float* W_K, const float* W_V, const float* W_O,
                        const float* ln2, const float* W_1, const float* b_1, const float* W_2,
                        const float* stats, const float* dZ, float* dx, float* d_ln1,
                        float* dW_Q, float* dW_K, float* dW_V, float* dW_O, float* d_ln2,
                        float* dW_1, float* db_1, float* dW_2, float* db_2, uint8_t* ws,
                        cudaStream_t s) {
  const int64_t M = P.B * P.N, d = P.d, d_ff = P.d_ff, h = P.h;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  float* qkv = reinterpret_cast<float*>(ws + P.off_qkv);
  float* so = reinterpret_cast<float*>(ws + P.off_o);
  float* sv = reinterpret_cast<float*>(ws + P.off_v);
  float* sh = reinterpret_cast<float*>(ws + P.off_h);
  float* hpre = reinterpret_cast<float*>(ws + L.off_hpre);
  float* dh = reinterpret_cast<float*>(ws + L.off_dh);
  float* dzw = reinterpret_cast<float*>(ws + L.off_dzw);
  float* dvn = reinterpret_cast<float*>(ws + L.off_dvn);
  float* dyw = reinterpret_cast<float*>(ws + L.off_dyw);
  float* dow = reinterpret_cast<float*>(ws + L.off_dow);
  float2* rt = reinterpret_cast<float2*>(ws + L.off_rt);
  float2* rowstat = reinterpret_cast<float2*>(ws + L.off_rowstat);
  float* y = reinterpret_cast<float*>(ws + L.off_y);
  float* u = reinterpret_cast<float*>(ws + L.off_u);
  float* dq = reinterpret_cast<float*>(ws + L.off_dq);
  float* dk = reinterpret_cast<float*>(ws + L.off_dk);
  float* dv = reinterpret_cast<float*>(ws + L.off_dv);
  float* du = reinterpret_cast<float*>(ws + L.off_du);
  float* part_a = reinterpret_cast<float*>(ws + L.off_part);
  float* part_b = part_a + size_t(kColChunks) * size_t(L.part_cols);
  const float* gamma1 = ln1;
  const float* gamma2 = ln2;

  const std::pair<float*, size_t> zero[] = {
      {dW_Q, size_t(d * d)}, {dW_K, size_t(d * d)}, {dW_V, size_t(d * d)}, {dW_O, size_t(d * d)},
      {dW_1, size_t(d * d_ff)}, {db_1, size_t(d_ff)}, {dW_2, size_t(d_ff * d)}, {db_2, size_t(d)},
      {d_ln1, size_t(2 * d)}, {d_ln2, size_t(2 * d)}, {dk, size_t(M * d)}, {dv, size_t(M * d)}};
  for (const auto& z : zero)
    if (cudaMemsetAsync(z.first, 0, z.second * sizeof(float), s) != cudaSuccess)
      return BPT_ERR_CUDA;
  // C (+)= op(A) op(B) on the CUDA cores
  auto gemm = [&](int64_t m, int64_t n, int64_t k, const float* A, int64_t lda, int a_t,
                  const float* B, int64_t ldb, int b_t, float* C, int64_t ldc, int acc) {
    bpt::GemmGenF32 g{int(m), int(n), int(k), A, lda, a_t, B, ldb, b_t, C, ldc, acc};
    const dim3 grid(unsigned((n + 63) / 64), unsigned((m + 63) / 64));
    bpt::gemm_f32_gen_kernel<<<grid, 256, 0, s>>>(g);
    return cudaGetLastError() == cudaSuccess;
  };
  auto blocks = [](int64_t n) { return unsigned(std::min<int64_t>((n + 255) / 256, 4096)); };
  RowMap ident{0, 1, 1, 1, 1};
  if (launch_ln<float, float, float>(x, ln1, u, M, d, ident, err, s) != cudaSuccess)
    return BPT_ERR_CUDA;
  const float* wqkv[3] = {W_Q, W_K, W_V};
  for (int i = 0; i < 3; ++i)
    if (!gemm(M, d, d, u, d, 0, wqkv[i], d, 0, qkv + i * d, 3 * d, 0)) return BPT_ERR_CUDA;
  const float scale = float(1.0 / std::sqrt(double(P.dk)));
  for (int64_t w = 0; w < P.n_waves; ++w) {
    const Wave wv = P.wave(w);
    const int64_t rows = wv.count * P.blk;
    RowMap map{int(wv.item0), int(P.nb), int(P.N), int(P.blk), 0};
    // forward recomputation of this wave: o, y, LN2(y), FFN pre-activation and hidden
    {
      bpt::AttnF32Params ap{};
      ap.qkv = qkv; ap.o = so; ap.N = int(P.N); ap.nb = int(P.nb); ap.h = int(h);
      ap.d = int(d); ap.causal = P.causal; ap.item0 = int(wv.item0); ap.blk = int(P.blk);
      ap.scale = scale;
      ap.stats = nullptr;
      const size_t smem = size_t(3 * 64 * P.dk + 64 * 65) * 4;
      bpt::attn_f32_kernel<<<unsigned(wv.count * h), 256, smem, s>>>(ap);
      if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
    }
    {
      bpt::GemmF32Params g{};
      g.M = int(rows); g.N = int(d); g.K = int(d); g.n_sub = int(d);
      g.A = so; g.B[0] = g.B[1] = g.B[2] = W_O;
      g.epi = bpt::kEpiResidX; g.out = y; g.ld_out = d; g.resid = x; g.ld_resid = d;
      g.bias = nullptr; g.map = map;
      const dim3 grid(unsigned((d + bpt::kF32Tile - 1) / bpt::kF32Tile),
                      unsigned((rows + bpt::kF32Tile - 1) / bpt::kF32Tile));
      bpt::gemm_f32_kernel<<<grid, 256, 0, s>>>(g);
      if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
    }
    if (launch_ln<float, float, float>(y, ln2, sv, rows, d, map, err, s) != cudaSuccess)
      return BPT_ERR_CUDA;
    if (!gemm(rows, d_ff, d, sv, d, 0, W_1, d_ff, 0, hpre, d_ff, 0)) return BPT_ERR_CUDA;
    bpt::bias_gelu_keep_f32_kernel<<<blocks(rows * d_ff), 256, 0, s>>>(hpre, b_1, sh, rows,
                                                                        int(d_ff));
    // FFN backward
    bpt::gather_rows_f32_kernel<<<blocks(rows * d), 256, 0, s>>>(dZ, dzw, rows, int(d), map);
    if (!gemm(d_ff, d, rows, sh, d_ff, 1, dzw, d, 0, dW_2, d, 1) ||
        !gemm(rows, d_ff, d, dzw, d, 0, W_2, d, 1, dh, d_ff, 0))
      return BPT_ERR_CUDA;
    bpt::gelu_grad_mul_f32_kernel<<<blocks(rows * d_ff), 256, 0, s>>>(dh, hpre, rows * d_ff);
    if (!gemm(d, d_ff, rows, sv, d, 1, dh, d_ff, 0, dW_1, d_ff, 1)) return BPT_ERR_CUDA;
    if (launch_colsum<float, float>(dh, 0, nullptr, nullptr, rows, d_ff, map, part_a, part_b,
                                    db_1, nullptr, s) != cudaSuccess ||
        launch_colsum<float, float>(dZ, 1, nullptr, nullptr, rows, d, map, part_a, part_b, db_2,
                                    nullptr, s) != cudaSuccess)
      return BPT_ERR_CUDA;
    if (!gemm(rows, d, d_ff, dh, d_ff, 0, W_1, d_ff, 1, dvn, d, 0)) return BPT_ERR_CUDA;
    // LN2 backward: dY = dZ + LN2'(dVn) -> dx (global rows), then its wave copy
    bpt::ln_backward_kernel<float, float><<<unsigned((rows * 32 + 255) / 256), 256, 0, s>>>(
        y, gamma2, dvn, dZ, dx, nullptr, rowstat, rows, int(d), map, 0);
    if (launch_colsum<float, float>(dvn, 0, y, rowstat, rows, d, map, part_a, part_b, d_ln2 + d,
                                    d_ln2, s) != cudaSuccess)
      return BPT_ERR_CUDA;
    bpt::gather_rows_f32_kernel<<<blocks(rows * d), 256, 0, s>>>(dx, dyw, rows, int(d), map);
    // W_O backward
    if (!gemm(d, d, rows, so, d, 1, dyw, d, 0, dW_O, d, 1) ||
        !gemm(rows, d, d, dyw, d, 0, W_O, d, 1, dow, d, 0))
      return BPT_ERR_CUDA;
    // attention backward of this wave's query rows
    bpt::attn_row_terms_f32_kernel<<<unsigned((rows * 32 + 255) / 256), 256, 0, s>>>(
        dow, so, reinterpret_cast<const float2*>(stats), rt, rows, int(d), int(h), map);
    bpt::AttnBwdF32Params ab{};
    ab.qkv = qkv; ab.dO = dow; ab.rt = rt; ab.dq = dq; ab.dk = dk; ab.dv = dv;
    ab.rows = rows; ab.N = int(P.N); ab.d = int(d); ab.h = int(h); ab.causal = P.causal;
    ab.scale = scale; ab.map = map;
    bpt::attn_bwd_dq_f32_kernel<<<unsigned((rows * h * 32 + 255) / 256), 256, 0, s>>>(ab);
    bpt::attn_bwd_dkv_f32_kernel<<<unsigned((M * h * 32 + 255) / 256), 256, 0, s>>>(ab, M);
    if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
  }
  // QKV projection and LN1 backward over all rows
  const float* dqkv[3] = {dq, dk, dv};
  float* dWqkv[3] = {dW_Q, dW_K, dW_V};
  for (int i = 0; i < 3; ++i)
    if (!gemm(d, d, M, u, d, 1, dqkv[i], d, 0, dWqkv[i], d, 1) ||
        !gemm(M, d, d, dqkv[i], d, 0, wqkv[i], d, 1, du, d, i > 0 ? 1 : 0))
      return BPT_ERR_CUDA;
  bpt::ln_backward_kernel<float, float><<<unsigned((M * 32 + 255) / 256), 256, 0, s>>>(
      x, gamma1, du, nullptr, dx, nullptr, rowstat, M, int(d), ident, 1);
  if (launch_colsum<float, float>(du, 0, x, rowstat, M, d, ident, part_a, part_b, d_ln1 + d,
                                  d_ln1, s) != cudaSuccess)
    return BPT_ERR_CUDA;
  return BPT_OK;
}

bpt_status backward_bf16(const Plan& P, const BwdLayout& L, const void* x, const void* ln1,
                         const void* W_Q, const void* W_K, const void* W_V, const void* W_O,
                         const void* ln2, const void* W_1, const void* b_1, const void* W_2,
                         const float* stats, const float* dZ, float* dx, float* d_ln1,
                         float* dW_Q, float* dW_K, float* dW_V, float* dW_O, float* d_ln2,
                         float* dW_1, float* db_1, float* dW_2, float* db_2, uint8_t* ws,
                         cudaStream_t s, int sms, const __half* o_keep) {
  using bf = __nv_bfloat16;
  using hf = __half;
  const int64_t M = P.B * P.N, d = P.d, d_ff = P.d_ff, h = P.h;
  const int64_t R = P.P * P.blk;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  hf* w16 = reinterpret_cast<hf*>(ws + P.off_w16);
  hf* wq = w16;
  hf* wk = wq + d * d;
  hf* wv = wk + d * d;
  hf* wo = wv + d * d;
  hf* w1 = wo + d * d;
  hf* w2 = w1 + d * d_ff;
  hf* qkv = reinterpret_cast<hf*>(ws + P.off_qkv);
  hf* so = reinterpret_cast<hf*>(ws + P.off_o);
  hf* sv = reinterpret_cast<hf*>(ws + P.off_v);
  hf* sh = reinterpret_cast<hf*>(ws + P.off_h);
  hf* hpre = reinterpret_cast<hf*>(ws + L.off_hpre);
  hf* dz16 = reinterpret_cast<hf*>(ws + L.off_dz16);
  float* dvn = reinterpret_cast<float*>(ws + L.off_dvn);
  hf* dy16 = reinterpret_cast<hf*>(ws + L.off_dy16);
  hf* do16 = reinterpret_cast<hf*>(ws + L.off_do16);
  float* qs = reinterpret_cast<float*>(ws + L.off_D);
  float2* rowstat = reinterpret_cast<float2*>(ws + L.off_rowstat);
  float* y = reinterpret_cast<float*>(ws + L.off_y);
  hf* u16 = reinterpret_cast<hf*>(ws + L.off_u16);
  float* dq = reinterpret_cast<float*>(ws + L.off_dq);
  float* dk = reinterpret_cast<float*>(ws + L.off_dk);
  float* dv = reinterpret_cast<float*>(ws + L.off_dv);
  hf* dqkv16 = reinterpret_cast<hf*>(ws + L.off_dqkv16);
  float* du = reinterpret_cast<float*>(ws + L.off_du);
  float* part_a = reinterpret_cast<float*>(ws + L.off_part);
  float* part_b = part_a + size_t(kColChunks) * size_t(L.part_cols);
  const bf* gamma1 = static_cast<const bf*>(ln1);
  const bf* gamma2 = static_cast<const bf*>(ln2);

  // Tensor maps (see map_a / map_b): forward recomputation, then the
  // backward's weight-gradient (A = X^T) and data-gradient (B = W^T) GEMMs.
  const int qkv_chunks = (d % 128 == 0) ? 2 : 1;
  CUtensorMap mU, mWq, mWk, mWv, mQKV, mO, mWo, mV, mW1;
  CUtensorMap mHt, mDzB, mDzA, mW2k, mVnt, mHpB, mHpA, mW1k, mOt, mDyB, mDyA, mWok, mUt;
  CUtensorMap mDqB[3], mDqA[3], mWk3[3], mDO;
  bool ok = map_a(&mU, u16, M, d) && map_b(&mWq, wq, d, d, qkv_chunks) &&
            map_b(&mWk, wk, d, d, qkv_chunks) && map_b(&mWv, wv, d, d, qkv_chunks) &&
            map_qkv(&mQKV, qkv, P.B, P.N, d, P.dk) && map_a(&mO, so, R, d) &&
            map_b(&mWo, wo, d, d, 2) && map_a(&mV, sv, R, d) && map_b(&mW1, w1, d, d_ff, 2) &&
            map_b(&mHt, sh, R, d_ff, 2) && map_b(&mDzB, dz16, R, d, 2) &&
            map_a(&mDzA, dz16, R, d) && map_a(&mW2k, w2, d_ff, d) &&
            map_b(&mVnt, sv, R, d, 2) && map_b(&mHpB, hpre, R, d_ff, 2) &&
            map_a(&mHpA, hpre, R, d_ff) && map_a(&mW1k, w1, d, d_ff) &&
            map_b(&mOt, so, R, d, 2) && map_b(&mDyB, dy16, R, d, 2) &&
            map_a(&mDyA, dy16, R, d) && map_a(&mWok, wo, d, d) && map_b(&mUt, u16, M, d, 2) &&
            map_a(&mDO, do16, R, d, 0, int(P.dk / 64));
  CUtensorMap mQKVh;
  if (P.opt.qpc == 4) ok = ok && map_qkv_half(&mQKVh, qkv, P.B, P.N, d);
  if (P.opt.b64) ok = ok && map_q64(&mQKVh, qkv, P.B, P.N, d, P.dk);
  const hf* wqkv[3] = {wq, wk, wv};
  for (int i = 0; i < 3 && ok; ++i)
    ok = map_b(&mDqB[i], dqkv16 + i * d, M, d, 2, 3 * d) &&
         map_a(&mDqA[i], dqkv16 + i * d, M, d, 3 * d) && map_a(&mWk3[i], wqkv[i], d, d);
  if (!ok) return BPT_ERR_CUDA;

  // Zero what is accumulated.
  const std::pair<float*, size_t> zero[] = {
      {dW_Q, size_t(d * d)}, {dW_K, size_t(d * d)}, {dW_V, size_t(d * d)}, {dW_O, size_t(d * d)},
      {dW_1, size_t(d * d_ff)}, {db_1, size_t(d_ff)}, {dW_2, size_t(d_ff * d)}, {db_2, size_t(d)},
      {d_ln1, size_t(2 * d)}, {d_ln2, size_t(2 * d)}, {dk, size_t(M * d)}, {dv, size_t(M * d)}};
  for (const auto& z : zero)
    if (cudaMemsetAsync(z.first, 0, z.second * sizeof(float), s) != cudaSuccess)
      return BPT_ERR_CUDA;
  {
    bpt::CvtSegments cs{};
    const void* src[6] = {W_Q, W_K, W_V, W_O, W_1, W_2};
    hf* dst[6] = {wq, wk, wv, wo, w1, w2};
    const int64_t n[6] = {d * d, d * d, d * d, d * d, d * d_ff, d_ff * d};
    long long acc = 0;
    for (int k = 0; k < 6; ++k) {
      cs.src[k] = static_cast<const bf*>(src[k]);
      cs.dst[k] = dst[k];
      acc += n[k] / 8;
      cs.n8_end[k] = acc;
    }
    cs.count = 6;
    const unsigned grid = unsigned(std::min<long long>((acc + 255) / 256, int64_t(sms) * 8));
    bpt::cvt_bf16_to_f16_kernel<<<grid, 256, 0, s>>>(cs, err);
    if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
  }
  RowMap ident{0, 1, 1, 1, 1};
  if (launch_ln<bf, hf, bf>(static_cast<const bf*>(x), gamma1, u16, M, d, ident, err, s) !=
      cudaSuccess)
    return BPT_ERR_CUDA;
  auto gemm = [&](const CUtensorMap& a, const CUtensorMap& b, int64_t m, int64_t n, int64_t k,
                  int epi, int layout, const RowMap& map, auto&& set) {
    bpt::GemmParams g{};
    g.M = int(m); g.N = int(n); g.K = int(k);
    g.n_sub = int(n); g.n_maps = 1; g.b_chunks = 2;
    g.epi = epi; g.map = map; g.err = err;
    set(g);
    return launch_gemm(a, b, b, b, g, sms, s, layout) == cudaSuccess;
  };
  {
    bpt::GemmParams g{};
    g.M = int(M); g.N = int(3 * d); g.K = int(d);
    g.n_sub = int(d); g.n_maps = 3; g.b_chunks = qkv_chunks;
    g.epi = bpt::kEpiStoreF16; g.out_h = qkv; g.ld_out = 3 * d; g.map = ident; g.err = err;
    if (launch_gemm(mU, mWq, mWk, mWv, g, sms, s) != cudaSuccess) return BPT_ERR_CUDA;
  }
  const float scale = float(1.0 / std::sqrt(double(P.dk)));
  for (int64_t w = 0; w < P.n_waves; ++w) {
    const Wave wv_ = P.wave(w);
    const int64_t rows = wv_.count * P.blk;
    RowMap map{int(wv_.item0), int(P.nb), int(P.N), int(P.blk), 0};
    // forward recomputation of this wave: o (or the forward's, kept), y, LN2(y),
    // FFN pre-activation and hidden
    if (o_keep != nullptr) {
      bpt::rows_copy_f16_kernel<<<unsigned(std::min<int64_t>((rows * d / 8 + 255) / 256,
                                                             int64_t(sms) * 16)),
                                  256, 0, s>>>(o_keep, d, so, d, rows, int(d), map, 0);
    } else if (launch_attn(P, wv_, mQKV, so, nullptr, err, 0, s, nullptr, false, nullptr,
                           &mQKVh) != cudaSuccess) {
      return BPT_ERR_CUDA;
    }
    if (!gemm(mO, mWo, rows, d, d, bpt::kEpiResidX, bpt::kLayAkBn, map, [&](bpt::GemmParams& g) {
          g.out_f32 = y; g.ld_f32 = d; g.resid = static_cast<const bf*>(x); g.ld_resid = d;
        }))
      return BPT_ERR_CUDA;
    if (launch_ln<float, hf, bf>(y, gamma2, sv, rows, d, map, err, s) != cudaSuccess)
      return BPT_ERR_CUDA;
    if (!gemm(mV, mW1, rows, d_ff, d, bpt::kEpiGeluBiasKeep, bpt::kLayAkBn, ident,
              [&](bpt::GemmParams& g) {
                g.out_h = sh; g.out_h2 = hpre; g.ld_out = d_ff;
                g.bias = static_cast<const bf*>(b_1);
              }))
      return BPT_ERR_CUDA;
    // FFN backward
    bpt::rows_f32_to_f16_kernel<<<unsigned(std::min<int64_t>((rows * d / 8 + 255) / 256,
                                                            int64_t(sms) * 16)),
                                  256, 0, s>>>(dZ, dz16, rows, int(d), map);
    if (!gemm(mHt, mDzB, d_ff, d, rows, bpt::kEpiAccumF32, bpt::kLayAnBn, ident,
              [&](bpt::GemmParams& g) { g.out_f32 = dW_2; g.ld_f32 = d; }))
      return BPT_ERR_CUDA;
    if (!gemm(mDzA, mW2k, rows, d_ff, d, bpt::kEpiGeluGrad, bpt::kLayAkBk, ident,
              [&](bpt::GemmParams& g) { g.out_h = hpre; g.ld_out = d_ff; }))
      return BPT_ERR_CUDA;
    if (!gemm(mVnt, mHpB, d, d_ff, rows, bpt::kEpiAccumF32, bpt::kLayAnBn, ident,
              [&](bpt::GemmParams& g) { g.out_f32 = dW_1; g.ld_f32 = d_ff; }))
      return BPT_ERR_CUDA;
    if (launch_colsum<hf, float>(hpre, 0, nullptr, nullptr, rows, d_ff, map, part_a, part_b,
                                 db_1, nullptr, s) != cudaSuccess ||
        launch_colsum<float, float>(dZ, 1, nullptr, nullptr, rows, d, map, part_a, part_b, db_2,
                                    nullptr, s) != cudaSuccess)
      return BPT_ERR_CUDA;
    if (!gemm(mHpA, mW1k, rows, d, d_ff, bpt::kEpiStoreF32, bpt::kLayAkBk, ident,
              [&](bpt::GemmParams& g) { g.out_f32 = dvn; g.ld_f32 = d; }))
      return BPT_ERR_CUDA;
    // LN2 backward: dY = dZ + LN2'(dVn) -> dx (global rows) and dy16 (block rows)
    bpt::ln_backward_kernel<float><<<unsigned((rows * 32 + 255) / 256), 256, 0, s>>>(
        y, gamma2, dvn, dZ, dx, dy16, rowstat, rows, int(d), map, 0);
    if (launch_colsum<float, float>(dvn, 0, y, rowstat, rows, d, map, part_a, part_b, d_ln2 + d,
                                    d_ln2, s) != cudaSuccess)
      return BPT_ERR_CUDA;
    // W_O backward
    if (!gemm(mOt, mDyB, d, d, rows, bpt::kEpiAccumF32, bpt::kLayAnBn, ident,
              [&](bpt::GemmParams& g) { g.out_f32 = dW_O; g.ld_f32 = d; }))
      return BPT_ERR_CUDA;
    if (!gemm(mDyA, mWok, rows, d, d, bpt::kEpiStoreF16, bpt::kLayAkBk, ident,
              [&](bpt::GemmParams& g) { g.out_h = do16; g.ld_out = d; }))
      return BPT_ERR_CUDA;
    // attention backward of this wave's query rows
    bpt::attn_row_terms_kernel<<<unsigned((rows * 32 + 255) / 256), 256, 0, s>>>(
        do16, so, reinterpret_cast<const float2*>(stats), qs, rows, int(d), int(h), map);
    bpt::AttnBwdTcParams ab{};
    ab.N = int(P.N); ab.nb = int(P.nb); ab.h = int(h); ab.d = int(d); ab.causal = P.causal;
    ab.item0 = int(wv_.item0); ab.count = int(wv_.count); ab.seqs = int(wv_.seqs);
    ab.qs = qs;
    ab.dq = dq; ab.dk = dk; ab.dv = dv; ab.scale = scale; ab.err = err;
    int64_t key_end = P.N;
    if (wv_.seqs == 0 && P.causal)
      key_end = std::min<int64_t>(P.N, (wv_.item0 % P.nb + wv_.count) * P.blk);
    const dim3 gq(unsigned(wv_.count), unsigned(h));
    const dim3 gkv(unsigned((key_end + 127) / 128), unsigned(h),
                   unsigned(wv_.seqs > 0 ? wv_.seqs : 1));
    if (P.dk == 128) {
      bpt::attn_bwd_dq_tc_kernel<128>
          <<<gq, bpt::kBwdThreads, bpt::AttnBwdCfg<128>::Q_SMEM, s>>>(mQKV, mDO, ab);
      bpt::attn_bwd_dkv_tc_kernel<128>
          <<<gkv, bpt::kBwdThreads, bpt::AttnBwdCfg<128>::KV_SMEM, s>>>(mQKV, mDO, ab);
    } else {
      bpt::attn_bwd_dq_tc_kernel<64><<<gq, bpt::kBwdThreads, bpt::AttnBwdCfg<64>::Q_SMEM, s>>>(mQKV, mDO, ab);
      bpt::attn_bwd_dkv_tc_kernel<64>
          <<<gkv, bpt::kBwdThreads, bpt::AttnBwdCfg<64>::KV_SMEM, s>>>(mQKV, mDO, ab);
    }
    if (cudaGetLastError() != cudaSuccess) return BPT_ERR_CUDA;
  }
  // QKV projection and LN1 backward over all rows
  bpt::pack3_f32_to_f16_kernel<<<unsigned(std::min<int64_t>((M * 3 * d / 8 + 255) / 256,
                                                           int64_t(sms) * 16)),
                                 256, 0, s>>>(dq, dk, dv, dqkv16, M, int(d));
  float* dWqkv[3] = {dW_Q, dW_K, dW_V};
  for (int i = 0; i < 3; ++i) {
    if (!gemm(mUt, mDqB[i], d, d, M, bpt::kEpiAccumF32, bpt::kLayAnBn, ident,
              [&](bpt::GemmParams& g) { g.out_f32 = dWqkv[i]; g.ld_f32 = d; }))
      return BPT_ERR_CUDA;
    if (!gemm(mDqA[i], mWk3[i], M, d, d, i == 0 ? bpt::kEpiStoreF32 : bpt::kEpiAccumF32,
              bpt::kLayAkBk, ident, [&](bpt::GemmParams& g) { g.out_f32 = du; g.ld_f32 = d; }))
      return BPT_ERR_CUDA;
  }
  bpt::ln_backward_kernel<bf><<<unsigned((M * 32 + 255) / 256), 256, 0, s>>>(
      static_cast<const bf*>(x), gamma1, du, nullptr, dx, nullptr, rowstat, M, int(d), ident, 1);
  if (launch_colsum<float, bf>(du, 0, static_cast<const bf*>(x), rowstat, M, d, ident, part_a,
                               part_b, d_ln1 + d, d_ln1, s) != cudaSuccess)
    return BPT_ERR_CUDA;
  return BPT_OK;
}

// Byte range of a buffer, for overlap checks.
struct Span {
  uintptr_t a, b;
  Span(const void* p, size_t n)
      : a(reinterpret_cast<uintptr_t>(p)), b(reinterpret_cast<uintptr_t>(p) + n) {}
  bool overlaps(const Span& o) const { return a < o.b && o.a < b; }
};

// The forward's input spans (x and every parameter).
std::vector<Span> forward_inputs(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                                 const void* W_V, const void* W_O, const void* ln2,
                                 const void* W_1, const void* b_1, const void* W_2,
                                 const void* b_2, int64_t B, int64_t N, int64_t d, int64_t d_ff,
                                 size_t esize) {
  return {Span(x, size_t(B * N * d) * esize), Span(ln1, size_t(2 * d) * esize),
          Span(W_Q, size_t(d * d) * esize),   Span(W_K, size_t(d * d) * esize),
          Span(W_V, size_t(d * d) * esize),   Span(W_O, size_t(d * d) * esize),
          Span(ln2, size_t(2 * d) * esize),   Span(W_1, size_t(d * d_ff) * esize),
          Span(b_1, size_t(d_ff) * esize),    Span(W_2, size_t(d_ff * d) * esize),
          Span(b_2, size_t(d) * esize)};
}

// Shared body of the forward entry points (stats may be null: no statistics
// are written; gate non-null: gated attention).
bpt_status layer_forward_impl(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                              const void* W_V, const void* W_O, const void* ln2, const void* W_1,
                              const void* b_1, const void* W_2, const void* b_2, int64_t B,
                              int64_t N, int64_t d, int64_t h, int64_t d_ff, int causal,
                              bpt_dtype dtype, float* out, float* stats, void* workspace,
                              size_t workspace_bytes, const bpt_options* opts,
                              bpt_stream_t stream, const AttnGate* gate = nullptr,
                              void* o_keep = nullptr) {
  bpt_status st = check_shape(B, N, d, h, d_ff, causal, dtype);
  if (st != BPT_OK) return st;
  Opts opt;
  st = read_opts(opts, &opt);
  if (st != BPT_OK) return st;
  if (gate != nullptr && dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  if (o_keep != nullptr && dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  // the b = 512 cluster and the b = 64 kernel are dense
  if (gate != nullptr && (opt.qpc == 4 || opt.b64)) return BPT_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return BPT_OK;
  const void* ptrs[] = {x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, out, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || misaligned(p)) return BPT_ERR_INVALID_ARG;
  const Plan P = make_plan(B, N, d, h, d_ff, causal, dtype, opt);
  if (workspace_bytes < P.total) return BPT_ERR_WORKSPACE;
  // out and the workspace are written while the inputs are still read: they
  // must overlap no input and not each other; stats likewise.
  const std::vector<Span> ins =
      forward_inputs(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, d_ff, P.esize);
  const Span so(out, size_t(B * N * d) * 4), sw(workspace, P.total);
  if (so.overlaps(sw)) return BPT_ERR_INVALID_ARG;
  for (const Span& in : ins)
    if (so.overlaps(in) || sw.overlaps(in)) return BPT_ERR_INVALID_ARG;
  if (stats != nullptr) {
    const Span ss(stats, size_t(B * h * N) * 2 * sizeof(float));
    if (misaligned(stats) || ss.overlaps(so) || ss.overlaps(sw)) return BPT_ERR_INVALID_ARG;
    for (const Span& in : ins)
      if (ss.overlaps(in)) return BPT_ERR_INVALID_ARG;
  }
  if (o_keep != nullptr) {
    const Span sk(o_keep, size_t(B * N * d) * 2);
    if (misaligned(o_keep) || sk.overlaps(so) || sk.overlaps(sw)) return BPT_ERR_INVALID_ARG;
    if (stats != nullptr && sk.overlaps(Span(stats, size_t(B * h * N) * 2 * sizeof(float))))
      return BPT_ERR_INVALID_ARG;
    for (const Span& in : ins)
      if (sk.overlaps(in)) return BPT_ERR_INVALID_ARG;
  }
  if (opt.fault != 0 && dtype != BPT_BF16) return BPT_ERR_INVALID_ARG;

  int sms = 0;
  st = device_info(&sms);
  if (st != BPT_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, s) != cudaSuccess) return BPT_ERR_CUDA;
  if (dtype == BPT_BF16) {
    st = get_encoder();
    if (st != BPT_OK) return st;
    return forward_bf16(P, x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, out, stats, ws, s,
                        sms, gate, nullptr, static_cast<__half*>(o_keep));
  }
  return forward_f32(P, static_cast<const float*>(x), static_cast<const float*>(ln1),
                     static_cast<const float*>(W_Q), static_cast<const float*>(W_K),
                     static_cast<const float*>(W_V), static_cast<const float*>(W_O),
                     static_cast<const float*>(ln2), static_cast<const float*>(W_1),
                     static_cast<const float*>(b_1), static_cast<const float*>(W_2),
                     static_cast<const float*>(b_2), out, stats, ws, s);
}

bpt_status bsfa_impl(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                     const void* W_V, const void* W_O, const void* ln2, const void* W_1,
                     const void* b_1, const void* W_2, const void* b_2, int64_t B, int64_t N,
                     int64_t d, int64_t h, int64_t d_ff, int causal, bpt_dtype dtype,
                     const float* thresholds, float* block_max, uint8_t* kept, float* out,
                     void* workspace, size_t workspace_bytes, const bpt_options* opts,
                     bpt_stream_t stream) {
  bpt_status st = check_shape(B, N, d, h, d_ff, causal, dtype);
  if (st != BPT_OK) return st;
  if (dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  if (thresholds == nullptr) return BPT_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return BPT_OK;
  const size_t nb = size_t((N + 127) / 128);
  const size_t tbytes = size_t(h) * nb * 4, pairs = size_t(B) * size_t(h) * nb * nb;
  const Span o(out, size_t(B * N * d) * 4), w(workspace, workspace_bytes),
      t(thresholds, tbytes);
  const std::vector<Span> ins =
      forward_inputs(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, d_ff, 2);
  if ((reinterpret_cast<uintptr_t>(thresholds) & 3u) || t.overlaps(o) || t.overlaps(w))
    return BPT_ERR_INVALID_ARG;
  if (block_max != nullptr) {
    const Span m(block_max, pairs * 4);
    if ((reinterpret_cast<uintptr_t>(block_max) & 3u) || m.overlaps(o) || m.overlaps(w) ||
        m.overlaps(t))
      return BPT_ERR_INVALID_ARG;
    for (const Span& in : ins)
      if (m.overlaps(in)) return BPT_ERR_INVALID_ARG;
  }
  if (kept != nullptr) {
    const Span k(kept, pairs);
    if (k.overlaps(o) || k.overlaps(w) || k.overlaps(t) ||
        (block_max != nullptr && k.overlaps(Span(block_max, pairs * 4))))
      return BPT_ERR_INVALID_ARG;
    for (const Span& in : ins)
      if (k.overlaps(in)) return BPT_ERR_INVALID_ARG;
  }
  const AttnGate gate{thresholds, block_max, kept};
  return layer_forward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff,
                            causal, dtype, out, nullptr, workspace, workspace_bytes, opts, stream,
                            &gate);
}

bpt_status backward_impl(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                         const void* W_V, const void* W_O, const void* ln2, const void* W_1,
                         const void* b_1, const void* W_2, const void* b_2, const float* stats,
                         const float* dZ, int64_t B, int64_t N, int64_t d, int64_t h,
                         int64_t d_ff, int causal, bpt_dtype dtype, float* dx, float* d_ln1,
                         float* dW_Q, float* dW_K, float* dW_V, float* dW_O, float* d_ln2,
                         float* dW_1, float* db_1, float* dW_2, float* db_2, void* workspace,
                         size_t workspace_bytes, const bpt_options* opts, bpt_stream_t stream,
                         const void* o_keep = nullptr) {
  (void)b_2;  // the output's bias does not enter any gradient but its own
  bpt_status st = check_shape(B, N, d, h, d_ff, causal, dtype);
  if (st != BPT_OK) return st;
  if (o_keep != nullptr && dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  Opts opt;
  st = read_opts(opts, &opt);
  if (st != BPT_OK) return st;
  if (opt.fault != 0) return BPT_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return BPT_OK;
  const void* ins[] = {x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats, dZ, workspace};
  for (const void* p : ins)
    if (p == nullptr || misaligned(p)) return BPT_ERR_INVALID_ARG;
  float* outs[] = {dx, d_ln1, dW_Q, dW_K, dW_V, dW_O, d_ln2, dW_1, db_1, dW_2, db_2};
  const size_t out_bytes[] = {size_t(B * N * d) * 4, size_t(2 * d) * 4, size_t(d * d) * 4,
                              size_t(d * d) * 4, size_t(d * d) * 4, size_t(d * d) * 4,
                              size_t(2 * d) * 4, size_t(d * d_ff) * 4, size_t(d_ff) * 4,
                              size_t(d_ff * d) * 4, size_t(d) * 4};
  const Plan P = make_plan(B, N, d, h, d_ff, causal, dtype, opt, false);
  const size_t ws_need =
      dtype == BPT_BF16 ? make_bwd_layout(P).total : make_bwd_layout_f32(P).total;
  if (workspace_bytes < ws_need) return BPT_ERR_WORKSPACE;
  // Outputs must be aligned and must not overlap each other, the workspace,
  // or any input (every input is read after some output is first written).
  std::vector<Span> reads =
      forward_inputs(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, d_ff, P.esize);
  reads.push_back(Span(stats, size_t(B * h * N) * 8));
  reads.push_back(Span(dZ, size_t(B * N * d) * 4));
  if (o_keep != nullptr) {
    if (misaligned(o_keep)) return BPT_ERR_INVALID_ARG;
    reads.push_back(Span(o_keep, size_t(B * N * d) * 2));
  }
  const Span sw(workspace, ws_need);
  for (const Span& r : reads)
    if (sw.overlaps(r)) return BPT_ERR_INVALID_ARG;
  reads.push_back(sw);
  for (int i = 0; i < 11; ++i) {
    if (outs[i] == nullptr || misaligned(outs[i])) return BPT_ERR_INVALID_ARG;
    const Span a(outs[i], out_bytes[i]);
    for (const Span& r : reads)
      if (a.overlaps(r)) return BPT_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (a.overlaps(Span(outs[j], out_bytes[j]))) return BPT_ERR_INVALID_ARG;
  }
  int sms = 0;
  st = device_info(&sms);
  if (st != BPT_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, s) != cudaSuccess) return BPT_ERR_CUDA;
  if (dtype == BPT_F32) {
    auto f = [](const void* q) { return static_cast<const float*>(q); };
    return backward_f32(P, make_bwd_layout_f32(P), f(x), f(ln1), f(W_Q), f(W_K), f(W_V), f(W_O),
                        f(ln2), f(W_1), f(b_1), f(W_2), stats, dZ, dx, d_ln1, dW_Q, dW_K, dW_V,
                        dW_O, d_ln2, dW_1, db_1, dW_2, db_2, ws, s);
  }
  st = get_encoder();
  if (st != BPT_OK) return st;
  const BwdLayout L = make_bwd_layout(P);
  return backward_bf16(P, L, x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, stats, dZ, dx, d_ln1,
                       dW_Q, dW_K, dW_V, dW_O, d_ln2, dW_1, db_1, dW_2, db_2, ws, s, sms,
                       static_cast<const __half*>(o_keep));
}

// Shared body of the sequence-shard entry points (phase 1: projection into
// kv_loc; phase 2: attention against kv_all + layer body).
bpt_status shard_impl(int phase, const void* x, const void* ln1, const void* W_Q,
                      const void* W_K, const void* W_V, const void* W_O, const void* ln2,
                      const void* W_1, const void* b_1, const void* W_2, const void* b_2,
                      int64_t B, int64_t N, int64_t G, int64_t rank, int64_t d, int64_t h,
                      int64_t d_ff, int causal, bpt_dtype dtype, void* kv, float* out,
                      void* workspace, size_t workspace_bytes, bpt_stream_t stream) {
  if (G < 1 || rank < 0 || rank >= G || N <= 0 || B <= 0) return BPT_ERR_INVALID_ARG;
  if (dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  if (N % (256 * G) != 0) return BPT_ERR_UNSUPPORTED;  // 2G chunks of whole blocks
  const int64_t n_loc = N / G;
  bpt_status st = check_shape(B, n_loc, d, h, d_ff, causal, dtype);
  if (st != BPT_OK) return st;
  if (B * N > (int64_t(1) << 30)) return BPT_ERR_UNSUPPORTED;
  const void* ptrs[] = {x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, out, workspace, kv};
  for (const void* p : ptrs)
    if (p == nullptr || misaligned(p)) return BPT_ERR_INVALID_ARG;
  const Plan P = make_plan(B, n_loc, d, h, d_ff, causal, dtype);
  if (workspace_bytes < P.total) return BPT_ERR_WORKSPACE;
  const std::vector<Span> ins =
      forward_inputs(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, n_loc, d, d_ff, 2);
  const Span so(out, size_t(B * n_loc * d) * 4), sw(workspace, P.total);
  const Span sk(kv, size_t(phase == 1 ? 1 : G) * size_t(B * n_loc * 2 * d) * 2);
  if (so.overlaps(sw) || sk.overlaps(so) || sk.overlaps(sw)) return BPT_ERR_INVALID_ARG;
  for (const Span& in : ins)
    if (so.overlaps(in) || sw.overlaps(in) || (phase == 1 && sk.overlaps(in)))
      return BPT_ERR_INVALID_ARG;
  int sms = 0;
  st = device_info(&sms);
  if (st != BPT_OK) return st;
  st = get_encoder();
  if (st != BPT_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (phase == 1 && cudaMemsetAsync(ws, 0, kHeaderBytes, s) != cudaSuccess) return BPT_ERR_CUDA;
  ShardSpec sh{};
  sh.phase = phase;
  sh.G = int(G);
  sh.rank = int(rank);
  sh.N = N;
  sh.kv_loc = phase == 1 ? static_cast<__half*>(kv) : nullptr;
  sh.kv_all = phase == 2 ? kv : nullptr;
  return forward_bf16(P, x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, out, nullptr, ws, s,
                      sms, nullptr, &sh);
}

bpt_status plan_for(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff, int causal,
                    bpt_dtype dtype, const bpt_options* opts, bool forward, Plan* P) {
  bpt_status st = check_shape(B, N, d, h, d_ff, causal, dtype);
  if (st != BPT_OK) return st;
  Opts opt;
  st = read_opts(opts, &opt);
  if (st != BPT_OK) return st;
  *P = make_plan(B, N, d, h, d_ff, causal, dtype, opt, forward);
  return BPT_OK;
}

// Device address of the allocation-free entry point's array (defined below).
bpt_status static_ws_address(void** ptr);

extern "C" {

bpt_status bpt_layer_workspace_size_opt(int64_t B, int64_t N, int64_t d, int64_t h,
                                        int64_t d_ff, int causal, bpt_dtype dtype,
                                        const bpt_options* opts, size_t* bytes) {
  if (!bytes) return BPT_ERR_INVALID_ARG;
  Plan P;
  const bpt_status st = plan_for(B, N, d, h, d_ff, causal, dtype, opts, true, &P);
  if (st != BPT_OK) return st;
  *bytes = P.total;
  return BPT_OK;
}

bpt_status bpt_layer_workspace_size(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                    int causal, bpt_dtype dtype, size_t* bytes) {
  return bpt_layer_workspace_size_opt(B, N, d, h, d_ff, causal, dtype, nullptr, bytes);
}

bpt_status bpt_layer_launch_count_opt(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                      int causal, bpt_dtype dtype, const bpt_options* opts,
                                      int64_t* launches) {
  if (!launches) return BPT_ERR_INVALID_ARG;
  Plan P;
  const bpt_status st = plan_for(B, N, d, h, d_ff, causal, dtype, opts, true, &P);
  if (st != BPT_OK) return st;
  if (P.items == 0)
    *launches = 0;
  else if (P.fused)
    *launches = 5;  // weight copy, LN1, QKV GEMM, attention, tail
  else
    *launches = (dtype == BPT_BF16 ? 3 : 2) + 5 * P.n_waves;
  return BPT_OK;
}

bpt_status bpt_layer_launch_count(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                  int causal, bpt_dtype dtype, int64_t* launches) {
  return bpt_layer_launch_count_opt(B, N, d, h, d_ff, causal, dtype, nullptr, launches);
}

bpt_status bpt_layer_tail_plan(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                               int causal, int32_t resident_pairs, int32_t* pairs,
                               int32_t* shared, int32_t* plan, int32_t plan_rows) {
  if (!pairs || !shared || resident_pairs < 1 || resident_pairs > BPT_TAIL_MAX_PAIRS ||
      plan_rows < 0 || (plan == nullptr && plan_rows > 0))
    return BPT_ERR_INVALID_ARG;
  Plan P;
  const bpt_status st = plan_for(B, N, d, h, d_ff, causal, BPT_BF16, nullptr, true, &P);
  if (st != BPT_OK) return st;
  *pairs = 0;
  *shared = 0;
  if (P.items == 0) return BPT_OK;
  // as the fused forward launches the layer body
  bpt::TailParams tp{};
  tp.blocks = int(P.items);
  tp.items = int((P.items + 1) / 2);
  const int np = int(std::max<int64_t>(1, std::min<int64_t>(P.tail_pairs, resident_pairs)));
  tp.split = (BPT_TAIL_SHARE_ITEMS && bpt::tail_shares(tp.items, np, int(d), int(d_ff))) ? 1 : 0;
  *pairs = np;
  *shared = tp.split ? tp.items % np : 0;
  for (int q = 0; q < std::min(np, int(plan_rows)); ++q) {
    const bpt::TailPlan pl = bpt::tail_plan(tp, q, np);
    int32_t* r = plan + 5 * q;
    r[0] = pl.J;
    r[1] = pl.Jfull;
    r[2] = pl.half >= 0 ? pl.hitem : -1;
    r[3] = pl.half;
    r[4] = pl.half >= 0 ? pl.partner : -1;
  }
  return BPT_OK;
}

bpt_status bpt_layer_forward(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                             const void* W_V, const void* W_O, const void* ln2, const void* W_1,
                             const void* b_1, const void* W_2, const void* b_2, int64_t B,
                             int64_t N, int64_t d, int64_t h, int64_t d_ff, int causal,
                             bpt_dtype dtype, float* out, void* workspace, size_t workspace_bytes,
                             bpt_stream_t stream) {
  return layer_forward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff,
                            causal, dtype, out, nullptr, workspace, workspace_bytes, nullptr,
                            stream);
}

bpt_status bpt_layer_forward_opt(const void* x, const void* ln1, const void* W_Q,
                                 const void* W_K, const void* W_V, const void* W_O,
                                 const void* ln2, const void* W_1, const void* b_1,
                                 const void* W_2, const void* b_2, int64_t B, int64_t N,
                                 int64_t d, int64_t h, int64_t d_ff, int causal, bpt_dtype dtype,
                                 float* out, float* stats, void* workspace,
                                 size_t workspace_bytes, const bpt_options* opts,
                                 bpt_stream_t stream) {
  return layer_forward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff,
                            causal, dtype, out, stats, workspace, workspace_bytes, opts, stream);
}

bpt_status bpt_layer_forward_train(const void* x, const void* ln1, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O,
                                   const void* ln2, const void* W_1, const void* b_1,
                                   const void* W_2, const void* b_2, int64_t B, int64_t N,
                                   int64_t d, int64_t h, int64_t d_ff, int causal,
                                   bpt_dtype dtype, float* out, float* stats, void* workspace,
                                   size_t workspace_bytes, bpt_stream_t stream) {
  if (stats == nullptr) return BPT_ERR_INVALID_ARG;
  return layer_forward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff,
                            causal, dtype, out, stats, workspace, workspace_bytes, nullptr,
                            stream);
}

bpt_status bpt_layer_forward_train_keep_o(const void* x, const void* ln1, const void* W_Q,
                                          const void* W_K, const void* W_V, const void* W_O,
                                          const void* ln2, const void* W_1, const void* b_1,
                                          const void* W_2, const void* b_2, int64_t B,
                                          int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                          int causal, bpt_dtype dtype, float* out, float* stats,
                                          void* o, void* workspace, size_t workspace_bytes,
                                          const bpt_options* opts, bpt_stream_t stream) {
  if (stats == nullptr || o == nullptr) return BPT_ERR_INVALID_ARG;
  return layer_forward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff,
                            causal, dtype, out, stats, workspace, workspace_bytes, opts, stream,
                            nullptr, o);
}

bpt_status bpt_layer_forward_bsfa(const void* x, const void* ln1, const void* W_Q,
                                  const void* W_K, const void* W_V, const void* W_O,
                                  const void* ln2, const void* W_1, const void* b_1,
                                  const void* W_2, const void* b_2, int64_t B, int64_t N,
                                  int64_t d, int64_t h, int64_t d_ff, int causal,
                                  bpt_dtype dtype, const float* thresholds, float* block_max,
                                  uint8_t* kept, float* out, void* workspace,
                                  size_t workspace_bytes, bpt_stream_t stream) {
  return bsfa_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff, causal,
                   dtype, thresholds, block_max, kept, out, workspace, workspace_bytes, nullptr,
                   stream);
}

bpt_status bpt_layer_forward_bsfa_opt(const void* x, const void* ln1, const void* W_Q,
                                      const void* W_K, const void* W_V, const void* W_O,
                                      const void* ln2, const void* W_1, const void* b_1,
                                      const void* W_2, const void* b_2, int64_t B, int64_t N,
                                      int64_t d, int64_t h, int64_t d_ff, int causal,
                                      bpt_dtype dtype, const float* thresholds, float* block_max,
                                      uint8_t* kept, float* out, void* workspace,
                                      size_t workspace_bytes, const bpt_options* opts,
                                      bpt_stream_t stream) {
  return bsfa_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff, causal,
                   dtype, thresholds, block_max, kept, out, workspace, workspace_bytes, opts,
                   stream);
}

bpt_status bpt_layer_backward_workspace_size_opt(int64_t B, int64_t N, int64_t d, int64_t h,
                                                 int64_t d_ff, int causal, bpt_dtype dtype,
                                                 const bpt_options* opts, size_t* bytes) {
  if (bytes == nullptr) return BPT_ERR_INVALID_ARG;
  Plan P;
  const bpt_status st = plan_for(B, N, d, h, d_ff, causal, dtype, opts, false, &P);
  if (st != BPT_OK) return st;
  *bytes = dtype == BPT_BF16 ? make_bwd_layout(P).total : make_bwd_layout_f32(P).total;
  return BPT_OK;
}

bpt_status bpt_layer_backward_workspace_size(int64_t B, int64_t N, int64_t d, int64_t h,
                                             int64_t d_ff, int causal, bpt_dtype dtype,
                                             size_t* bytes) {
  return bpt_layer_backward_workspace_size_opt(B, N, d, h, d_ff, causal, dtype, nullptr, bytes);
}

bpt_status bpt_layer_backward(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                              const void* W_V, const void* W_O, const void* ln2, const void* W_1,
                              const void* b_1, const void* W_2, const void* b_2,
                              const float* stats, const float* dZ, int64_t B, int64_t N,
                              int64_t d, int64_t h, int64_t d_ff, int causal, bpt_dtype dtype,
                              float* dx, float* d_ln1, float* dW_Q, float* dW_K, float* dW_V,
                              float* dW_O, float* d_ln2, float* dW_1, float* db_1, float* dW_2,
                              float* db_2, void* workspace, size_t workspace_bytes,
                              bpt_stream_t stream) {
  return backward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats, dZ, B, N, d, h,
                       d_ff, causal, dtype, dx, d_ln1, dW_Q, dW_K, dW_V, dW_O, d_ln2, dW_1, db_1,
                       dW_2, db_2, workspace, workspace_bytes, nullptr, stream);
}

bpt_status bpt_layer_backward_opt(const void* x, const void* ln1, const void* W_Q,
                                  const void* W_K, const void* W_V, const void* W_O,
                                  const void* ln2, const void* W_1, const void* b_1,
                                  const void* W_2, const void* b_2, const float* stats,
                                  const float* dZ, int64_t B, int64_t N, int64_t d, int64_t h,
                                  int64_t d_ff, int causal, bpt_dtype dtype, float* dx,
                                  float* d_ln1, float* dW_Q, float* dW_K, float* dW_V,
                                  float* dW_O, float* d_ln2, float* dW_1, float* db_1,
                                  float* dW_2, float* db_2, void* workspace,
                                  size_t workspace_bytes, const bpt_options* opts,
                                  bpt_stream_t stream) {
  return backward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats, dZ, B, N, d, h,
                       d_ff, causal, dtype, dx, d_ln1, dW_Q, dW_K, dW_V, dW_O, d_ln2, dW_1, db_1,
                       dW_2, db_2, workspace, workspace_bytes, opts, stream);
}

bpt_status bpt_layer_backward_keep_o(const void* x, const void* ln1, const void* W_Q,
                                     const void* W_K, const void* W_V, const void* W_O,
                                     const void* ln2, const void* W_1, const void* b_1,
                                     const void* W_2, const void* b_2, const float* stats,
                                     const void* o, const float* dZ, int64_t B, int64_t N,
                                     int64_t d, int64_t h, int64_t d_ff, int causal,
                                     bpt_dtype dtype, float* dx, float* d_ln1, float* dW_Q,
                                     float* dW_K, float* dW_V, float* dW_O, float* d_ln2,
                                     float* dW_1, float* db_1, float* dW_2, float* db_2,
                                     void* workspace, size_t workspace_bytes,
                                     const bpt_options* opts, bpt_stream_t stream) {
  if (o == nullptr) return BPT_ERR_INVALID_ARG;
  return backward_impl(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, stats, dZ, B, N, d, h,
                       d_ff, causal, dtype, dx, d_ln1, dW_Q, dW_K, dW_V, dW_O, d_ln2, dW_1, db_1,
                       dW_2, db_2, workspace, workspace_bytes, opts, stream, o);
}

bpt_status bpt_layer_shard_workspace_size(int64_t B, int64_t N, int64_t G, int64_t d,
                                          int64_t h, int64_t d_ff, int causal, bpt_dtype dtype,
                                          size_t* bytes) {
  if (bytes == nullptr || G < 1 || N <= 0 || B <= 0) return BPT_ERR_INVALID_ARG;
  if (dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  if (N % (256 * G) != 0) return BPT_ERR_UNSUPPORTED;
  return bpt_layer_workspace_size(B, N / G, d, h, d_ff, causal, dtype, bytes);
}

bpt_status bpt_layer_shard_project(const void* x, const void* ln1, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O,
                                   const void* ln2, const void* W_1, const void* b_1,
                                   const void* W_2, const void* b_2, int64_t B, int64_t N,
                                   int64_t G, int64_t rank, int64_t d, int64_t h, int64_t d_ff,
                                   int causal, bpt_dtype dtype, void* kv_loc, float* out,
                                   void* workspace, size_t workspace_bytes,
                                   bpt_stream_t stream) {
  return shard_impl(1, x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, G, rank, d, h,
                    d_ff, causal, dtype, kv_loc, out, workspace, workspace_bytes, stream);
}

bpt_status bpt_layer_shard_forward(const void* x, const void* ln1, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O,
                                   const void* ln2, const void* W_1, const void* b_1,
                                   const void* W_2, const void* b_2, int64_t B, int64_t N,
                                   int64_t G, int64_t rank, int64_t d, int64_t h, int64_t d_ff,
                                   int causal, bpt_dtype dtype, const void* kv_all, float* out,
                                   void* workspace, size_t workspace_bytes,
                                   bpt_stream_t stream) {
  return shard_impl(2, x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, G, rank, d, h,
                    d_ff, causal, dtype, const_cast<void*>(kv_all), out, workspace,
                    workspace_bytes, stream);
}

bpt_status bpt_read_device_error(void* workspace, bpt_stream_t stream, uint32_t* site) {
  if (!workspace) {
    const bpt_status st = static_ws_address(&workspace);
    if (st != BPT_OK) return st;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BPT_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return BPT_ERR_CUDA;
  if (word == 0) {
    if (site) *site = 0;
    return BPT_OK;
  }
  if (cudaMemset(workspace, 0, 4) != cudaSuccess) return BPT_ERR_CUDA;
  if (site) *site = word >> 8;
  return static_cast<bpt_status>(word & 0xFFu);
}

const char* bpt_status_string(bpt_status status) {
  switch (status) {
    case BPT_OK: return "BPT_OK";
    case BPT_ERR_INVALID_ARG: return "BPT_ERR_INVALID_ARG: null or misaligned pointer, or inconsistent sizes";
    case BPT_ERR_UNSUPPORTED: return "BPT_ERR_UNSUPPORTED: shape or device not handled by the kernels";
    case BPT_ERR_WORKSPACE: return "BPT_ERR_WORKSPACE: workspace smaller than bpt_layer_workspace_size";
    case BPT_ERR_CUDA: return "BPT_ERR_CUDA: a CUDA call failed";
    case BPT_ERR_TIMEOUT: return "BPT_ERR_TIMEOUT: a kernel gave up waiting on a barrier";
    case BPT_ERR_RANGE: return "BPT_ERR_RANGE: a tensor-core operand exceeded the fp16 range";
  }
  return "BPT_UNKNOWN_STATUS";
}

bpt_status bpt_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_prof_on = enable != 0;
  return BPT_OK;
}

bpt_status bpt_profile_read(double* ms, int64_t* launches, int n) {
  std::lock_guard<std::mutex> lk(g_mu);
  bpt_status st = BPT_OK;
  for (const ProfRec& r : g_prof) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      st = BPT_ERR_CUDA;
    if (r.kind < n) {
      if (ms) ms[r.kind] += double(t);
      if (launches) launches[r.kind] += 1;
    }
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  return st;
}

}  // extern "C"

// ------------------------------------------------ allocation-free variant --
// Workspace of bpt_layer_forward_static: a file-scope device array, so that
// callers that may not allocate still get the full layer.  In host code the
// symbol is only a stand-in; its device address comes from
// cudaGetSymbolAddress, looked up with the device current and cached per
// (device, CUDA context): a caller that switches contexts, or a context
// created after a device reset, gets a fresh lookup.
static __device__ __align__(256) uint8_t g_bpt_static_ws[BPT_STATIC_WORKSPACE_BYTES];

namespace {
struct StaticWs {
  void* ctx = nullptr;
  void* ptr = nullptr;
};
StaticWs g_static_ws[64];
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
}  // namespace

bpt_status static_ws_address(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BPT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ctx_get_current == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return BPT_ERR_CUDA;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return BPT_ERR_CUDA;
  StaticWs& e = g_static_ws[dev];
  if (ctx == nullptr || e.ptr == nullptr || e.ctx != static_cast<void*>(ctx)) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bpt_static_ws) != cudaSuccess || p == nullptr)
      return BPT_ERR_CUDA;
    // the lookup made the runtime's context current if none was
    if (ctx == nullptr && (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr))
      return BPT_ERR_CUDA;
    e.ctx = static_cast<void*>(ctx);
    e.ptr = p;
  }
  *ptr = e.ptr;
  return BPT_OK;
}

extern "C" bpt_status bpt_layer_forward_static(const void* x, const void* ln1, const void* W_Q,
                                               const void* W_K, const void* W_V, const void* W_O,
                                               const void* ln2, const void* W_1, const void* b_1,
                                               const void* W_2, const void* b_2, int64_t B,
                                               int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                               int causal, bpt_dtype dtype, float* out,
                                               bpt_stream_t stream) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_prof_on) return BPT_ERR_INVALID_ARG;
  }
  bpt_status st = check_shape(B, N, d, h, d_ff, causal, dtype);
  if (st != BPT_OK) return st;
  if (B == 0 || N == 0) return BPT_OK;
  const void* ptrs[] = {x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, out};
  for (const void* p : ptrs)
    if (p == nullptr || misaligned(p)) return BPT_ERR_INVALID_ARG;
  if (make_plan(B, N, d, h, d_ff, causal, dtype).total > size_t(BPT_STATIC_WORKSPACE_BYTES))
    return BPT_ERR_WORKSPACE;
  void* ws = nullptr;
  st = static_ws_address(&ws);
  if (st != BPT_OK) return st;
  return bpt_layer_forward(x, ln1, W_Q, W_K, W_V, W_O, ln2, W_1, b_1, W_2, b_2, B, N, d, h, d_ff,
                           causal, dtype, out, ws, size_t(BPT_STATIC_WORKSPACE_BYTES), stream);
}
