// Host side of the C ABI declared in include/prism.h: argument validation,
// workspace layout, TMA descriptors and the kernel launch sequence.
//
// Method: "Prism: Spectral-Aware Block-Sparse Attention" -- the
// paper.rainbus.top review's method paragraph, steps (1)-(7), and the
// gist.science Technical Summary, sections 1, 2A and 2B.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/prism.h"
#include "attention.cuh"
#include "estimate.cuh"

namespace {

using namespace prism;

constexpr int kVersion = 100;  // 0.1.0

// ---------------------------------------------------------------------------
// validated problem description and workspace layout
// ---------------------------------------------------------------------------
struct Plan {
  int b, hq, hkv, n, nb, W;
  int q_rows, kv_rows;
  BandLayout bl;
  float p_eff;
  int explicit_tau;
  float tau_hi, tau_lo;
  float scale;
  int force;
  int varlen;            // per-sequence lengths given
  int seq_n[kMaxSeqs];   // tokens of each batch element (n when not varlen)
  size_t off_pool[kTerms], off_part, off_tau, off_scores, off_sync, sync_bytes, est_bytes, off_mask, total;
};
static_assert(kMaxSeqs == attn::kMaxSeqs, "one sequence limit for both kernels");

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int validate(const prism_config* cfg, Plan* pl) {
  if (!cfg) return PRISM_ERR_NULL;
  if (cfg->batch <= 0 || cfg->hq <= 0 || cfg->hkv <= 0 || cfg->seqlen <= 0) return PRISM_ERR_SHAPE;
  if (cfg->head_dim != 128 || cfg->block != 128 || cfg->causal != 1) return PRISM_ERR_UNSUPPORTED;
  if (cfg->hq % cfg->hkv != 0) return PRISM_ERR_SHAPE;
  if (cfg->hq / cfg->hkv > kMaxGroupHeads) return PRISM_ERR_UNSUPPORTED;
  const long long nb = ((long long)cfg->seqlen + cfg->block - 1) / cfg->block;  // the last block may be short
  // TMA row coordinates are 32-bit; Top-P indices are 16-bit
  if ((long long)cfg->batch * cfg->hq * cfg->seqlen >= (1ll << 31)) return PRISM_ERR_SHAPE;
  if (nb > 16384) return PRISM_ERR_UNSUPPORTED;
  if (cfg->tau_mode != PRISM_TAU_RMS && cfg->tau_mode != PRISM_TAU_EXPLICIT) return PRISM_ERR_UNSUPPORTED;
  if (cfg->tau_mode == PRISM_TAU_EXPLICIT &&
      (!(cfg->tau_hi > 0.f) || !(cfg->tau_lo > 0.f) || !std::isfinite(cfg->tau_hi) ||
       !std::isfinite(cfg->tau_lo)))
    return PRISM_ERR_TAU;
  if (!(cfg->p > 0.f)) return PRISM_ERR_P;  // also rejects NaN
  if (cfg->force_blocks & ~(PRISM_FORCE_SINK | PRISM_FORCE_DIAG)) return PRISM_ERR_UNSUPPORTED;
  if (cfg->seqlens) {  // one length per batch element, 1 .. seqlen
    if (cfg->batch > kMaxSeqs) return PRISM_ERR_UNSUPPORTED;
    for (int x = 0; x < cfg->batch; ++x)
      if (cfg->seqlens[x] < 1 || cfg->seqlens[x] > cfg->seqlen) return PRISM_ERR_SHAPE;
  }
  if (!cfg->band_hi || !cfg->band_lo) return PRISM_ERR_NULL;
  if (cfg->n_hi <= 0 || cfg->n_lo <= 0 || cfg->n_hi > 128 || cfg->n_lo > 128) return PRISM_ERR_BAND;
  bool in_hi[128] = {}, in_lo[128] = {};
  for (int x = 0; x < cfg->n_hi; ++x) {
    const int d = cfg->band_hi[x];
    if (d < 0 || d >= 128 || in_hi[d]) return PRISM_ERR_BAND;
    in_hi[d] = true;
  }
  for (int x = 0; x < cfg->n_lo; ++x) {
    const int d = cfg->band_lo[x];
    if (d < 0 || d >= 128 || in_lo[d]) return PRISM_ERR_BAND;
    in_lo[d] = true;
  }
  if (!pl) return PRISM_OK;
  Plan& P = *pl;
  P.varlen = cfg->seqlens != nullptr;
  for (int x = 0; x < cfg->batch && x < kMaxSeqs; ++x) P.seq_n[x] = P.varlen ? cfg->seqlens[x] : cfg->seqlen;
  P.b = cfg->batch;
  P.hq = cfg->hq;
  P.hkv = cfg->hkv;
  P.n = cfg->seqlen;
  P.nb = (int)nb;
  P.W = (P.nb + 31) / 32;
  P.q_rows = P.b * P.hq;
  P.kv_rows = P.b * P.hkv;
  // pooled row layout: [high only | both | low only], each segment zero-padded
  // to a multiple of 16 columns (one MMA K step), total padded to 64
  std::memset(P.bl.src, 0xff, sizeof(P.bl.src));
  std::memset(P.bl.col, 0xff, sizeof(P.bl.col));
  int c = 0;
  auto segment = [&](bool want_hi, bool want_lo) {
    for (int d = 0; d < 128; ++d)
      if (in_hi[d] == want_hi && in_lo[d] == want_lo) {
        P.bl.col[d] = (uint8_t)c;
        P.bl.src[c++] = (uint8_t)d;
      }
    c = (c + 15) & ~15;
  };
  segment(true, false);
  P.bl.s1 = c;
  segment(true, true);
  P.bl.s2 = c;
  segment(false, true);
  P.bl.s3 = c;
  P.bl.dp = (c + 63) & ~63;
  P.bl.d_hi = cfg->n_hi;
  P.bl.d_lo = cfg->n_lo;
  P.p_eff = cfg->p >= 1.f ? 1.f : cfg->p;
  P.explicit_tau = cfg->tau_mode == PRISM_TAU_EXPLICIT;
  P.tau_hi = cfg->tau_hi;
  P.tau_lo = cfg->tau_lo;
  P.scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / std::sqrt(128.0f);
  P.force = cfg->force_blocks;
  const size_t rows = (size_t)P.q_rows + P.kv_rows;
  size_t off = 0;
  for (int term = 0; term < kTerms; ++term) {
    P.off_pool[term] = off;
    off = align_up(off + rows * P.nb * P.bl.dp * sizeof(__nv_bfloat16), 256);
  }
  P.off_part = off;
  off = align_up(off + rows * P.nb * 4 * sizeof(float), 256);
  P.off_tau = off;
  off = align_up(off + (size_t)P.q_rows * 4 * sizeof(float), 256);
  P.off_scores = off;
  const size_t nch = ((size_t)P.nb + 127) / 128;
  off = align_up(off + (size_t)P.q_rows * (nch * (nch + 1) / 2) * 2 * 128 * 128 * sizeof(float), 256);
  P.off_sync = off;
  // queue heads, per-group counters and ready flags, per (batch, Q head, score chunk) part counters,
  // per (batch, Q head, kToppRows-row segment) mask-rows-written counters
  // and the row maxima of the band scores ([q_rows, nb, 2], combined with atomicMax from 0)
  P.sync_bytes = (2 + 2 * (size_t)P.kv_rows + (size_t)P.q_rows * nch +
                  (size_t)P.q_rows * (((size_t)P.nb + kToppRows - 1) / kToppRows) + (size_t)P.q_rows * P.nb * 2) *
                 sizeof(uint32_t);
  off = align_up(off + P.sync_bytes, 256);
  P.est_bytes = off;  // the estimator uses [0, est_bytes); the mask slot after it is prism_prefill's
  P.off_mask = off;
  off = align_up(off + (size_t)P.q_rows * P.nb * P.W * sizeof(uint32_t), 256);
  P.total = off;
  return PRISM_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------------------
// per-device one-time setup: architecture check and kernel attributes
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_dev_state[kMaxDevices];  // 0 unknown, 1 ready, <0 error code

// Shared memory of the persistent estimator: the stream lane's region (the
// pool ring or the score items' operands; Top-P rows for its warps once the
// stream queue is empty) followed by the Top-P lane's region.
// the widest product layout and the static scratch share one CTA's 227 KB
static_assert(kGemmSmemBytes + sizeof(PoolSmem) + 256 <= 232448, "estimator shared memory over the per-CTA limit");
constexpr size_t kEstMaxDyn = 232448 - sizeof(PoolSmem) - 256;

struct EstLaunch {
  int lane_warps, lane_stride;
  int team_warps, team_stride;
  size_t stream, smem;
  int stages;
};
// Per Top-P warp: a row's logits (replaced by their keys), 256 64-bit bins
// and the mask bit row.
static size_t topp_stride(int nb) {
  const size_t W = ((size_t)nb + 31) / 32, nbp = ((size_t)nb + 7) & ~(size_t)7;
  return align_up(nbp * 4 + kTopPBins * 8 + W * 4, 16);
}
// Fills L; false if the score operands or not even one Top-P warp fit.  The
// Top-P lane takes what the score operands leave; the stream lane's warps use
// the stream region once the stream queue is empty.
bool est_launch_shape(int nb, int dp, EstLaunch& L) {
  const size_t gemm = (size_t)gemm_smem_bytes(dp, score_cols(dp, nb));
  const size_t st = topp_stride(nb);
  L.lane_warps = gemm >= kEstMaxDyn ? 0 : (int)std::min<size_t>(kLaneWarpsMax, (kEstMaxDyn - gemm) / st);
  L.lane_stride = (int)st;
  const size_t lane_bytes = (size_t)L.lane_warps * st;
  L.stream = (kEstMaxDyn - lane_bytes) & ~(size_t)15;  // what the lane leaves: more ring stages
  L.team_warps = (int)std::min<size_t>(kTeamWarpsMax, L.stream / st);
  L.team_stride = (int)st;
  L.smem = L.stream + lane_bytes;
  L.stages = (int)std::min<size_t>(kMaxPoolStages, (L.stream - 1024) / kTileBytes);  // 1 KB-aligned ring
  return gemm <= L.stream && L.stages >= 2 && (L.lane_warps > 0 || L.team_warps > 0);
}

int g_num_sms[kMaxDevices];

int ensure_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev_state[dev] != 0) return g_dev_state[dev] > 0 ? PRISM_OK : g_dev_state[dev];
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return PRISM_ERR_CUDA;
  if (major != 10 || minor != 0) {
    g_dev_state[dev] = PRISM_ERR_DEVICE;
    return PRISM_ERR_DEVICE;
  }
  // The attention kernel re-splits its registers per warpgroup (setmaxnreg);
  // the increase can only be granted if the CTA was launched with at least
  // kMinLaunchRegs per thread, so refuse to run a build that has fewer.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, attn::sparse_attn_kernel) != cudaSuccess) return PRISM_ERR_CUDA;
  if (fa.numRegs < attn::kMinLaunchRegs) {
    g_dev_state[dev] = PRISM_ERR_UNSUPPORTED;
    return PRISM_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(attn::sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)attn::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(estimator_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kEstMaxDyn) != cudaSuccess ||
      cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PRISM_ERR_CUDA;
  g_dev_state[dev] = 1;
  return PRISM_OK;
}

// ---------------------------------------------------------------------------
// TMA descriptors: a [rows, 128] bf16 matrix, boxes of 128 rows x 64 columns,
// 128-byte swizzle (the tcgen05 K-major / MN-major operand layout)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int make_map(CUtensorMap* map, const void* base, size_t rows, int cols = 128, int box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PRISM_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * sizeof(__nv_bfloat16)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PRISM_OK : PRISM_ERR_CUDA;
}

// Q, K or V of `heads` heads of n tokens as a 3-D [heads, n, 128] bf16 view:
// boxes of 64 dims x 128 tokens x 1 head, 128-byte swizzle; tokens past n
// (a short last block) read as zeros.
int make_map_tokens(CUtensorMap* map, const void* base, size_t heads, size_t n) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PRISM_ERR_CUDA;
  cuuint64_t dims[3] = {128, (cuuint64_t)n, (cuuint64_t)heads};
  cuuint64_t strides[2] = {128 * sizeof(__nv_bfloat16), (cuuint64_t)n * 128 * sizeof(__nv_bfloat16)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PRISM_OK : PRISM_ERR_CUDA;
}

// Failure-path self test: thread 0 waits, with the kernels' own bounded-wait
// helpers and a short limit, on a device word nothing writes and on an mbarrier
// phase nothing completes; both give up, record PRISM_ERR_TIMEOUT and the kernel
// returns normally.
__device__ uint32_t g_never_set;

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1u);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    flag_wait_ns(&g_never_set, limit_ns);
    mbar_wait_ns(smem_u32(&bar), 0u, limit_ns);
  }
}

int launched() { return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA; }

// ---------------------------------------------------------------------------
// launch sequences
// ---------------------------------------------------------------------------
// Word offset of the mask-rows-written flags in the estimator's sync region.
size_t ready_offset(const Plan& P) {
  const size_t nch = ((size_t)P.nb + 127) / 128;
  return 2 + 2 * (size_t)P.kv_rows + (size_t)P.q_rows * nch;
}

int run_estimate(const Plan& P, const void* q, const void* k, uint32_t* mask, unsigned char* ws,
                 cudaStream_t st, const prism_debug* dbg) {
  EstParams E;
  E.q = reinterpret_cast<const __nv_bfloat16*>(q);
  E.k = reinterpret_cast<const __nv_bfloat16*>(k);
  for (int term = 0; term < kTerms; ++term)
    E.pool_t[term] = reinterpret_cast<__nv_bfloat16*>(ws + P.off_pool[term]);
  E.part = reinterpret_cast<float*>(ws + P.off_part);
  E.tau = reinterpret_cast<float*>(ws + P.off_tau);
  E.scores = reinterpret_cast<float*>(ws + P.off_scores);
  E.dbg_scores = dbg ? dbg->scores : nullptr;
  E.dbg_weights = dbg ? dbg->weights : nullptr;
  E.dbg_tau = dbg ? dbg->tau : nullptr;
  E.dbg_pooled = dbg ? dbg->pooled : nullptr;
  E.mask = mask;
  E.sync = reinterpret_cast<uint32_t*>(ws + P.off_sync);
  E.ready = E.sync + ready_offset(P);
  E.rmax = E.ready + (size_t)P.q_rows * (((size_t)P.nb + kToppRows - 1) / kToppRows);
  E.hq = P.hq;
  E.hkv = P.hkv;
  E.G = P.hq / P.hkv;
  E.n = P.n;
  E.nb = P.nb;
  E.W = P.W;
  E.q_rows = P.q_rows;
  E.n_groups = P.kv_rows;
  E.pool_item_span = (P.nb + kPoolTilesPerItem - 1) / kPoolTilesPerItem;
  E.pool_items = (E.G + 1) * E.pool_item_span;
  {
    const int nchunk = (P.nb + kScoreRows - 1) / kScoreRows;
    E.score_span = E.score_span_fine = 0;
    for (int c = 0; c < nchunk; ++c) {
      E.score_span += score_parts(c, kScorePartBlocks);
      E.score_span_fine += score_parts(c, kScorePartFine);
    }
    E.score_items = E.G * E.score_span;
    E.score_items_fine = E.G * E.score_span_fine;
    E.topp_rows = nchunk * E.G * kScoreRows;
  }
  EstLaunch L;
  if (!est_launch_shape(P.nb, P.bl.dp, L)) return PRISM_ERR_UNSUPPORTED;
  E.lane_warps = L.lane_warps;
  E.lane_stride = L.lane_stride;
  E.team_warps = L.team_warps;
  E.team_stride = L.team_stride;
  E.lane_off = (int)L.stream;
  E.stream_bytes = (int)L.stream;
  E.ncolw = score_cols(P.bl.dp, P.nb);
  E.pool_stages = L.stages;
  E.p = P.p_eff;
  E.explicit_tau = P.explicit_tau;
  E.tau_hi = P.tau_hi;
  E.tau_lo = P.tau_lo;
  E.force = P.force;
  E.bl = P.bl;
  E.varlen = P.varlen;
  for (int x = 0; x < kMaxSeqs; ++x) E.seq_n[x] = x < P.b ? P.seq_n[x] : 0;
  int dev = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, estimator_kernel, kEstThreads, L.smem) !=
          cudaSuccess)
    return PRISM_ERR_CUDA;
  const long long items = (long long)E.n_groups * (E.pool_items + E.score_items + E.topp_rows / kScoreRows);
  const long long grid = std::min<long long>(items, (long long)g_num_sms[dev] * std::max(per_sm, 1));
  // the score items' operands: pooled rows as bf16 [rows, dp], boxes of 64
  // dims x 128 rows (A, and B when dp <= 128) or x 64 rows (B when dp = 192)
  TermMaps tms;
  const size_t prow = ((size_t)P.q_rows + P.kv_rows) * P.nb;
  for (int term = 0; term < kTerms; ++term)
    if (make_map(&tms.m[term], E.pool_t[term], prow, P.bl.dp, 128) != PRISM_OK ||
        make_map(&tms.m[3 + term], E.pool_t[term], prow, P.bl.dp, 64) != PRISM_OK)
      return PRISM_ERR_CUDA;
  // the pool items' tiles: Q and K as [heads, tokens, 128], boxes of 64 dims x 128 tokens
  if (make_map_tokens(&tms.m[6], q, (size_t)P.q_rows, (size_t)P.n) != PRISM_OK ||
      make_map_tokens(&tms.m[7], k, (size_t)P.kv_rows, (size_t)P.n) != PRISM_OK)
    return PRISM_ERR_CUDA;
  // the queue head and the per-group counters start at zero on every call
  if (cudaMemsetAsync(E.sync, 0, P.sync_bytes, st) != cudaSuccess) return PRISM_ERR_CUDA;
  estimator_kernel<<<(unsigned)grid, kEstThreads, L.smem, st>>>(E, tms);
  return launched();
}

// `ready` (nullable): the estimator's per-segment mask flags; then the kernel
// is launched with programmatic serialization, so it may start on SMs the
// estimator has left while that still finishes other rows.
int run_attention(const Plan& P, const void* q, const void* k, const void* v, const uint32_t* mask,
                  void* o, cudaStream_t st, const uint32_t* ready = nullptr) {
  CUtensorMap mq, mk, mv;
  if (make_map_tokens(&mq, q, (size_t)P.q_rows, (size_t)P.n) != PRISM_OK ||
      make_map_tokens(&mk, k, (size_t)P.kv_rows, (size_t)P.n) != PRISM_OK ||
      make_map_tokens(&mv, v, (size_t)P.kv_rows, (size_t)P.n) != PRISM_OK)
    return PRISM_ERR_CUDA;
  const float scale_log2 = P.scale * 1.4426950408889634f;
  const unsigned grid = attn::grid_size(P.b, P.hq, P.hkv, P.nb);
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(o);
  attn::SeqLens lens;
  lens.varlen = P.varlen;
  for (int x = 0; x < attn::kMaxSeqs; ++x) lens.n[x] = x < P.b ? P.seq_n[x] : 0;
  if (!ready) {
    attn::sparse_attn_kernel<<<grid, attn::kThreads, attn::kSmemBytes, st>>>(
        mq, mk, mv, mask, out, P.b, P.hq, P.hkv, P.n, P.nb, scale_log2, nullptr, kToppRows, lens);
    return launched();
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(attn::kThreads);
  lc.dynamicSmemBytes = attn::kSmemBytes;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, attn::sparse_attn_kernel, mq, mk, mv, mask, out, P.b, P.hq, P.hkv, P.n, P.nb,
                         scale_log2, ready, kToppRows, lens) != cudaSuccess)
    return PRISM_ERR_CUDA;
  return launched();
}

// ---------------------------------------------------------------------------
// Built-in scratch for prism_estimate_noalloc.  A file-scope device array of
// fixed size: every GPU that loads this library holds it until the process
// exits.  Host code may not use the symbol itself as a device address (in host
// code it names a host-side stand-in); the device address is looked up once
// per device with cudaGetSymbolAddress while that device is current.
// ---------------------------------------------------------------------------
constexpr size_t kStaticScratchBytes = 32u << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];

int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return PRISM_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PRISM_OK;
}

}  // namespace

extern "C" {

int prism_version(void) { return kVersion; }

const char* prism_status_str(int s) {
  switch (s) {
    case PRISM_OK: return "ok";
    case PRISM_ERR_NULL: return "a required pointer is NULL";
    case PRISM_ERR_SHAPE: return "invalid shape (sizes, hq % hkv, or size overflow)";
    case PRISM_ERR_ALIGN: return "a pointer is not suitably aligned";
    case PRISM_ERR_BAND: return "invalid band index set";
    case PRISM_ERR_P: return "p must be > 0";
    case PRISM_ERR_UNSUPPORTED: return "unsupported configuration (head_dim/block must be 128, causal must be 1)";
    case PRISM_ERR_WORKSPACE: return "workspace missing or too small";
    case PRISM_ERR_CUDA: return "a CUDA runtime call failed";
    case PRISM_ERR_DEVICE: return "the current device is not sm_100 (B200-class)";
    case PRISM_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case PRISM_ERR_TAU: return "explicit temperatures must be finite and > 0";
    case PRISM_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than the 32 MiB built into prism_estimate_noalloc";
    default: return "unknown status";
  }
}

int prism_workspace_size(const prism_config* cfg, size_t* bytes) {
  if (!bytes) return PRISM_ERR_NULL;
  Plan P;
  const int s = validate(cfg, &P);
  if (s != PRISM_OK) return s;
  *bytes = P.total;
  return PRISM_OK;
}

int prism_estimate(const prism_config* cfg, const void* q, const void* k, uint32_t* mask,
                   void* workspace, size_t workspace_bytes, prism_stream_t stream, const prism_debug* dbg) {
  Plan P;
  int s = validate(cfg, &P);
  if (s != PRISM_OK) return s;
  if (!q || !k || !mask) return PRISM_ERR_NULL;
  if (!workspace || workspace_bytes < P.total) return PRISM_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(mask, 4) || !aligned(workspace, 256))
    return PRISM_ERR_ALIGN;
  if (dbg && ((dbg->scores && !aligned(dbg->scores, 16)) || (dbg->weights && !aligned(dbg->weights, 16)) ||
              (dbg->tau && !aligned(dbg->tau, 4)) || (dbg->pooled && !aligned(dbg->pooled, 16))))
    return PRISM_ERR_ALIGN;
  if ((s = ensure_device()) != PRISM_OK) return s;
  return run_estimate(P, q, k, mask, static_cast<unsigned char*>(workspace),
                      reinterpret_cast<cudaStream_t>(stream), dbg);
}

int prism_sparse_attn(const prism_config* cfg, const void* q, const void* k, const void* v,
                      const uint32_t* mask, void* o, prism_stream_t stream) {
  Plan P;
  int s = validate(cfg, &P);
  if (s != PRISM_OK) return s;
  if (!q || !k || !v || !mask || !o) return PRISM_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(mask, 4) || !aligned(o, 16))
    return PRISM_ERR_ALIGN;
  if ((s = ensure_device()) != PRISM_OK) return s;
  return run_attention(P, q, k, v, mask, o, reinterpret_cast<cudaStream_t>(stream));
}

int prism_prefill(const prism_config* cfg, const void* q, const void* k, const void* v,
                  uint32_t* mask_out, void* o, void* workspace, size_t workspace_bytes,
                  prism_stream_t stream) {
  Plan P;
  int s = validate(cfg, &P);
  if (s != PRISM_OK) return s;
  if (!q || !k || !v || !o) return PRISM_ERR_NULL;
  if (!workspace || workspace_bytes < P.total) return PRISM_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(workspace, 256) || (mask_out && !aligned(mask_out, 4)))
    return PRISM_ERR_ALIGN;
  if ((s = ensure_device()) != PRISM_OK) return s;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  uint32_t* mask = mask_out ? mask_out : reinterpret_cast<uint32_t*>(ws + P.off_mask);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((s = run_estimate(P, q, k, mask, ws, st, nullptr)) != PRISM_OK) return s;
  // the attention starts on query blocks whose masks are final while the
  // estimator finishes the others
  const uint32_t* ready = reinterpret_cast<const uint32_t*>(ws + P.off_sync) + ready_offset(P);
  return run_attention(P, q, k, v, mask, o, st, ready);
}

// Same estimator as prism_estimate, with the library's built-in scratch array in
// place of a caller-provided workspace.  The work-queue counters, the only
// words that must start at zero, are cleared on the stream at the start of
// every call (as for prism_estimate); every other word a kernel reads is
// written earlier in the same call.
int prism_estimate_noalloc(const prism_config* cfg, const void* q, const void* k, uint32_t* mask,
                           prism_stream_t stream) {
  Plan P;
  int s = validate(cfg, &P);
  if (s != PRISM_OK) return s;
  if (!q || !k || !mask) return PRISM_ERR_NULL;
  if (P.est_bytes > kStaticScratchBytes) return PRISM_ERR_SCRATCH_LIMIT;  // the estimator's part of the workspace
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(mask, 4)) return PRISM_ERR_ALIGN;
  if ((s = ensure_device()) != PRISM_OK) return s;
  void* scratch = nullptr;
  if ((s = static_scratch(&scratch)) != PRISM_OK) return s;
  return run_estimate(P, q, k, mask, static_cast<unsigned char*>(scratch),
                      reinterpret_cast<cudaStream_t>(stream), nullptr);
}

size_t prism_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

int prism_selftest_wait_timeout(prism_stream_t stream, unsigned timeout_us) {
  if (timeout_us == 0 || timeout_us > 2000000u) return PRISM_ERR_SHAPE;
  int s = ensure_device();
  if (s != PRISM_OK) return s;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)timeout_us * 1000ull);
  return launched();
}

int prism_get_last_device_error(prism_stream_t stream) {
  if (ensure_device() != PRISM_OK) return PRISM_ERR_DEVICE;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return PRISM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, prism::g_device_error, sizeof(int)) != cudaSuccess) return PRISM_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(prism::g_device_error, &zero, sizeof(int)) != cudaSuccess) return PRISM_ERR_CUDA;
  return v;
}

}  // extern "C"
