// Prism block-importance estimator, steps (1)-(7) of the method paragraph of
// the paper.rainbus.top review of "Prism: Spectral-Aware Block-Sparse
// Attention": band slicing, mean pooling per block of B = 128 tokens, RMS of
// each pooled band, temperatures tau_z, dual-band pooled softmax, Top-P per
// query-block row and band, union of the two masks.
//
// One persistent kernel, one CTA per SM.  Its warps form two lanes with a
// device queue each, working at the same time:
//
// * the stream lane takes pool and score items, per KV group g (the Q heads
//   that share one KV head) in the order
//     pool(0), pool(1), pool(2), score(0), pool(3), score(1), ..., score(n-2), score(n-1)
//   pool items (HBM-bound) stream 128x128 bf16 tiles of Q and K once (TMA into
//   a ring of shared-memory stages, several tiles in flight); the block sums
//   are products on the tensor cores (the tile, read transposed, times a
//   column of ones: D[dim] += sum over the block's tokens), so the CUDA cores
//   only turn the sums into the fp32 block means (steps 1-2) and per-block
//   energy partials (step 3); the CTA that finishes the last pool item of a
//   group computes the group's temperatures (steps 3-4) and publishes "group
//   ready".  score items wait for their group and compute both bands' pooled
//   logits on the tensor cores (step 5; tcgen05 on a three-term bf16 split,
//   fp32 accuracy), in row chunks of 128 query blocks and parts of at most 512
//   key blocks, keeping the row maxima;
// * the Top-P lane takes Top-P items (16 query-block rows of one head) once
//   their score chunk is complete: softmax + Top-P + union per row (steps
//   5-7), on the CUDA cores, beside the stream lane's pooling.  When the
//   stream queue is empty its warps take Top-P items too.
//
// An item only ever waits for items that running lanes hold and that never
// wait on the other lane, so the schedule cannot deadlock; every wait is
// bounded all the same.
//
// Band slicing is folded into the pooled layout: the pool items write each
// pooled row as [high-only | both | low-only] dims, every segment padded with
// zeros to a multiple of 16 (one MMA K step), so each band is a contiguous,
// aligned column range: high = [0, s2), low = [s1, s3).  Dims in neither band
// are not stored.  The values are stored as three bf16 terms h + m + l (each
// the rounding error of the ones before, 24 significant bits in all); the
// products sum the six cross terms of order >= 2^-24 (hh, hm, mh, hl, lh,
// mm), which matches an fp32 dot product.
#pragma once
#include "ptx.cuh"

namespace prism {

struct BandLayout {
  uint8_t src[192];  // pooled column c holds original dim src[c]; 255 = zero padding
  uint8_t col[128];  // inverse: the pooled column of dim d; 255 = in neither band
  int s1, s2, s3;    // 16-aligned segment boundaries (see above)
  int dp;            // stored row length: a multiple of 64 (64, 128 or 192)
  int d_hi, d_lo;    // band sizes
};

constexpr int kEstThreads = 512;      // 16 warps, one CTA per SM
constexpr int kPoolTilesPerItem = 32;  // 32 x 32 KB of Q or K per pool item (its block sums fill tensor memory)
constexpr uint32_t kTileBytes = 128 * 128 * 2;
constexpr int kMaxPoolStages = 6;      // TMA ring depth (32 KB stages)
constexpr int kPoolN = 16;             // N of a pooling product: block b sums into TMEM columns [16 b, 16 b + 16)
constexpr int kScoreRows = 128;       // query blocks (of one head) per score item = MMA M
constexpr int kScorePartBlocks = 512;  // key blocks per score item: longer rows are split into parts
constexpr int kScorePartFine = 128;    // the same for the last groups' items (spread over every SM)
constexpr int kToppRows = 16;         // mask rows per ready counter (what the attention of a prefill waits on)
constexpr uint32_t kOpChunk = 128 * 64 * 2;  // one 64-dim x 128-row bf16 operand chunk (SW128)
constexpr int kTerms = 3;             // bf16 terms per pooled value
// product operands: A (3 terms x dp/64 chunks of 128 rows) once, B one term at
// a time in kBSlots slots (dp/64 chunks of N rows)
constexpr int kBSlots = 2;
// N, the key blocks of one product: 128, or 64 when the pooled rows are 192
// wide (the operands must fit) or the rows are long (from nb = 2048 on, the
// Top-P warps' key buffers need the shared memory; halving the B slots leaves
// room for more of them)
constexpr int kWideRowsNb = 2048;
__host__ __device__ constexpr int score_cols(int dp, int nb) { return dp <= 128 && nb < kWideRowsNb ? 128 : 64; }
__host__ __device__ constexpr int gemm_smem_bytes(int dp, int ncolw) {
  return kTerms * (dp / 64) * (int)kOpChunk + kBSlots * (dp / 64) * ncolw * 128 + 1024;
}
constexpr int kGemmSmemBytes = gemm_smem_bytes(192, 64);  // the largest layout: 144 + 2 x 24 KB + alignment

// The CTA's warps form two lanes that take items from two queues at once:
// the stream lane (warps 0, 1, 4-7) runs pool and score items, the Top-P
// lane (warps 2, 3, 8-15) runs Top-P items, so the Top-P work of earlier
// groups proceeds on the CUDA cores while the same SM streams Q and K.  Once
// the stream queue is empty the stream lane's warps take Top-P items too.
// Each lane synchronises on its own named barrier (1 is the pool read-out
// warps' own).
constexpr int kStreamThreads = 192;  // warps 0, 1, 4-7
constexpr int kLaneThreads = 320;    // warps 2, 3, 8-15
constexpr int kLaneWarpsMax = kLaneThreads / 32;
constexpr int kTeamWarpsMax = kStreamThreads / 32;
enum : int { kBarStream = 2, kBarLane = 3 };
__device__ __forceinline__ bool in_stream_lane(int warp) { return warp < 2 || (warp >= 4 && warp < 8); }
__device__ __forceinline__ int stream_tid(int t) { return t < 64 ? t : t - 64; }            // 0 .. 191
__device__ __forceinline__ int stream_warp(int warp) { return warp < 2 ? warp : warp - 2; }  // 0 .. 5
__device__ __forceinline__ int lane_warp(int warp) { return warp < 4 ? warp - 2 : warp - 6; }    // 0 .. 9
constexpr int kMaxGroupHeads = 64;    // Q heads per KV head supported by the tau step
constexpr int kMaxSeqs = 256;         // sequences of a batch with per-sequence lengths
constexpr int kTauBatch = 5;          // head rows whose energy partials the tau step sums at once
constexpr float kLog2e = 1.4426950408889634f;

// TMA descriptors of the three pooled bf16 terms [rows, dp]: boxes of 64 dims
// x 128 rows (m[0..2]) and 64 dims x 64 rows (m[3..5]); Q and K as
// [rows x tokens, 128] with boxes of 64 dims x 128 tokens (m[6], m[7])
struct TermMaps {
  CUtensorMap m[8];
};

struct EstParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  __nv_bfloat16* pool_t[kTerms];  // [q_rows + kv_rows, nb, dp] band-segment means, bf16 terms h, m, l
  float* part;    // [q_rows + kv_rows, nb, 4] sum(mean^2): hi, lo, all
  float* tau;     // [q_rows, 4]: tau_hi, tau_lo, 1/(tau_hi sqrt d_hi), 1/(tau_lo sqrt d_lo)
  float* scores;      // scaled band logits in 128 x 128 tiles: [q_rows][tile (cr, cc), cc <= cr][band][128][128]
  float* dbg_scores;   // optional copy in packed lower-triangular rows [q_rows, 2, nb(nb+1)/2]
  float* dbg_weights;  // optional: the Top-P's softmax weights e_j, same packing
  uint32_t* mask;
  float* dbg_tau;
  float* dbg_pooled;   // optional: block means [q_rows + kv_rows, nb, 128], all dims
  uint32_t* ready;  // [q_rows, ceil(nb / kToppRows)] mask rows written, per kToppRows-row segment
  uint32_t* rmax;   // [q_rows, nb, 2] the scaled band logits' row maxima over j <= i, order-preserving
                    // encoding (max_enc), combined over the score parts with atomicMax from 0
  uint32_t* sync;  // [0] stream queue head, [1] Top-P queue head, [2 + g] pool items done,
                   // [2 + n_groups + g] group ready,
                   // [2 + 2 n_groups + bh * nchunk + c] parts of score chunk c of (batch, Q head) bh written
  int hq, hkv, G, n, nb, W, q_rows, n_groups;  // n: tokens per head (the last block may be short)
  int pool_items;      // per group
  int score_items;     // per group (kScorePartBlocks parts)
  int score_span;      // score items per head: (row chunk, key-block part) pairs
  int score_items_fine, score_span_fine;  // the same with kScorePartFine parts (score_fine groups)
  int topp_rows;       // Top-P queue entries per group: nchunk x G x kScoreRows (rows past nb skipped)
  int pool_item_span;  // pool items per head row
  // Top-P warps of each lane: how many take rows and bytes of shared memory
  // each (topp_scratch)
  int lane_warps, lane_stride;
  int team_warps, team_stride;
  int lane_off;      // byte offset of the Top-P lane's shared memory
  int stream_bytes;  // dynamic shared memory of the stream lane (pool ring, score operands)
  int ncolw;         // key blocks per score product (score_cols)
  int pool_stages;   // TMA ring depth (<= kMaxPoolStages)
  float p;
  int explicit_tau;
  float tau_hi, tau_lo;
  int force;  // optional forced blocks: 1 = key block 0, 2 = the diagonal
  BandLayout bl;
  int varlen;              // 1: batch element b holds seq_n[b] <= n tokens (the rest is padding)
  int seq_n[kMaxSeqs];
};

// Tokens and blocks of batch element bi (the layout keeps n tokens, nb blocks per head).
__device__ __forceinline__ int seq_tokens(const EstParams& P, int bi) { return P.varlen ? P.seq_n[bi] : P.n; }
__device__ __forceinline__ int seq_blocks(const EstParams& P, int bi) { return (seq_tokens(P, bi) + 127) >> 7; }

// The 128 x 128 score tile (row chunk cr, column chunk cc <= cr) of one
// (batch, Q head): rows = query blocks 128 cr + r, columns = key blocks 128 cc + c.
__device__ __forceinline__ float* score_tile(const EstParams& P, int bh, int cr, int cc) {
  const int nch = (P.nb + 127) / 128;
  const size_t pairs = (size_t)nch * (nch + 1) / 2;
  return P.scores + ((size_t)bh * pairs + (size_t)cr * (cr + 1) / 2 + cc) * (2 * 128 * 128);
}

// Score items: row chunk c (kScoreRows query blocks) against the key blocks
// j <= its last row, in parts of `pb` key blocks: kScorePartBlocks, or
// kScorePartFine for the groups scored last, whose items then spread over
// every SM instead of ending the launch on a few long ones.
__host__ __device__ __forceinline__ int score_parts(int chunk, int pb) {
  return (chunk * kScoreRows + kScoreRows + pb - 1) / pb;
}
constexpr int kScoreLag = 2;  // scoring of group g follows pooling of group g + kScoreLag
__device__ __forceinline__ bool score_fine(const EstParams& P, int g) {
  return g >= P.n_groups - min(kScoreLag, P.n_groups);
}
__device__ __forceinline__ int score_part_blocks(const EstParams& P, int g) {
  return score_fine(P, g) ? kScorePartFine : kScorePartBlocks;
}
// Item z of one head (longest rows first) -> (row chunk, part).
__device__ __forceinline__ void score_part_of(const EstParams& P, int z, int pb, int& chunk, int& part) {
  const int nchunk = (P.nb + kScoreRows - 1) / kScoreRows;
  for (chunk = nchunk - 1; chunk > 0; --chunk) {
    const int np = score_parts(chunk, pb);
    if (z < np) break;
    z -= np;
  }
  part = z;
}

// ---------------------------------------------------------------------------
// warp / ordering helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_release_gpu_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// An order-preserving map of floats to unsigned words (larger float, larger
// word; 0 lies below every float), so maxima combine with integer atomicMax.
__device__ __forceinline__ uint32_t max_enc(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float max_dec(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// ---------------------------------------------------------------------------
// static shared memory of the kernel
// ---------------------------------------------------------------------------
struct PoolSmem {
  // all-ones bf16 B operand of the pooling products: 16 rows x 128 bytes in
  // the 128-byte-swizzled K-major layout (every element is one, so the
  // swizzle does not matter)
  __align__(1024) uint32_t ones[16 * 32];
  union {                                   // pool and score items never overlap in a CTA
    float wred[16][16];                     // temperatures: per-warp partial sums (kTauBatch slots x 3)
    float bpart[kPoolTilesPerItem][4][3];  // pool item: per block and read-out warp: hi, lo, all
  };
  float sums[kMaxGroupHeads + 1][3];
  uint64_t bars[kMaxPoolStages];       // pool ring: stage loaded
  uint64_t bars_free[kMaxPoolStages];  // pool ring: stage multiplied
  uint64_t bar_pool;                   // pool item: every block sum is in tensor memory
  uint64_t bar_pool_half;              // pool item: the sums of its first 16 blocks are done
  uint64_t bar_a, bar_b[kBSlots], bar_free[kBSlots], bar_mma[2], bar_acc[2];  // score item: operands, slots,
                                                                            // products, accumulators read
  uint32_t tmem;
  int flag;
};

// Transpose-reduction across a warp of N (8, 16 or 32) values per lane: lane
// L ends with the warp's sum of value L % N, in a fixed order (N - 1
// shuffles, plus log2(32 / N)).
template <int N>
__device__ __forceinline__ float warp_reduce_n(float (&v)[N], int lane) {
#pragma unroll
  for (int o = N / 2; o > 0; o >>= 1) {
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const bool up = (lane & o) != 0;
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
#pragma unroll
  for (int o = N; o < 32; o <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
  return v[0];
}

// steps (3b)-(4): RMS of every pooled band of the group's heads over all
// blocks and the temperatures of its Q heads (reading R1 of the pages: the
// band's pooled Q x K energy relative to the full spectrum's).
__device__ __forceinline__ void group_temperatures(const EstParams& P, int g, PoolSmem& sm) {
  const int t = stream_tid(threadIdx.x), warp = t >> 5, lane = t & 31;  // the stream lane
  const int bi = g / P.hkv, kv = g - bi * P.hkv;
  const int nbb = seq_blocks(P, bi);
  // slots 0..G-1: Q heads, G: the KV head; kTauBatch slots at a time, so the
  // loads of all of them are in flight together (the partials come from L2)
  for (int s0 = 0; s0 <= P.G; s0 += kTauBatch) {
    const int ns = min(kTauBatch, P.G + 1 - s0);
    float s[kTauBatch][3];
#pragma unroll
    for (int q = 0; q < kTauBatch; ++q) s[q][0] = s[q][1] = s[q][2] = 0.f;
#pragma unroll 2
    for (int i = t; i < nbb; i += kStreamThreads) {
      float4 v[kTauBatch];
#pragma unroll
      for (int q = 0; q < kTauBatch; ++q) {
        const int slot = s0 + q;
        const int hr = slot < P.G ? bi * P.hq + kv * P.G + slot : P.q_rows + g;
        v[q] = q < ns ? __ldcg(reinterpret_cast<const float4*>(P.part + ((size_t)hr * P.nb + i) * 4))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < kTauBatch; ++q) {
        s[q][0] += v[q].x;
        s[q][1] += v[q].y;
        s[q][2] += v[q].z;
      }
    }
#pragma unroll
    for (int q = 0; q < kTauBatch; ++q)
#pragma unroll
      for (int e = 0; e < 3; ++e) {
        const float r = warp_sum(s[q][e]);
        if (lane == 0) sm.wred[warp][3 * q + e] = r;
      }
    named_barrier(kBarStream, kStreamThreads);
    if (t < 3 * ns) {
      float a = 0.f;
      for (int w = 0; w < kStreamThreads / 32; ++w) a += sm.wred[w][t];
      sm.sums[s0 + t / 3][t % 3] = a;
    }
    named_barrier(kBarStream, kStreamThreads);
  }
  if (t < P.G) {
    const int row = bi * P.hq + kv * P.G + t;
    float th, tl;
    if (P.explicit_tau) {
      th = P.tau_hi;
      tl = P.tau_lo;
    } else {
      const float n = (float)nbb;
      const float* sq = sm.sums[t];
      const float* sk = sm.sums[P.G];
      const float rq_hi = sqrtf(sq[0] / (n * P.bl.d_hi)), rq_lo = sqrtf(sq[1] / (n * P.bl.d_lo));
      const float rq_f = sqrtf(sq[2] / (n * 128.f));
      const float rk_hi = sqrtf(sk[0] / (n * P.bl.d_hi)), rk_lo = sqrtf(sk[1] / (n * P.bl.d_lo));
      const float rk_f = sqrtf(sk[2] / (n * 128.f));
      const float den = rq_f * rk_f;
      const float nh = rq_hi * rk_hi, nl = rq_lo * rk_lo;
      th = (den > 0.f && nh > 0.f) ? nh / den : 1.f;
      tl = (den > 0.f && nl > 0.f) ? nl / den : 1.f;
    }
    P.tau[row * 4 + 0] = th;
    P.tau[row * 4 + 1] = tl;
    P.tau[row * 4 + 2] = 1.0f / (th * sqrtf((float)P.bl.d_hi));
    P.tau[row * 4 + 3] = 1.0f / (tl * sqrtf((float)P.bl.d_lo));
    if (P.dbg_tau) {
      P.dbg_tau[row * 2 + 0] = th;
      P.dbg_tau[row * 2 + 1] = tl;
    }
  }
}

// One pool item: kPoolTilesPerItem consecutive blocks of one head row of the
// group (its Q heads, then its KV head).  Warp roles: thread 0 streams the
// tiles into the ring (TMA, two 64-dim boxes per tile, 128-byte swizzle);
// thread 32 issues the block sums as tensor-core products: the tile is the A
// operand read dim-major (M = 128 dims, K = 16 tokens a step), the all-ones
// matrix the B operand (N = 16), block b accumulating into TMEM columns
// [16 b, 16 b + 16), each stage released when its products are done; warps
// 4-7 (thread = dim) read the sums, write the means in the band-segment layout
// as three bf16 terms and the per-block energy partials.
struct PoolState {  // per-role counters of ring stages and items, carried across items
  uint32_t prod, cons, done, half;
  int pre;  // producer: tiles of the next pool item already streamed into the ring
};

// Stream queue order, with PI / SI pool / score items per group g of n and a
// lag of two groups (the last two groups' score items, SF each, have finer
// parts):
//   pool(0) pool(1) | pool(2) score(0) | pool(3) score(1) | ... | pool(n-1) score(n-3) | score(n-2) score(n-1)
// so scoring of group g overlaps pooling of group g + 2, by which time the
// pooling of g has ended and the score items do not wait.  Returns the item
// kind (0 pool, 1 score, -1 past the end) and sets (g, y), y the index within
// the group's items of that kind.
enum : int { kItemPool = 0, kItemScore = 1, kItemNone = -1 };
__device__ __forceinline__ int decode_stream(const EstParams& P, int x, int& g, int& y) {
  const int n = P.n_groups, PI = P.pool_items;
  const int lag = min(kScoreLag, n), M = n - lag;
  if (x < lag * PI) {
    g = x / PI;
    y = x - g * PI;
    return kItemPool;
  }
  x -= lag * PI;
  const int L = PI + P.score_items;
  if (x < M * L) {  // pairs p = 0 .. M-1: pool(p + lag) score(p)
    const int p = x / L, rem = x - p * L;
    if (rem < PI) {
      g = p + lag;
      y = rem;
      return kItemPool;
    }
    g = p;
    y = rem - PI;
    return kItemScore;
  }
  x -= M * L;
  const int SF = P.score_items_fine;  // the last lag groups: finer parts
  if (x < lag * SF) {
    const int q = x / SF;
    g = M + q;
    y = x - q * SF;
    return kItemScore;
  }
  return kItemNone;
}
// The tiles of pool item (g, y): tensor map ([heads, n, 128]), head, first
// token, tile count.
struct PoolCoords {
  const CUtensorMap* map;
  int head, tok0, nt;
};
__device__ __forceinline__ PoolCoords pool_coords(const EstParams& P, const CUtensorMap* tm, int g, int y) {
  const int slot = y / P.pool_item_span;
  const int blk0 = (y - slot * P.pool_item_span) * kPoolTilesPerItem;
  const int bi = g / P.hkv, kv = g - bi * P.hkv;
  const bool is_q = slot < P.G;
  PoolCoords c;
  c.map = &tm[is_q ? 6 : 7];
  c.head = is_q ? bi * P.hq + kv * P.G + slot : g;
  c.tok0 = blk0 * 128;
  c.nt = max(min(blk0 + kPoolTilesPerItem, seq_blocks(P, bi)) - blk0, 0);  // 0: past the sequence
  return c;
}

// Producer: streams tiles [t0, t1) of an item into the ring.
__device__ __forceinline__ void pool_stream(const PoolCoords& c, int t0, int t1, PoolSmem& sm, uint32_t ring0,
                                            int stages, PoolState& st) {
  for (int tt = t0; tt < t1; ++tt, ++st.prod) {
    const uint32_t s = st.prod % (uint32_t)stages;
    if (st.prod >= (uint32_t)stages)  // the stage's previous tile has been multiplied
      mbar_wait(smem_u32(&sm.bars_free[s]), (st.prod / (uint32_t)stages - 1u) & 1u);
    const uint32_t dst = ring0 + s * kTileBytes, bar = smem_u32(&sm.bars[s]);
    mbar_arrive_expect_tx(bar, kTileBytes);
    // read once: first out of L2, so the score tiles the Top-P rows read
    // back stay resident
    const uint64_t pol = l2_policy_evict_first();
    tma_load_3d_hint(dst, c.map, 0, c.tok0 + tt * 128, c.head, bar, pol);
    tma_load_3d_hint(dst + kTileBytes / 2, c.map, 64, c.tok0 + tt * 128, c.head, bar, pol);
  }
}

//
// When the CTA's next queue item (x_next, already claimed) is a pool item too,
// the producer goes on to stream its first tiles (up to the ring depth) as soon
// as this item's products release the stages, so the next item's loads are in
// flight while this one is read out and published.
__device__ __forceinline__ void pool_item(const EstParams& P, const CUtensorMap* tm, int g, int y, int x_next,
                                          PoolSmem& sm, unsigned char* ring, int stages, PoolState& st) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int slot = y / P.pool_item_span;
  const int blk0 = (y - slot * P.pool_item_span) * kPoolTilesPerItem;
  const int bi = g / P.hkv, kv = g - bi * P.hkv;
  const int nbb = seq_blocks(P, bi);
  const int nt = max(min(blk0 + kPoolTilesPerItem, nbb) - blk0, 0);  // 0: past the sequence, only counted
  const bool is_q = slot < P.G;
  const int hr = is_q ? bi * P.hq + kv * P.G + slot : P.q_rows + g;
  const uint32_t ring0 = (smem_u32(ring) + 1023u) & ~1023u;
  if (nt == 0) {
    // nothing to pool (no tile of it was prefetched either)
  } else if (t == 0) {  // producer
    fence_proxy_async_smem();  // generic writes of the last item before the async ones
    pool_stream(pool_coords(P, tm, g, y), st.pre, nt, sm, ring0, stages, st);
    st.pre = 0;
    int gn, yn;
    if (decode_stream(P, x_next, gn, yn) == kItemPool) {
      const PoolCoords cn = pool_coords(P, tm, gn, yn);
      st.pre = min(cn.nt, stages);
      pool_stream(cn, 0, st.pre, sm, ring0, stages, st);
    }
  } else if (t == 32) {  // product issuer
    const uint32_t idesc = idesc_bf16_f32(128, kPoolN, 1, 0);
    const uint64_t bdesc = smem_desc_sw128(smem_u32(sm.ones), 16, 1024);
    for (int tt = 0; tt < nt; ++tt, ++st.cons) {
      const uint32_t s = st.cons % (uint32_t)stages;
      mbar_wait(smem_u32(&sm.bars[s]), (st.cons / (uint32_t)stages) & 1u);
      tc_fence_after();
      // A: 128 tokens x 128 dims, dims contiguous: MN-major, the two 64-dim
      // halves 16 KB apart, 8-token groups 1 KB apart, 16 tokens = 2 KB a step
      const uint64_t adesc = smem_desc_sw128(ring0 + s * kTileBytes, kTileBytes / 2, 1024);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16_ss(sm.tmem + (uint32_t)(tt * kPoolN), adesc + (uint64_t)((k * 2048) >> 4), bdesc, idesc,
                    k > 0 ? 1u : 0u);
      mma_commit(smem_u32(&sm.bars_free[s]));
      if (tt == 15 && nt > 16) mma_commit(smem_u32(&sm.bar_pool_half));  // the read-out can start
    }
    mma_commit(smem_u32(&sm.bar_pool));
  } else if (warp >= 4 && warp < 8) {  // read-out: thread = dim
    const int q4 = warp & 3, d = q4 * 32 + lane;
    const int c = P.bl.col[d];
    const bool ih = c < P.bl.s2, il = c >= P.bl.s1 && c < P.bl.s3;  // c = 255: neither
    const size_t o0 = ((size_t)hr * P.nb + blk0) * P.bl.dp;
    // the item's blocks in groups of 16 (one tensor-memory read of 16 columns each)
    for (int b0 = 0; b0 < nt; b0 += 16) {
      // the first 16 blocks are read while the products of the others run
      if (b0 == 0 && nt > 16) {
        mbar_wait(smem_u32(&sm.bar_pool_half), st.half & 1u);
        ++st.half;
      } else {
        mbar_wait(smem_u32(&sm.bar_pool), st.done & 1u);
        ++st.done;
      }
      tc_fence_after();
      uint32_t v[16];
#pragma unroll
      for (int b = 0; b < 16; ++b)
        v[b] = tmem_ld1(sm.tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)((b0 + b) * kPoolN));
      tmem_wait_ld_dep16(v);
      float ehl[32], ea[16];
#pragma unroll
      for (int b = 0; b < 16; ++b) {
        // block mean: the last block may hold fewer than 128 tokens (zeros past the end)
        const int blk = blk0 + b0 + b;
        const float inv = blk == nbb - 1 ? 1.0f / (float)(seq_tokens(P, bi) - 128 * (nbb - 1)) : (1.0f / 128.0f);
        const float m = __uint_as_float(v[b]) * inv;
        const bool ok = b0 + b < nt;
        if (ok && P.dbg_pooled) P.dbg_pooled[((size_t)hr * P.nb + blk) * 128 + d] = m;
        if (ok && c != 255) {
          const __nv_bfloat16 th = __float2bfloat16_rn(m);
          const float r1 = m - __bfloat162float(th);
          const __nv_bfloat16 tmid = __float2bfloat16_rn(r1);
          const __nv_bfloat16 tl = __float2bfloat16_rn(r1 - __bfloat162float(tmid));
          const size_t o = o0 + (size_t)(b0 + b) * P.bl.dp + c;
          P.pool_t[0][o] = th;
          P.pool_t[1][o] = tmid;
          P.pool_t[2][o] = tl;
        }
        const float x = ok ? m * m : 0.f;
        ehl[b] = ih ? x : 0.f;
        ehl[16 + b] = il ? x : 0.f;
        ea[b] = x;
      }
      // energy partials: lane L holds the warp's hi (L < 16) or lo sum of
      // block b0 + L % 16, and its all-dims sum
      const float rhl = warp_reduce_n<32>(ehl, lane);
      const float ra = warp_reduce_n<16>(ea, lane);
      sm.bpart[b0 + (lane & 15)][q4][lane >> 4] = rhl;
      if (lane < 16) sm.bpart[b0 + lane][q4][2] = ra;
    }
    tc_fence_before();
    // zero padding columns of the segment layout
    for (int cc = d; cc < P.bl.dp; cc += 128)
      if (P.bl.src[cc] == 255)
        for (int b = 0; b < nt; ++b) {
          const size_t o = o0 + (size_t)b * P.bl.dp + cc;
          P.pool_t[0][o] = __float2bfloat16_rn(0.f);
          P.pool_t[1][o] = __float2bfloat16_rn(0.f);
          P.pool_t[2][o] = __float2bfloat16_rn(0.f);
        }
    // the four warps' partials of each block, added in a fixed order
    named_barrier(1, 128);
    for (int q = d; q < nt * 3; q += 128) {
      const int b = q / 3, e = q - 3 * b;
      P.part[((size_t)hr * P.nb + blk0 + b) * 4 + e] =
          (sm.bpart[b][0][e] + sm.bpart[b][1][e]) + (sm.bpart[b][2][e] + sm.bpart[b][3][e]);
    }
  }
  // publish: count the item; the CTA that completes the group computes tau
  named_barrier(kBarStream, kStreamThreads);
  if (t == 0) {
    __threadfence();
    const uint32_t done = atomicAdd(&P.sync[2 + g], 1u);
    sm.flag = (done == (uint32_t)P.pool_items - 1u);
    if (sm.flag) __threadfence();
  }
  named_barrier(kBarStream, kStreamThreads);
  if (sm.flag) {
    group_temperatures(P, g, sm);
    named_barrier(kBarStream, kStreamThreads);
    if (t == 0) {
      __threadfence();
      st_release_gpu(&P.sync[2 + P.n_groups + g], 1u);
    }
  }
}

// ---------------------------------------------------------------------------
// step (6): exact Top-P of one band row
// ---------------------------------------------------------------------------
// Shared-memory scratch of one Top-P warp.
struct ToppScratch {
  uint32_t* d;            // [n] the row's rank keys d_j (below)
  unsigned long long* h;  // [256] bin masses; then the member records of the exact step
};

constexpr int kTopPBins = 256;
constexpr float kFix = 2147483648.0f;  // 2^31: e_j in [0, 2) -> 32-bit fixed point

// e_j (in (0, 2)) -> rank key d_j = 0x40000000 - bits(e_j): an exact,
// order-reversing map (smaller key = larger e_j; equal keys = equal e_j).
__device__ __forceinline__ uint32_t rank_key(float e) { return 0x40000000u - __float_as_uint(e); }
__device__ __forceinline__ float key_value(uint32_t d) { return __uint_as_float(0x40000000u - d); }
__device__ __forceinline__ uint32_t fixmass(float e) { return __float2uint_rn(e * kFix); }

// Warp-wide inclusive scan of 64-bit values.
__device__ __forceinline__ unsigned long long warp_scan_u64(unsigned long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// Warp-wide exclusive scan of small counts.
__device__ __forceinline__ int warp_excl_scan(int c, int lane, int& total) {
  int v = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  total = __shfl_sync(0xffffffffu, v, 31);
  return v - c;
}

// A member record of the exact step: key, block, fixed-point mass.
__device__ __forceinline__ uint4 member_record(const ToppScratch& S, uint32_t j) {
  const uint32_t d = S.d[j];
  return make_uint4(d, j, fixmass(key_value(d)), 0u);
}

// Writes the records of the (at most 32) blocks whose key lies in [rlo, rhi]
// to rec[0 .. cnt), in block order (a scan over the row's n keys).
__device__ __forceinline__ void list_range(const ToppScratch& S, int n, uint32_t rlo, uint32_t rhi, uint4* rec,
                                           int lane) {
  const unsigned lt = (1u << lane) - 1u;
  int base = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    bool in = false;
    if (j < n) {
      const uint32_t d = S.d[j];
      in = d >= rlo && d <= rhi;
    }
    const unsigned mk = __ballot_sync(0xffffffffu, in);
    if (in) rec[base + __popc(mk & lt)] = member_record(S, (uint32_t)j);
    base += __popc(mk);
  }
}

// Exact crossing among `cnt` (<= 32) member records rec[], all ranked behind
// mass `base`: returns the member c with ahead(c) < target <= ahead(c) + e_c
// (ahead in (d, j) order), or -1 if none reaches the target.  The members are
// sorted across the warp by (d, j) with a bitonic network, then an inclusive
// scan of their masses in that order finds the crossing.
__device__ __forceinline__ int topp_exact32(const uint4* rec, int cnt, unsigned long long base,
                                            unsigned long long target, int lane) {
  unsigned long long key = ~0ull;  // (d << 32) | j; absent members sort last
  if (lane < cnt) {
    const uint4 r = rec[lane];
    key = ((unsigned long long)r.x << 32) | r.y;
  }
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, jj);
      const bool take_min = ((lane & jj) == 0) == ((lane & k) == 0);
      key = take_min ? (other < key ? other : key) : (other > key ? other : key);
    }
  }
  const bool valid = lane < cnt;
  const unsigned long long m = valid ? (unsigned long long)fixmass(key_value((uint32_t)(key >> 32))) : 0ull;
  const unsigned long long incl = warp_scan_u64(m, lane);
  const unsigned hit = __ballot_sync(0xffffffffu, valid && base + incl >= target);
  if (hit == 0u) return -1;
  return (int)(uint32_t)__shfl_sync(0xffffffffu, key, __ffs(hit) - 1);
}

// A bin's 64-bit mass is kept as two 32-bit sums, of the low 16 bits and of
// the high 16 bits of each added value, so a bin mass is hi * 2^16 + lo
// (kTopPBins words of each, low sums first).  Neither sum can wrap (at most
// 2^14 values of < 2^16 each), so the adds need no carry and no result:
// fire-and-forget 32-bit shared-memory reductions (faster here than 64-bit
// ones), exact and independent of the order of the adds.  (No "memory"
// clobber: the bins are read only after a __syncwarp, and leaving the
// compiler free to move other loads across the reductions keeps several
// blocks' arithmetic in flight.)
__device__ __forceinline__ void bin_add(unsigned long long* bins, int b, uint32_t x) {
  uint32_t* lo = reinterpret_cast<uint32_t*>(bins);
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_u32(lo + b)), "r"(x & 0xFFFFu));
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_u32(lo + kTopPBins + b)), "r"(x >> 16));
}
__device__ __forceinline__ unsigned long long bin_mass(const unsigned long long* bins, int b) {
  const uint32_t* lo = reinterpret_cast<const uint32_t*>(bins);
  return ((unsigned long long)lo[kTopPBins + b] << 16) + lo[b];
}

// Softmax (step 5) + Top-P (step 6) of one band row of n scaled logits:
//
// e_j = 2^((L_j - max) log2 e); blocks ranked by (-e_j, j) == (d_j, j) with
// the exact order-reversing key d_j.  Radix selection on the keys: bins of 16
// per octave of e (bin = d >> 19, the last one collecting everything below
// 2^-14) hold their mass exactly (e_j in 2^-31 fixed point, 64-bit exact
// sums), so one scan gives Z, the crossing bin and the mass ranked before it
// as exact integers.  Blocks of earlier bins are kept, of later bins dropped.
// A member x of the crossing bin is kept iff the mass ranked strictly ahead
// of it is below the target p Z (the top block always): with <= 32 members
// every member sums the masses of the members ahead of it directly, else the
// bin is refined on the lower key bits the same way.  The histogram pass of
// a Top-P row leaves the keys at S.d and the bin masses in S.h; topp_select
// does the rest.
constexpr size_t kTilePair = 2 * 128 * 128;  // floats per score tile pair (both bands)

// Zeroes the warp's 2 KB of bins (16-byte stores).
__device__ __forceinline__ void topp_zero_bins(const ToppScratch& S, int lane) {
  uint4* h = reinterpret_cast<uint4*>(S.h);
  for (int q = lane; q < 2 * kTopPBins / 4; q += 32) h[q] = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
}

// e_j, rank key and exact bin mass of one block (the key stored at S.d[j]).
__device__ __forceinline__ void topp_hist1(const ToppScratch& S, int j, float x, float m) {
  const float e = fast_exp2(fmaf(x, kLog2e, -m));
  const uint32_t d = rank_key(e);
  S.d[j] = d;
  bin_add(S.h, (int)min(d >> 19, (uint32_t)(kTopPBins - 1)), fixmass(e));
}

// Every causal block of a row (p >= 1).
__device__ __forceinline__ void topp_keep_all(int n, uint32_t* bits, int lane) {
  const int nw = (n + 31) >> 5;
  for (int w = lane; w < nw; w += 32) {
    const int lo = w * 32;
    bits[w] |= lo + 32 <= n ? 0xffffffffu : ((1u << (n - lo)) - 1u);
  }
  __syncwarp();
}

// The crossing bin of a band row from its bin masses (after a histogram
// pass): lim = max(floor(p Z), 1) and the first bin whose cumulative mass
// reaches it, with the mass ranked before that bin.  Each lane sums the two
// halves of its 8 bins, the two sums are scanned across the warp side by
// side, and each lane then walks its own 8 bins, so only the lane holding the
// crossing bin finds it.
struct ToppCross {
  unsigned long long target, lim, base;
  int xb;
};
__device__ __forceinline__ ToppCross topp_cross_bin(float p, const ToppScratch& S, int lane) {
  const uint32_t* hlo = reinterpret_cast<const uint32_t*>(S.h);
  const uint32_t* hhi = hlo + kTopPBins;
  const uint4 l0 = reinterpret_cast<const uint4*>(hlo)[2 * lane], l1 = reinterpret_cast<const uint4*>(hlo)[2 * lane + 1];
  const uint4 h0 = reinterpret_cast<const uint4*>(hhi)[2 * lane], h1 = reinterpret_cast<const uint4*>(hhi)[2 * lane + 1];
  const uint32_t bl[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
  const uint32_t bh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  // the warp's sums of the low halves (< 2^30) and of the high halves fit 32 bits
  const uint32_t sl = (bl[0] + bl[1]) + (bl[2] + bl[3]) + (bl[4] + bl[5]) + (bl[6] + bl[7]);
  const uint32_t sh = (bh[0] + bh[1]) + (bh[2] + bh[3]) + (bh[4] + bh[5]) + (bh[6] + bh[7]);
  uint32_t il = sl, ih = sh;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t ul = __shfl_up_sync(0xffffffffu, il, o), uh = __shfl_up_sync(0xffffffffu, ih, o);
    if (lane >= o) {
      il += ul;
      ih += uh;
    }
  }
  const unsigned long long Z = ((unsigned long long)__shfl_sync(0xffffffffu, ih, 31) << 16) +
                               __shfl_sync(0xffffffffu, il, 31);
  ToppCross C;
  C.target = (unsigned long long)((double)p * (double)Z);
  C.lim = C.target > 0ull ? C.target : 1ull;
  unsigned long long run = (((unsigned long long)(ih - sh)) << 16) + (il - sl);  // mass before this lane's bins
  int q_hit = -1;
  unsigned long long b_hit = 0ull;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const unsigned long long m = ((unsigned long long)bh[q] << 16) + bl[q];
    if (q_hit < 0 && run + m >= C.lim) {
      q_hit = q;
      b_hit = run;
    }
    run += m;
  }
  const int F = __ffs(__ballot_sync(0xffffffffu, q_hit >= 0)) - 1;  // lim <= Z: some lane holds it
  C.xb = 8 * F + __shfl_sync(0xffffffffu, q_hit, F);
  C.base = __shfl_sync(0xffffffffu, b_hit, F);
  return C;
}

__device__ __forceinline__ void topp_refine(int n, const ToppScratch& S, const ToppCross& C, uint32_t* bits,
                                            float* dbgw, int lane);

// The selection of step (6) on a band row whose keys are at S.d and whose
// bin masses are in S.h (after a histogram pass); ORs the kept blocks into
// bits[].  One pass over the keys keeps the blocks of earlier bins (lane u
// collects the word of slot u of each batch of 32 slots) and lists the
// crossing bin's members (the first 32, in block order) by ballot; with <= 32
// members every member sums the masses of the members ranked ahead of it,
// else the bin is refined.
__device__ __forceinline__ void topp_select(int n, float p, const ToppScratch& S, uint32_t* bits, float* dbgw,
                                            int lane) {
  const unsigned lt = (1u << lane) - 1u;
  const int ns = (n + 31) >> 5;
  uint4* rec = reinterpret_cast<uint4*>(S.h);  // member records, over the bins once they are read
  const ToppCross C = topp_cross_bin(p, S, lane);
  __syncwarp();  // the bins are read before member records overwrite them
  const uint32_t key_lo = (uint32_t)C.xb << 19;
  const uint32_t key_hi = C.xb == kTopPBins - 1 ? 0xffffffffu : ((uint32_t)(C.xb + 1) << 19);
  int cnt = 0;
  for (int u0 = 0; u0 < ns; u0 += 32) {
    const int u1 = min(u0 + 32, ns);
    uint32_t myw = 0u;
#pragma unroll 4
    for (int uu = u0; uu < u1; ++uu) {
      const int j = uu * 32 + lane;
      const uint32_t d = j < n ? S.d[j] : 0xffffffffu;
      const unsigned kb = __ballot_sync(0xffffffffu, d < key_lo);
      const bool in = d >= key_lo && d < key_hi;
      const unsigned mk = __ballot_sync(0xffffffffu, in);
      const int pos = cnt + __popc(mk & lt);
      if (in && pos < 32) rec[pos] = make_uint4(d, (uint32_t)j, fixmass(key_value(d)), 0u);
      cnt += __popc(mk);
      if (lane == uu - u0) myw = kb;
    }
    if (lane < u1 - u0) bits[u0 + lane] |= myw;
  }
  __syncwarp();
  if (cnt <= 32) {
    const uint4 me = lane < cnt ? rec[lane] : make_uint4(0xffffffffu, 0x7fffffffu, 0u, 0u);
    unsigned long long ahead = C.base;
#pragma unroll 4
    for (int y = 0; y < cnt; ++y) {
      const uint4 o = rec[y];
      if (o.x < me.x || (o.x == me.x && o.y < me.y)) ahead += o.z;
    }
    if (lane < cnt && ahead < C.lim) atomicOr(&bits[me.y >> 5], 1u << (me.y & 31));
    if (dbgw)
      for (int j = lane; j < n; j += 32) dbgw[j] = key_value(S.d[j]);
    __syncwarp();
    return;
  }
  topp_refine(n, S, C, bits, dbgw, lane);
}

// A crossing bin with more than 32 members: refine it on lower key bits (the
// keys at S.d), then keep every block ranked at or ahead of the crossing.
__device__ __forceinline__ void topp_refine(int n, const ToppScratch& S, const ToppCross& C, uint32_t* bits,
                                            float* dbgw, int lane) {
  const unsigned lt = (1u << lane) - 1u;
  uint4* rec = reinterpret_cast<uint4*>(S.h);
  const unsigned long long target = C.target, lim = C.lim;
  unsigned long long base = C.base;
  const int xb = C.xb;
  const uint32_t key_lo = (uint32_t)xb << 19;
  const uint32_t key_hi = xb == kTopPBins - 1 ? 0xffffffffu : ((uint32_t)(xb + 1) << 19);
  (void)lim;
  // refine on lower key bits, 8-bit digits: a regular bin spans 2^19 keys
  // (digits at shifts 11, 3, 0), the catch-all bin up to 2^30 (22, 14, 6, 0).
  // The members are the row's keys in [rlo, rhi], found by scanning the keys.
  int cross = -1;
  uint32_t rlo = key_lo, rhi = key_hi - 1u;
  const bool wide = xb == kTopPBins - 1;
  for (int level = 0;; ++level) {
    const int sh = wide ? (level == 0 ? 22 : level == 1 ? 14 : level == 2 ? 6 : 0)
                        : (level == 0 ? 11 : level == 1 ? 3 : 0);
    for (int b = lane; b < kTopPBins; b += 32) S.h[b] = 0ull;  // both halves: 2 x 256 words
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const uint32_t d = S.d[j];
      if (d >= rlo && d <= rhi)
        bin_add(S.h, (int)min((d - rlo) >> sh, (uint32_t)(kTopPBins - 1)), fixmass(key_value(d)));
    }
    __syncwarp();
    unsigned long long h2[8], t2 = 0ull;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      h2[q] = bin_mass(S.h, lane * 8 + q);
      t2 += h2[q];
    }
    const unsigned long long inc2 = warp_scan_u64(t2, lane);
    unsigned long long run = inc2 - t2;
    int bin2 = -1;
    unsigned long long bb = 0ull;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (bin2 < 0 && base + run + h2[q] >= target && h2[q] > 0ull) {
        bin2 = lane * 8 + q;
        bb = base + run;
      }
      run += h2[q];
    }
    const unsigned f2 = __ballot_sync(0xffffffffu, bin2 >= 0);
    __syncwarp();  // the bins are read before the member records overwrite them
    if (f2 == 0u) {
      // (exact sums make this unreachable) the members' mass stays below
      // the target: all of them are kept -- the cut is the last member
      uint32_t bd = 0u;
      int bj = -1;
      for (int j = lane; j < n; j += 32) {
        const uint32_t dd = S.d[j];
        if (dd >= rlo && dd <= rhi && (bj < 0 || dd > bd || (dd == bd && j > bj))) {
          bd = dd;
          bj = j;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint32_t od = __shfl_xor_sync(0xffffffffu, bd, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (bj < 0 || (oj >= 0 && (od > bd || (od == bd && oj > bj)))) {
          bd = od;
          bj = oj;
        }
      }
      cross = bj;
      break;
    }
    const int sl = __ffs(f2) - 1;
    const int xb2 = __shfl_sync(0xffffffffu, bin2, sl);
    base = __shfl_sync(0xffffffffu, bb, sl);
    const uint32_t blo = rlo + ((uint32_t)xb2 << sh);
    // the last digit bin also holds every key above its start
    const uint32_t bhi = sh == 0 ? blo : (xb2 == kTopPBins - 1 ? rhi : blo + ((1u << sh) - 1u));
    int c2 = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      bool in = false;
      if (j < n) {
        const uint32_t d = S.d[j];
        in = d >= blo && d <= bhi;
      }
      c2 += __popc(__ballot_sync(0xffffffffu, in));
    }
    rlo = blo;
    rhi = bhi;
    if (c2 <= 32) {
      list_range(S, n, rlo, rhi, rec, lane);
      __syncwarp();
      cross = topp_exact32(rec, c2, base, target, lane);
      break;
    }
    if (sh == 0) {
      // equal keys: the first member (by index) whose cumulative mass
      // reaches the target
      const unsigned long long me = (unsigned long long)fixmass(key_value(blo));
      unsigned long long acc = base;
      for (int j0 = 0; j0 < n && cross < 0; j0 += 32) {
        const int j = j0 + lane;
        const bool ok = j < n && S.d[j] == blo;
        const unsigned mk = __ballot_sync(0xffffffffu, ok);
        const int pos = __popc(mk & lt);
        const bool hit = ok && acc + me * (unsigned long long)(pos + 1) >= target;
        const unsigned hm = __ballot_sync(0xffffffffu, hit);
        if (hm) cross = __shfl_sync(0xffffffffu, j, __ffs(hm) - 1);
        acc += me * (unsigned long long)__popc(mk);
      }
      break;
    }
  }
  __syncwarp();
  // the weights e_j as ranked and summed (debug output)
  if (dbgw)
    for (int j = lane; j < n; j += 32) dbgw[j] = key_value(S.d[j]);
  // every block ranked at or ahead of the crossing
  const uint32_t dc = cross >= 0 ? S.d[cross] : 0xffffffffu;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    bool keep = false;
    if (j < n) {
      const uint32_t d = S.d[j];
      keep = cross < 0 || d < dc || (d == dc && j <= cross);
    }
    const unsigned word = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) bits[j0 >> 5] |= word;
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// score item: up to 128 consecutive query blocks i of one Q head (the rows of
// one MMA, M = 128) against every key block j <= i of its KV head, in column
// chunks of N = 128 (64 for the widest band layout).  Step (5): logits of
// both bands on the tensor cores, accumulators in tensor memory, double
// buffered; warp roles: warp 0 lane 0 streams the operands (TMA), warp 1
// lane 0 issues the products, warps 4-7 read the accumulators of a finished
// chunk, scale them, write the score tiles and keep the row maxima.  The
// chunk's rows then wait for a Top-P item (steps 5-7 per row).
// ---------------------------------------------------------------------------
struct ScoreState {  // mbarrier parities, carried across items (each role keeps its own)
  uint32_t a, b, free, mma, acc;
};

// The B operand is streamed one term at a time ("units": chunk c, term t,
// u = 3c + t) through kBSlots shared-memory slots.  Unit u's products pair
// its B term with every A term whose cross term matters: t = h with A = h, m,
// l; t = m with A = h, m; t = l with A = h.  High band K steps accumulate
// into d, low band K steps into d + N.
__device__ __forceinline__ void score_mma_unit(const EstParams& P, uint32_t d, uint32_t a0, uint32_t b, int term,
                                               int n_cols, uint32_t idesc) {
  const uint32_t nch = (uint32_t)P.bl.dp / 64;
  const uint32_t b_bytes = (uint32_t)n_cols * 128;  // one 64-dim chunk of N rows
  const int na = term == 0 ? 3 : (term == 1 ? 2 : 1);
  const int k_hi = P.bl.s2 / 16, k_lo0 = P.bl.s1 / 16, k_lo1 = P.bl.s3 / 16;
  // a descriptor's start address field is the byte address / 16, so an
  // operand offset is added to the descriptor directly
  const uint64_t bdesc = smem_desc_sw128(b, 16, 1024);
  for (int ta = 0; ta < na; ++ta) {
    const uint64_t adesc = smem_desc_sw128(a0 + (uint32_t)ta * nch * kOpChunk, 16, 1024);
    const bool first = term == 0 && ta == 0;
    for (int k = 0; k < k_hi; ++k) {
      const uint32_t ka = ((uint32_t)(k >> 2) * kOpChunk + (uint32_t)(k & 3) * 32) >> 4;
      const uint32_t kb = ((uint32_t)(k >> 2) * b_bytes + (uint32_t)(k & 3) * 32) >> 4;
      mma_bf16_ss(d, adesc + ka, bdesc + kb, idesc, (first && k == 0) ? 0u : 1u);
    }
    for (int k = k_lo0; k < k_lo1; ++k) {
      const uint32_t ka = ((uint32_t)(k >> 2) * kOpChunk + (uint32_t)(k & 3) * 32) >> 4;
      const uint32_t kb = ((uint32_t)(k >> 2) * b_bytes + (uint32_t)(k & 3) * 32) >> 4;
      mma_bf16_ss(d + (uint32_t)n_cols, adesc + ka, bdesc + kb, idesc, (first && k == k_lo0) ? 0u : 1u);
    }
  }
}

__device__ __forceinline__ void score_item(const EstParams& P, const CUtensorMap* tm, int g, int y,
                                           unsigned char* smem, PoolSmem& sm, ScoreState& ps) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int bi = g / P.hkv, kv = g - bi * P.hkv;
  const int nchunk = (P.nb + kScoreRows - 1) / kScoreRows;
  int chunk, part;
  const int pb = score_part_blocks(P, g);
  score_part_of(P, y / P.G, pb, chunk, part);  // longest rows first
  const int bh = bi * P.hq + kv * P.G + y % P.G;
  const int i0 = chunk * kScoreRows;
  const int nbb = seq_blocks(P, bi);
  const int max_i = min(nbb, i0 + kScoreRows) - 1;  // < i0: the chunk is past the sequence, only counted
  const uint32_t nch = (uint32_t)P.bl.dp / 64;
  const int ncolw = P.ncolw;  // N: key blocks per column chunk
  // this part's key blocks [j0, j1): column chunks c0 .. c0 + ncol - 1
  const int j0 = part * pb, j1 = min(j0 + pb, max_i + 1);
  const int c0 = j0 / ncolw;
  const int ncol = (j1 - 1) / ncolw + 1 - c0;
  const int units = 3 * ncol;
  const uint32_t idesc = ncolw == 128 ? idesc_bf16_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 64, 0, 0);
  const uint32_t sbase = (smem_u32(smem) + 1023u) & ~1023u;
  if (sbase - smem_u32(smem) + (uint32_t)gemm_smem_bytes(P.bl.dp, ncolw) - 1024u > (uint32_t)P.stream_bytes) {
    if (t == 0) set_device_error(-6);  // PRISM_ERR_UNSUPPORTED (host sizing makes this unreachable)
    return;
  }
  const uint32_t a0 = sbase;                                 // 3 terms x nch chunks x 16 KB
  const uint32_t slot_bytes = nch * (uint32_t)ncolw * 128;  // one B term of N rows
  const uint32_t b_base = sbase + kTerms * nch * kOpChunk;
  auto slot_addr = [&](int u) { return b_base + (uint32_t)(u % kBSlots) * slot_bytes; };
  auto bar_b = [&](int u) { return smem_u32(&sm.bar_b[u % kBSlots]); };
  auto bar_f = [&](int u) { return smem_u32(&sm.bar_free[u % kBSlots]); };
  auto bar_m = [&](int c) { return smem_u32(&sm.bar_mma[c & 1]); };
  auto bar_e = [&](int c) { return smem_u32(&sm.bar_acc[c & 1]); };
  auto dacc = [&](int c) { return sm.tmem + 256u * (uint32_t)(c & 1); };

  if (max_i < i0) {
    // past the sequence: no rows, only the part count below
  } else if (warp == 0) {
    if (lane == 0) {  // operand producer
      const int arow = bh * P.nb + i0;          // pooled rows of the Q head
      const int brow0 = (P.q_rows + g) * P.nb;  // pooled rows of the KV head
      fence_proxy_async_smem();                 // generic writes of the last item before async ones
      const uint32_t bar_a = smem_u32(&sm.bar_a);
      mbar_arrive_expect_tx(bar_a, kTerms * nch * kOpChunk);
      for (int term = 0; term < kTerms; ++term)
        for (uint32_t k = 0; k < nch; ++k)
          tma_load_2d(a0 + ((uint32_t)term * nch + k) * kOpChunk, &tm[term], (int)(64 * k), arow, bar_a);
      for (int u = 0; u < units; ++u) {
        const int sl = u % kBSlots;
        if (u >= kBSlots) {  // the slot's previous unit has been multiplied
          mbar_wait(bar_f(u), (ps.free >> sl) & 1u);
          ps.free ^= 1u << sl;
        }
        const int c = u / 3, term = u - 3 * c;
        mbar_arrive_expect_tx(bar_b(u), slot_bytes);
        for (uint32_t k = 0; k < nch; ++k)
          tma_load_2d(slot_addr(u) + k * (uint32_t)ncolw * 128, &tm[term + (ncolw == 128 ? 0 : 3)],
                      (int)(64 * k), brow0 + (c0 + c) * ncolw, bar_b(u));
      }
      for (int u = max(units - kBSlots, 0); u < units; ++u) {  // the last releases
        mbar_wait(bar_f(u), (ps.free >> (u % kBSlots)) & 1u);
        ps.free ^= 1u << (u % kBSlots);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // product issuer
      mbar_wait(smem_u32(&sm.bar_a), ps.a & 1u);
      ps.a ^= 1u;
      for (int c = 0; c < ncol; ++c) {
        if (c >= 2) {  // the accumulators of chunk c - 2 have been read out
          mbar_wait(bar_e(c), (ps.acc >> (c & 1)) & 1u);
          ps.acc ^= 1u << (c & 1);
        }
        for (int tt = 0; tt < 3; ++tt) {
          const int u = 3 * c + tt, sl = u % kBSlots;
          mbar_wait(bar_b(u), (ps.b >> sl) & 1u);
          ps.b ^= 1u << sl;
          tc_fence_after();
          score_mma_unit(P, dacc(c), a0, slot_addr(u), tt, ncolw, idesc);
          mma_commit(bar_f(u));
        }
        mma_commit(bar_m(c));
      }
      for (int c = max(ncol - 2, 0); c < ncol; ++c) {  // the last read-outs
        mbar_wait(bar_e(c), (ps.acc >> (c & 1)) & 1u);
        ps.acc ^= 1u << (c & 1);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // warp w reads TMEM lane quarter w % 4 in the 16 x 256-bit shape, 32
    // columns at a time: four threads share a row, each holding two adjacent
    // key blocks, so every store instruction writes eight whole 32-byte
    // sectors of the score tiles.
    const float sc_hi = P.tau[bh * 4 + 2], sc_lo = P.tau[bh * 4 + 3];
    const int q4 = warp & 3;
    const int gr = lane >> 2, cq = (lane & 3) * 2;
    float mx[2][2][2];  // [lane half][row of the pair][band]: row maxima over this part's j <= i
#pragma unroll
    for (int a = 0; a < 8; ++a) (&mx[0][0][0])[a] = -INFINITY;
    for (int c = 0; c < ncol; ++c) {
      mbar_wait(bar_m(c), (ps.mma >> (c & 1)) & 1u);
      ps.mma ^= 1u << (c & 1);
      tc_fence_after();
#pragma unroll
      for (int lh = 0; lh < 2; ++lh) {
#pragma unroll 1
        for (int col0 = 0; col0 < ncolw; col0 += 32) {  // column in the chunk
          const uint32_t taddr = dacc(c) + ((uint32_t)(q4 * 32 + lh * 16) << 16) + (uint32_t)col0;
          uint32_t vh[16], vl[16];
          tmem_ld_16x256b_x4(taddr, vh);
          tmem_ld_16x256b_x4(taddr + (uint32_t)ncolw, vl);
          tmem_wait_ld_dep16(vh);
          tmem_wait_ld_dep16(vl);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int j = (c0 + c) * ncolw + col0 + 8 * k + cq;  // key block of the first value
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const int rl = q4 * 32 + lh * 16 + gr + 8 * rr;  // row in the item
              float* dst = score_tile(P, bh, chunk, j >> 7) + rl * 128 + (j & 127);
              const float h0 = __uint_as_float(vh[4 * k + 2 * rr]) * sc_hi;
              const float h1 = __uint_as_float(vh[4 * k + 2 * rr + 1]) * sc_hi;
              const float l0 = __uint_as_float(vl[4 * k + 2 * rr]) * sc_lo;
              const float l1 = __uint_as_float(vl[4 * k + 2 * rr + 1]) * sc_lo;
              *reinterpret_cast<float2*>(dst) = make_float2(h0, h1);
              *reinterpret_cast<float2*>(dst + 128 * 128) = make_float2(l0, l1);
              const int i = i0 + rl;
              if (j <= i) {
                mx[lh][rr][0] = fmaxf(mx[lh][rr][0], h0);
                mx[lh][rr][1] = fmaxf(mx[lh][rr][1], l0);
              }
              if (j + 1 <= i) {
                mx[lh][rr][0] = fmaxf(mx[lh][rr][0], h1);
                mx[lh][rr][1] = fmaxf(mx[lh][rr][1], l1);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_e(c));
    }
    // the four threads of a row combine their maxima; one of them folds them
    // into the row's maxima over every part
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      float& v = (&mx[0][0][0])[a];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    }
    if ((lane & 3) == 0) {
#pragma unroll
      for (int lh = 0; lh < 2; ++lh)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int i = i0 + q4 * 32 + lh * 16 + gr + 8 * rr;
          if (i <= max_i && mx[lh][rr][0] > -INFINITY) {  // this part holds keys j <= i of the row
            atomicMax(&P.rmax[((size_t)bh * P.nb + i) * 2 + 0], max_enc(mx[lh][rr][0]));
            atomicMax(&P.rmax[((size_t)bh * P.nb + i) * 2 + 1], max_enc(mx[lh][rr][1]));
          }
        }
    }
  }
  named_barrier(kBarStream, kStreamThreads);  // score tiles complete
  // publish: count the part for the chunk's Top-P rows
  if (t == 0) {
    __threadfence();
    red_release_gpu_add(&P.sync[2 + 2 * P.n_groups + bh * nchunk + chunk], 1u);
  }
  named_barrier(kBarStream, kStreamThreads);  // shared memory is reused by the next item
}

// ---------------------------------------------------------------------------
// Top-P rows: steps (5)-(7) for one query-block row i of one (batch, Q head),
// both bands, union, the whole mask row.  Every warp of the Top-P lane (and,
// once the stream queue is empty, of the stream lane) claims rows one at a
// time from a device queue -- no team barriers -- and waits (bounded) until
// every part of the row's score chunk is written.  Rows are queued per KV
// group in the order their score chunks complete (longest rows first).
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void l2_discard_line(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// The warp's shared memory for Top-P rows: keys [nbp] | bins (2 KB, then the
// member records) | mask bit row [W].
__device__ __forceinline__ ToppScratch topp_scratch(const EstParams& P, unsigned char* wb, uint32_t*& bits) {
  const int nbp = (P.nb + 7) & ~7;
  ToppScratch S;
  S.d = reinterpret_cast<uint32_t*>(wb);
  S.h = reinterpret_cast<unsigned long long*>(wb + (size_t)nbp * 4);
  bits = reinterpret_cast<uint32_t*>(wb + (size_t)nbp * 4 + kTopPBins * 8);
  return S;
}

// One query-block row i of one (batch, Q head), both bands: each band's
// logits are read once, straight from the score tiles in L2, and turned into
// weights, rank keys (stored for the selection) and exact bin masses against
// the row maximum the score items published; then the selection runs on
// shared memory.  The loads are software-pipelined: eight 128-byte lines per
// lane group, the next group's loads issued before the current group is
// ranked, and the next band's first group issued before this band's
// selection, so L2 latency is paid about once per band rather than once per
// group.  Once a band is read, the row's lines of its tiles are dropped from
// L2 (never read again, so never written back).  The mask row is built in the
// warp's bit row and written whole.  One compact routine for every row
// length: the warps of an SM run several roles at once, and the code they
// share must stay small.
constexpr int kToppGroup = 8;  // slots (32-block columns of a row) per load group
__device__ __forceinline__ void topp_row(const EstParams& P, int bh, int i, int chunk, unsigned char* wb, int lane) {
  const int n = i + 1, ns = (n + 31) >> 5;
  uint32_t* bits;
  const ToppScratch T = topp_scratch(P, wb, bits);
  const float* row = score_tile(P, bh, chunk, 0) + (size_t)(i - chunk * kScoreRows) * 128;
  const size_t tri = (size_t)P.nb * (P.nb + 1) / 2;
  const bool all = P.p >= 1.0f;
  // slot u of lane L = block 32 u + L: tile u / 4, columns 32 (u % 4) + L
  auto slot_ptr = [&](int band, int u) {
    return row + band * (128 * 128) + (size_t)(u >> 2) * kTilePair + ((u & 3) << 5) + lane;
  };
  float v[kToppGroup];
  auto load_group = [&](int band, int u0) {
#pragma unroll
    for (int q = 0; q < kToppGroup; ++q)
      v[q] = 32 * (u0 + q) + lane < n ? __ldcg(slot_ptr(band, u0 + q)) : 0.f;
  };
  const uint32_t* rm = P.rmax + ((size_t)bh * P.nb + i) * 2;
  const uint32_t rm0 = __ldcg(rm), rm1 = __ldcg(rm + 1);
  for (int w = lane; w < P.W; w += 32) bits[w] = 0u;
  load_group(0, 0);
  for (int band = 0; band < 2; ++band) {
    const size_t drow = ((size_t)bh * 2 + band) * tri + (size_t)i * (i + 1) / 2;
    float* dbg = P.dbg_scores ? P.dbg_scores + drow : nullptr;
    const float m = max_dec(band == 0 ? rm0 : rm1) * kLog2e;
    if (!all) topp_zero_bins(T, lane);
    for (int u0 = 0; u0 < ns; u0 += kToppGroup) {
      float cur[kToppGroup];
#pragma unroll
      for (int q = 0; q < kToppGroup; ++q) cur[q] = v[q];
      if (u0 + kToppGroup < ns) load_group(band, u0 + kToppGroup);  // in flight while this group is ranked
#pragma unroll
      for (int q = 0; q < kToppGroup; ++q) {
        const int j = 32 * (u0 + q) + lane;
        if (j < n) {
          if (dbg) dbg[j] = cur[q];
          if (!all) topp_hist1(T, j, cur[q], m);
        }
      }
    }
    __syncwarp();
    // the row's 4 (chunk + 1) lines of this band, the unused ones above the
    // diagonal included
    for (int u = lane; u < 4 * (chunk + 1); u += 32)
      l2_discard_line(row + band * (128 * 128) + (size_t)(u >> 2) * kTilePair + ((u & 3) << 5));
    if (band == 0) load_group(1, 0);  // in flight during this band's selection
    if (all)
      topp_keep_all(n, bits, lane);
    else
      topp_select(n, P.p, T, bits, P.dbg_weights ? P.dbg_weights + drow : nullptr, lane);
  }
  if (P.force && lane == 0) {  // optional additions to M_high | M_low
    if (P.force & 1) bits[0] |= 1u;
    if (P.force & 2) bits[i >> 5] |= 1u << (i & 31);
  }
  __syncwarp();
  uint32_t* dst = P.mask + ((size_t)bh * P.nb + i) * P.W;
  for (int w = lane; w < P.W; w += 32) dst[w] = bits[w];
  __syncwarp();
}

// A warp's loop over the Top-P queue: entries x = 0, 1, ... of P.n_groups *
// P.topp_rows, one row per claim (finer claims balance the end of the launch
// better than batches of rows); per group g, entry y -> score chunk nchunk -
// 1 - y / (G 128) (longest rows first), Q head y / 128 % G, row y % 128 of the
// chunk.  The warp claims its next row before it works on the current one,
// so the claim's latency is hidden.  After its mask row is written a row is
// counted for its kToppRows-row segment (the attention of a prefill waits on
// the count).  `wb`: the warp's shared memory (topp_scratch).
__device__ __forceinline__ void topp_warp_loop(const EstParams& P, unsigned char* wb) {
  const int lane = threadIdx.x & 31;
  const int nchunk = (P.nb + kScoreRows - 1) / kScoreRows;
  const int nseg = (P.nb + kToppRows - 1) / kToppRows;
  const int total = P.n_groups * P.topp_rows;
  int xc = 0;
  if (lane == 0) xc = (int)atomicAdd(&P.sync[1], 1u);
  for (;;) {
    const int x = __shfl_sync(0xffffffffu, xc, 0);
    if (x >= total) break;
    if (lane == 0) xc = (int)atomicAdd(&P.sync[1], 1u);  // the next row, used in the next iteration
    const int g = x / P.topp_rows, y = x - g * P.topp_rows;
    const int chunk = nchunk - 1 - y / (P.G * kScoreRows);
    const int hh = (y / kScoreRows) % P.G;
    const int i = chunk * kScoreRows + y % kScoreRows;
    if (i >= P.nb) continue;  // past the layout's last block
    const int bi = g / P.hkv, kv = g - bi * P.hkv;
    const int bh = bi * P.hq + kv * P.G + hh;
    if (i >= seq_blocks(P, bi)) {  // past the sequence: an empty mask row
      for (int w = lane; w < P.W; w += 32) P.mask[((size_t)bh * P.nb + i) * P.W + w] = 0u;
    } else {
      int ok = 1;
      if (lane == 0)
        ok = count_wait_ns(&P.sync[2 + 2 * P.n_groups + bh * nchunk + chunk],
                           (uint32_t)score_parts(chunk, score_part_blocks(P, g)), kWaitLimitNs) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;  // (timed out: error recorded)
      __syncwarp();  // orders the lanes' loads of the chunk after lane 0's acquire
      topp_row(P, bh, i, chunk, wb, lane);
    }
    __syncwarp();  // every lane's mask words are written before lane 0 releases them
    if (lane == 0) red_release_gpu_add(&P.ready[(size_t)bh * nseg + i / kToppRows], 1u);
  }
}

// ---------------------------------------------------------------------------
// the persistent kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kEstThreads, 1)
estimator_kernel(const __grid_constant__ EstParams P, const __grid_constant__ TermMaps tms) {
  extern __shared__ __align__(16) unsigned char est_smem[];
  __shared__ PoolSmem psm;
  // a kernel launched after this one with programmatic serialization (the
  // attention of a prefill) may be scheduled on SMs this grid leaves; it
  // waits for the mask rows it reads through the `ready` counters
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int s_next, s_ok;
  const int stages = P.pool_stages;
  PoolState pst = {0u, 0u, 0u, 0u, 0};
  ScoreState ss = {0u, 0u, 0u, 0u, 0u};
  for (int i = threadIdx.x; i < 16 * 32; i += kEstThreads) psm.ones[i] = 0x3F803F80u;  // bf16 1.0 pairs
  fence_proxy_async_smem();  // read by the tensor cores
  if (threadIdx.x == 0) {
    for (int st = 0; st < stages; ++st) {
      mbar_init(smem_u32(&psm.bars[st]), 1u);
      mbar_init(smem_u32(&psm.bars_free[st]), 1u);
    }
    mbar_init(smem_u32(&psm.bar_pool), 1u);
    mbar_init(smem_u32(&psm.bar_pool_half), 1u);
    mbar_init(smem_u32(&psm.bar_a), 1u);
    for (int sl = 0; sl < kBSlots; ++sl) {
      mbar_init(smem_u32(&psm.bar_b[sl]), 1u);
      mbar_init(smem_u32(&psm.bar_free[sl]), 1u);
    }
    mbar_init(smem_u32(&psm.bar_mma[0]), 1u);
    mbar_init(smem_u32(&psm.bar_mma[1]), 1u);
    mbar_init(smem_u32(&psm.bar_acc[0]), 4u);  // one arrival per read-out warp
    mbar_init(smem_u32(&psm.bar_acc[1]), 4u);
    fence_mbar_init();
    for (int m = 0; m < 8; ++m) tma_prefetch_desc(&tms.m[m]);
  }
  if ((threadIdx.x >> 5) == 0) {  // score items: 2 chunks x (hi, lo) x 128 columns; pool items: 32 x 16
    tmem_alloc(smem_u32(&psm.tmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int warp = threadIdx.x >> 5;
  if (in_stream_lane(warp)) {
    const int sid = stream_tid(threadIdx.x);
    int total = P.n_groups * P.pool_items;
    for (int gg = 0; gg < P.n_groups; ++gg) total += score_fine(P, gg) ? P.score_items_fine : P.score_items;
    // During a pool item thread 0 already claims the lane's next item (the
    // claim's latency is hidden, and a following pool item's tiles can start
    // streaming); a score item claims its successor only when it is done, so
    // no pool item is held back behind it.  A claimed item only waits for
    // items earlier in the queue, so the schedule cannot deadlock.
    if (sid == 0) s_next = (int)atomicAdd(&P.sync[0], 1u);
    for (;;) {
      named_barrier(kBarStream, kStreamThreads);
      const int x = s_next;
      named_barrier(kBarStream, kStreamThreads);
      if (x >= total) break;
      int g, y;
      const int kind = decode_stream(P, x, g, y);
      if (kind == kItemPool) {
        const int x_next = sid == 0 ? (int)atomicAdd(&P.sync[0], 1u) : total;
        if (sid == 0) s_next = x_next;  // read by all after the item's last barrier
        pool_item(P, tms.m, g, y, x_next, psm, est_smem, stages, pst);
        continue;
      }
      // a score item waits until its group's pooling and temperatures are published
      if (sid == 0) s_ok = flag_wait_ns(&P.sync[2 + P.n_groups + g], kWaitLimitNs) ? 1 : 0;
      named_barrier(kBarStream, kStreamThreads);
      if (s_ok) score_item(P, tms.m, g, y, est_smem, psm, ss);
      named_barrier(kBarStream, kStreamThreads);
      if (sid == 0) s_next = (int)atomicAdd(&P.sync[0], 1u);
    }
    // the stream queue is empty (this CTA's last item is done, its shared
    // memory free): the lane's warps join the Top-P queue
    const int sw = stream_warp(warp);
    if (sw < P.team_warps) topp_warp_loop(P, est_smem + (size_t)sw * P.team_stride);
  } else {
    const int lw = lane_warp(warp);
    if (lw < P.lane_warps) topp_warp_loop(P, est_smem + P.lane_off + (size_t)lw * P.lane_stride);
  }
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) {
    tc_fence_after();
    tmem_dealloc(psm.tmem, 512);
  }
}

}  // namespace prism
