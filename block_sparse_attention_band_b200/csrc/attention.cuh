// Causal block-sparse attention prefill on the 5th-generation tensor cores.
//
// "Prism: Spectral-Aware Block-Sparse Attention", gist.science Technical
// Summary section 1: block-sparse attention computes only a subset of the
// attention blocks; here the subset is the estimator's mask M (one bit per
// (query block i, key block j)), token-causal inside the diagonal block.
//
// Work item = two 128-query tiles of one Q head, adjacent query blocks i and
// i - 1: they read the same KV head, so every K/V tile fetched by TMA serves
// both, and their kept key blocks overlap most (a step that feeds only one
// tile leaves the other tile's softmax nothing to overlap).  The key blocks
// visited are the union of the two tiles' kept sets; each tile computes only
// its own kept blocks.
//
// 384 threads (12 warps; registers re-split per warpgroup: warps 0-3 keep 72,
// the two softmax warpgroups get 216 so a whole S row stays in registers):
//   warp 0      TMA producer: Q_A, Q_B once; K_j, V_j of every visited block
//               into a 2-stage ring (128-byte swizzled, two 16 KB halves
//               each).  A K stage is refilled once the Q K^T products that
//               read it are done, a V stage once its P V products are.
//   warp 1      MMA issuer (one thread), tcgen05.mma kind::f16, bf16 in /
//               fp32 accumulate in tensor memory (512 columns):
//                 S_A = cols [0,128)  S_B = [128,256)  O_A = [256,384)  O_B = [384,512)
//               S = Q K_j^T (A and B from shared memory), then O += P V_j
//               with P read from tensor memory (bf16, written over S).
//               Issue order: PV_A(t), QK_A(t+1), PV_B(t), QK_B(t+1), so one
//               tile's softmax overlaps the other tile's matrix products;
//               each P V product starts on keys 0-95 as soon as the softmax
//               has published that part of P, while it computes keys 96-127,
//               so only a 32-key product separates the end of a tile's
//               softmax from its next Q K^T.
//               A tile that skips step t but takes step t + 1 gets its Q K^T
//               at the start of step t when K(t + 1) has already landed, so
//               its softmax runs beside the other tile's (at low density more
//               than half the steps feed one tile only, mostly alternating).
//   warps 2-3   idle
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: thread =
//               query row = tensor-memory lane 32*(warp%4)+lane.  Online
//               softmax in base 2; O is rescaled in tensor memory only when
//               the running max grows by more than 8 (a factor 256), so the
//               unnormalised values stay bounded and most steps skip it.
// The grid runs the items of one KV head after the other, within a head from
// the last query block (most key blocks) down.
#pragma once
#include "ptx.cuh"

namespace prism {
namespace attn {

constexpr int kThreads = 384;
// register split: 128 * kRegsLow + 256 * kRegsHigh must not exceed the
// 384 * (registers per thread at launch) the CTA is given
constexpr uint32_t kRegsLow = 72;
constexpr uint32_t kRegsHigh = 216;
constexpr int kMinLaunchRegs = (128 * kRegsLow + 256 * kRegsHigh + 383) / 384;
static_assert(kMinLaunchRegs <= 168, "register split exceeds what a 384-thread CTA can be given");
constexpr uint32_t kHalfBytes = 128 * 64 * 2;    // 128 rows x 64 bf16 (one swizzle span)
constexpr uint32_t kTileBytes = 2 * kHalfBytes;  // 128 x 128 bf16
constexpr uint32_t kOffQ = 0;                    // Q_A, Q_B
constexpr uint32_t kOffK = 2 * kTileBytes;       // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffV + 2 * kTileBytes;
constexpr int kMaxMaskWords = 16384 / 32;  // mask words of one row at the largest nb
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// P is published in two parts: keys [0, 16 kPFirstSteps) first, so the P V
// product on them runs while the softmax computes the rest; only the short
// second part's product then stands between the end of the softmax and the
// tile's next Q K^T
constexpr int kPFirstSteps = 6;

// Barrier slots (8 bytes each) after kOffBar.
enum : uint32_t {
  kBarQ = 0,
  kBarKFull = 1,    // [2]
  kBarVFull = 3,    // [2]
  kBarKEmpty = 5,   // [2] the Q K^T products that read the K stage are done
  kBarSFull = 7,    // [2] per tile
  kBarPFull = 9,    // [2] per tile
  kBarODone = 11,   // [2] per tile
  kBarPHalf = 13,   // [2] per tile: P of keys [0, 16 kPFirstSteps) written
  kBarDone = 15,    // softmax threads finished with tensor memory
  kBarVEmpty = 16,  // [2] the P V products that read the V stage are done
  kNumBars = 18
};

// Per-sequence token counts of a batch whose sequences differ in length
// (varlen = 0: every sequence fills the layout's seqlen).
constexpr int kMaxSeqs = 256;
struct SeqLens {
  int varlen;
  int n[kMaxSeqs];
};

// One 128-query tile of a work item.
struct Tile {
  int valid;  // 0: no such tile (past the item's rows or its sequence)
  int i;      // query block
  int bh;     // batch * hq + head
  int ntok;   // tokens of its sequence
  const uint32_t* mrow;  // the mask row: in global memory, then its copy in shared memory
  int last_word;
  uint32_t last_mask;
  __device__ __forceinline__ uint32_t word(int w) const {
    if (!valid || w > last_word) return 0u;
    const uint32_t b = mrow[w];
    return w == last_word ? (b & last_mask) : b;
  }
};

// Tile of query block i (< 0: none) of Q head hg (within its KV group).
__device__ __forceinline__ void make_tile(Tile& t, int i, int hg, int G, int nb, int kv_global, int hq,
                                          const uint32_t* mask, int W, int seqlen, const SeqLens& lens) {
  t.valid = i >= 0;
  t.i = t.valid ? i : 0;
  const int bi = kv_global / (hq / G);  // batch of this KV head
  t.ntok = lens.varlen ? lens.n[bi] : seqlen;
  if (t.i * 128 >= t.ntok) t.valid = 0;  // a query block past its sequence
  const int kv = kv_global - bi * (hq / G);
  const int h = kv * G + hg;
  t.bh = bi * hq + h;
  t.mrow = mask + ((size_t)t.bh * nb + t.i) * W;
  t.last_word = t.i >> 5;
  t.last_mask = ((t.i & 31) == 31) ? 0xffffffffu : ((2u << (t.i & 31)) - 1u);
}

// Walks the union of the two tiles' kept blocks in ascending order.
struct UnionIter {
  const Tile* a;
  const Tile* b;
  int w, last_word;
  uint32_t bits;
  __device__ __forceinline__ void init(const Tile* ta, const Tile* tb) {
    a = ta;
    b = tb;
    last_word = max(ta->valid ? ta->last_word : -1, tb->valid ? tb->last_word : -1);
    w = 0;
    bits = last_word >= 0 ? (a->word(0) | b->word(0)) : 0u;
  }
  // returns j or -1; sets in_a / in_b
  __device__ __forceinline__ int next(bool& in_a, bool& in_b) {
    while (bits == 0u) {
      if (++w > last_word) return -1;
      bits = a->word(w) | b->word(w);
    }
    const int bit = __ffs(bits) - 1;
    bits &= bits - 1u;
    in_a = (a->word(w) >> bit) & 1u;
    in_b = (b->word(w) >> bit) & 1u;
    return (w << 5) + bit;
  }
};

__device__ __forceinline__ int count_kept(const Tile& t) {
  if (!t.valid) return 0;
  int n = 0;
  for (int w = 0; w <= t.last_word; ++w) n += __popc(t.word(w));
  return n;
}

// S = Q K^T.  q_lo / k_lo: low words of the shared memory descriptors of the
// Q tile and the K stage (K-major, 128-byte swizzle; hi the common high
// word); the eight K steps of 16 dims move the address field (16-byte units).
__device__ __forceinline__ void mma_qk(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo, uint32_t hi) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);  // Q K-major, K K-major
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16;
    mma_bf16_ss_lo(d_tmem, q_lo + off, k_lo + off, hi, idesc, kk > 0);
  }
}

// O += P V over keys [64 part, 64 part + 64): four K steps of 16 keys
// O += P V over keys [16 k0, 16 k1): K steps of 16 keys; P in tensor memory at
// p_tmem (two bf16 per column), v_lo: low word of the V stage's descriptor
// (MN-major, 2 KB per 16 keys)
template <int K0, int K1>
__device__ __forceinline__ void mma_pv_part(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_lo, uint32_t hi,
                                            bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 1);  // P K-major (TMEM), V MN-major
#pragma unroll
  for (int kk = K0; kk < K1; ++kk)
    mma_bf16_ts_lo(o_tmem, p_tmem + kk * 8, v_lo + (uint32_t)(kk * 2048 / 16), hi, idesc,
                   (accumulate || kk > 0) ? 1u : 0u);
}

// Row max of this thread's S row held in registers; DIAG skips keys c > r.
template <bool DIAG>
__device__ __forceinline__ float row_max(const uint32_t (&sv)[128], int r) {
  if (DIAG) {
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 128; ++c) mx = (c > r) ? mx : fmaxf(mx, __uint_as_float(sv[c]));
    return mx;
  }
  float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int e = 0; e < 64; ++e)
    mc[e & 3] = max3f(mc[e & 3], __uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1]));
  return fmaxf(max3f(mc[0], mc[1], mc[2]), mc[3]);
}

// P = exp2(S * scale_log2 - m) for the key pairs [e0, e0 + ne) of this
// thread's S row (keys 2 e, 2 e + 1), two bf16 per word into pk; the fp32
// values are added into acc.  Packed f32x2 arithmetic for the scale/shift and
// the sums; four independent partial sums keep the dependency chains short.
// DIAG zeroes keys c > r (causal diagonal).
template <bool DIAG>
__device__ __forceinline__ void p_pairs(const uint32_t (&sv)[128], int e0, int ne, uint64_t sc2, uint64_t nm2, int r,
                                        uint64_t (&acc)[4], uint32_t* pk) {
#pragma unroll
  for (int e = 0; e < ne; ++e) {
    const int c = 2 * (e0 + e);
    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sc2, nm2);
    float x0, x1;
    f2_unpack(x2, x0, x1);
    float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
    if (DIAG) {
      if (c > r) p0 = 0.f;
      if (c + 1 > r) p1 = 0.f;
    }
    acc[e & 3] = f2_add(acc[e & 3], f2_pack(p0, p1));
    pk[e] = pack_bf16x2(p0, p1);
  }
}

// Writes P = exp2(S * scale_log2 - m) as bf16 over columns [0, 64) of this
// thread's S row and returns the row sum of the fp32 values.  Keys
// [0, 16 kPFirstSteps) are published on bar_first as soon as they are in
// tensor memory, so the P V product can start on them while the rest is
// computed.
template <bool DIAG>
__device__ __forceinline__ float softmax_p(const uint32_t (&sv)[128], uint32_t tS, float scale_log2, float m,
                                           int r, uint32_t bar_first) {
  static_assert(kPFirstSteps == 6, "the store shapes below assume 96 + 32 keys");
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  {
    uint32_t pk[48];
    p_pairs<DIAG>(sv, 0, 48, sc2, nm2, r, acc, pk);
    tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(pk));
    tmem_st16(tS + 32, *reinterpret_cast<const uint32_t(*)[16]>(pk + 32));
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(bar_first);
  }
  {
    uint32_t pk[16];
    p_pairs<DIAG>(sv, 48, 16, sc2, nm2, r, acc, pk);
    tmem_st16(tS + 48, pk);
  }
  const uint64_t t2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float a0, a1;
  f2_unpack(t2, a0, a1);
  return a0 + a1;
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const uint32_t* mask,
                   __nv_bfloat16* __restrict__ out, int batch, int hq, int hkv, int seqlen, int nb,
                   float scale_log2, const uint32_t* ready, int ready_rows, const __grid_constant__ SeqLens lens) {
  __shared__ int s_masks_ok;
  __shared__ uint32_t s_mask[2][kMaxMaskWords];  // the two tiles' mask rows
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + kOffBar;
  auto bar = [&](uint32_t slot) { return bars + 8u * slot; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sgen + kOffBar + 8 * kNumBars + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = hq / hkv;
  const int items_per_kv = G * ((nb + 1) >> 1);
  // KV-head-major order: the CTAs running at any time share one KV head, whose
  // K/V (2 N x 256 bytes) then stays in L2 for all its query blocks.  A CTA
  // takes two adjacent query blocks of one Q head (their kept key blocks
  // overlap most, so most steps feed both tiles), longest rows first.
  const int m = (int)(blockIdx.x % items_per_kv);
  const int kv_global = (int)(blockIdx.x / items_per_kv);
  const int W = (nb + 31) >> 5;
  const int pair = m / G, hg = m - pair * G;
  Tile tiles[2];
  make_tile(tiles[0], nb - 1 - 2 * pair, hg, G, nb, kv_global, hq, mask, W, seqlen, lens);
  make_tile(tiles[1], nb - 2 - 2 * pair, hg, G, nb, kv_global, hq, mask, W, seqlen, lens);

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < kNumBars; ++s)
      mbar_init(bar(s), (s == kBarPFull || s == kBarPFull + 1 || s == kBarPHalf || s == kBarPHalf + 1)
                            ? 128u
                            : (s == kBarDone ? 256u : 1u));
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    // launched while the estimator still runs: wait (bounded) until the
    // estimator has counted every mask row of the segments of both tiles
    int ok = 1;
    if (ready) {
      const int nseg = (nb + ready_rows - 1) / ready_rows;
      for (int x = 0; x < 2; ++x)
        if (ok && tiles[x].valid) {
          const int sg = tiles[x].i / ready_rows;
          const uint32_t rows = (uint32_t)min(ready_rows, nb - sg * ready_rows);
          ok = count_wait_ns(&ready[(size_t)tiles[x].bh * nseg + sg], rows, kWaitLimitNs) ? 1 : 0;
        }
    }
    s_masks_ok = ok;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (!s_masks_ok) tiles[0].valid = tiles[1].valid = 0;  // (timed out: error recorded, no work)
  // the tiles' mask rows, read once through L2 (they may have been written
  // during this launch), then from shared memory by every role
  for (int x = 0; x < 2; ++x)
    if (tiles[x].valid)
      for (int w = threadIdx.x; w <= tiles[x].last_word; w += kThreads) s_mask[x][w] = __ldcg(tiles[x].mrow + w);
  __syncthreads();
  tiles[0].mrow = s_mask[0];
  tiles[1].mrow = s_mask[1];
  const uint32_t tmem = *tmem_holder;
  // Each warpgroup sets its register budget first and then runs only its own
  // roles (no code is shared across the split); warp 1 frees tensor memory
  // once the 256 softmax threads are done with it.
  if (warp < 4) {
  regs_dec<kRegsLow>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int nA = count_kept(tiles[0]), nB = count_kept(tiles[1]);
      if (nA + nB > 0) {
        mbar_arrive_expect_tx(bar(kBarQ), (nA > 0 ? kTileBytes : 0) + (nB > 0 ? kTileBytes : 0));
        for (int x = 0; x < 2; ++x) {
          if ((x == 0 ? nA : nB) == 0) continue;
          const int q_tok = tiles[x].i * 128;  // rows past the sequence end read as zeros
          tma_load_3d(sbase + kOffQ + x * kTileBytes, &tmQ, 0, q_tok, tiles[x].bh, bar(kBarQ));
          tma_load_3d(sbase + kOffQ + x * kTileBytes + kHalfBytes, &tmQ, 64, q_tok, tiles[x].bh, bar(kBarQ));
        }
        UnionIter it;
        it.init(&tiles[0], &tiles[1]);
        bool ia, ib;
        for (int t = 0;; ++t) {
          const int j = it.next(ia, ib);
          if (j < 0) break;
          const int s = t & 1;
          // a K stage is refilled once the Q K^T products that read it are
          // done, a V stage once its P V products are: K(t + 1) then lands
          // about a step ahead of its first use
          if (t >= 2 && !mbar_wait(bar(kBarKEmpty + s), ((t >> 1) - 1) & 1)) break;
          const int kr = j * 128;
          const uint32_t kd = sbase + kOffK + s * kTileBytes, vd = sbase + kOffV + s * kTileBytes;
          mbar_arrive_expect_tx(bar(kBarKFull + s), kTileBytes);
          tma_load_3d(kd, &tmK, 0, kr, kv_global, bar(kBarKFull + s));
          tma_load_3d(kd + kHalfBytes, &tmK, 64, kr, kv_global, bar(kBarKFull + s));
          if (t >= 2 && !mbar_wait(bar(kBarVEmpty + s), ((t >> 1) - 1) & 1)) break;
          mbar_arrive_expect_tx(bar(kBarVFull + s), kTileBytes);
          tma_load_3d(vd, &tmV, 0, kr, kv_global, bar(kBarVFull + s));
          tma_load_3d(vd + kHalfBytes, &tmV, 64, kr, kv_global, bar(kBarVFull + s));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int nA = count_kept(tiles[0]), nB = count_kept(tiles[1]);
      if (nA + nB > 0 && mbar_wait(bar(kBarQ), 0)) {
        const uint32_t tS[2] = {tmem, tmem + 128};
        const uint32_t tO[2] = {tmem + 256, tmem + 384};
        // descriptor low words: Q tile x, K / V stage s at + x (s) * kStep
        constexpr uint32_t kStep = kTileBytes / 16;
        const uint64_t qdesc = smem_desc_sw128(sbase + kOffQ, 16, 1024);
        const uint32_t hi = (uint32_t)(qdesc >> 32);  // the same for every descriptor here
        const uint32_t qs0 = (uint32_t)qdesc;
        const uint32_t qs[2] = {qs0, qs0 + kStep};
        const uint32_t kd0 = qs0 + (kOffK - kOffQ) / 16;
        const uint32_t vd0 = (uint32_t)smem_desc_sw128(sbase + kOffV, kHalfBytes, 1024);
        int u[2] = {0, 0};  // per-tile count of P V products issued
        UnionIter it;
        it.init(&tiles[0], &tiles[1]);
        bool in_cur[2], in_nxt[2];
        int j = it.next(in_cur[0], in_cur[1]);
        bool ok = mbar_wait(bar(kBarKFull + 0), 0);
        if (ok) {
          tc_fence_after();
          for (int x = 0; x < 2; ++x)
            if (in_cur[x]) {
              mma_qk(tS[x], qs[x], kd0, hi);
              mma_commit(bar(kBarSFull + x));
            }
          mma_commit(bar(kBarKEmpty + 0));
        }
        for (int t = 0; ok && j >= 0; ++t) {
          const int s = t & 1;
          const int jn = it.next(in_nxt[0], in_nxt[1]);
          bool k_ready = false;
          // a tile that skips step t but takes step t + 1 gets its Q K^T right
          // away if K(t + 1) has landed (no wait here), so its softmax runs
          // beside this step's; else in its place below
          const uint32_t late =
              jn >= 0 ? ((in_nxt[0] && !in_cur[0]) ? 1u : 0u) | ((in_nxt[1] && !in_cur[1]) ? 2u : 0u) : 0u;
          uint32_t early = 0;
          if (late && mbar_test_wait(bar(kBarKFull + (s ^ 1)), ((t + 1) >> 1) & 1)) {
            tc_fence_after();
            k_ready = true;
            early = late;
#pragma unroll 1
            for (int x = 0; x < 2; ++x)
              if ((late >> x) & 1u) {
                mma_qk(tmem + 128 * x, qs0 + x * kStep, kd0 + (s ^ 1) * kStep, hi);
                mma_commit(bar(kBarSFull + x));
              }
          }
          if (!(ok = mbar_wait(bar(kBarVFull + s), (t >> 1) & 1))) break;
          for (int x = 0; x < 2; ++x) {
            if (in_cur[x]) {
              if (!(ok = mbar_wait(bar(kBarPHalf + x), u[x] & 1))) break;
              tc_fence_after();
              mma_pv_part<0, kPFirstSteps>(tO[x], tS[x], vd0 + s * kStep, hi, u[x] > 0);
              if (!(ok = mbar_wait(bar(kBarPFull + x), u[x] & 1))) break;
              tc_fence_after();
              mma_pv_part<kPFirstSteps, 8>(tO[x], tS[x], vd0 + s * kStep, hi, true);
              mma_commit(bar(kBarODone + x));
              ++u[x];
            }
            if (jn >= 0 && in_nxt[x] && !((early >> x) & 1u)) {
              if (!k_ready) {
                if (!(ok = mbar_wait(bar(kBarKFull + (s ^ 1)), ((t + 1) >> 1) & 1))) break;
                tc_fence_after();
                k_ready = true;
              }
              mma_qk(tS[x], qs[x], kd0 + (s ^ 1) * kStep, hi);
              mma_commit(bar(kBarSFull + x));
            }
          }
          if (!ok) break;
          mma_commit(bar(kBarVEmpty + s));
          if (jn >= 0) mma_commit(bar(kBarKEmpty + (s ^ 1)));
          j = jn;
          in_cur[0] = in_nxt[0];
          in_cur[1] = in_nxt[1];
        }
      }
    }
    __syncwarp();
    mbar_wait(bar(kBarDone), 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  return;
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ softmax
    const int x = (warp - 4) >> 2;          // tile
    const int qw = warp & 3;                // TMEM lane quarter of this warp
    const int r = qw * 32 + lane;           // query row == TMEM lane
    const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
    const uint32_t tS = tmem + 128 * x + lane_base;
    const uint32_t tO = tmem + 256 + 128 * x + lane_base;
    const Tile& T = tiles[x];
    const int n = count_kept(T);
    bool ok = true;
    float m_run = -INFINITY, l_run = 0.f;
    int w = 0;
    uint32_t bits = T.word(0);
    for (int u = 0; u < n; ++u) {
      while (bits == 0u) bits = T.word(++w);
      const int j = (w << 5) + __ffs(bits) - 1;
      bits &= bits - 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarSFull + x), u & 1));
      if (!ok) break;
      tc_fence_after();
      // the S row (128 fp32) into registers, one tensor-memory round trip
      const bool diag = (j == T.i);
      uint32_t sv[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(sv + 64));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(sv + 96));
      tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(sv + 0));
      tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(sv + 64));
      tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(sv + 96));
      // row max (diagonal block: keys c <= r only)
      float mx = diag ? row_max<true>(sv, r) : row_max<false>(sv, r);
      mx *= scale_log2;
      // lazy rescale: move the reference max only when it grows by > threshold
      const bool grow = (u == 0) || (mx > m_run + kRescaleThreshold);
      const float m_new = grow ? fmaxf(mx, m_run) : m_run;
      if (u > 0) {
        // P V of the previous step must finish before O is touched or P rewritten
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarODone + x), (u - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
          const float alpha = grow ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t v[32];
            tmem_ld32(tO + c4 * 32, v);
            tmem_wait_ld_dep(v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(tO + c4 * 32, v);
          }
          l_run *= alpha;
        }
      }
      m_run = m_new;
      // pass 2 over S: P = exp2(S * scale - m) in bf16, written over S[:, 0:64)
      const float rs = diag ? softmax_p<true>(sv, tS, scale_log2, m_run, r, bar(kBarPHalf + x))
                            : softmax_p<false>(sv, tS, scale_log2, m_run, r, bar(kBarPHalf + x));
      l_run += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + x));
    }
    // ------------------------------------------------------------ epilogue
    // query rows past the end of a short last block are computed but not stored
    const bool row_ok = T.valid && T.i * 128 + r < T.ntok;
    __nv_bfloat16* orow = row_ok ? out + ((size_t)T.bh * seqlen + (size_t)T.i * 128 + r) * 128 : nullptr;
    if (T.valid && n == 0) {  // (warp-uniform branches: the loads below are warp-collective)
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      if (row_ok)
#pragma unroll
        for (int c = 0; c < 16; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
    } else if (T.valid && ok && __all_sync(0xffffffffu, mbar_wait(bar(kBarODone + x), (n - 1) & 1))) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t v[32];
        tmem_ld32(tO + c4 * 32, v);
        tmem_wait_ld_dep(v);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 pk;
          pk.x = pack_bf16x2(__uint_as_float(v[q4 * 8 + 0]) * inv, __uint_as_float(v[q4 * 8 + 1]) * inv);
          pk.y = pack_bf16x2(__uint_as_float(v[q4 * 8 + 2]) * inv, __uint_as_float(v[q4 * 8 + 3]) * inv);
          pk.z = pack_bf16x2(__uint_as_float(v[q4 * 8 + 4]) * inv, __uint_as_float(v[q4 * 8 + 5]) * inv);
          pk.w = pack_bf16x2(__uint_as_float(v[q4 * 8 + 6]) * inv, __uint_as_float(v[q4 * 8 + 7]) * inv);
          if (row_ok) reinterpret_cast<uint4*>(orow)[c4 * 4 + q4] = pk;
        }
      }
    }
    tc_fence_before();
    mbar_arrive(bar(kBarDone));
  }
}

// Number of work items (CTAs) for a problem.
__host__ __forceinline__ unsigned grid_size(int batch, int hq, int hkv, int nb) {
  const int G = hq / hkv;
  return (unsigned)batch * hkv * (unsigned)(G * ((nb + 1) / 2));
}

}  // namespace attn
}  // namespace prism
