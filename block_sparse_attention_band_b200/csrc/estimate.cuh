// Prism block-importance estimator, steps (1)-(7) of the method paragraph of
// the paper.rainbus.top review of "Prism: Spectral-Aware Block-Sparse
// Attention": band slicing, mean pooling per block of B = 128 tokens, RMS of
// each pooled band, temperatures tau_z, dual-band pooled softmax, Top-P per
// query-block row and band, union of the two masks.
//
// One persistent kernel.  CTAs take work items from a device queue in a fixed
// order that interleaves the two kinds of work per KV group g (the Q heads
// that share one KV head):
//
//   pool(0), pool(1), score(0), pool(2), score(1), ..., pool(n-1), score(n-2), score(n-1)
//
// pool items (HBM-bound) stream 128x128 bf16 tiles of Q and K once (bulk
// copies into a ring of shared-memory stages, several tiles in flight) and write
// the fp32 block means (steps 1-2) and per-block energy partials (step 3);
// the CTA that finishes the last pool item of a group also computes the
// group's temperatures (steps 3-4) and publishes "group ready".  score items
// (ALU-bound) wait for their group, compute both bands' pooled logits with an
// fp32 register-tiled product (step 5) and run softmax + Top-P + union per
// row (steps 5-7).  Scoring of group g overlaps pooling of group g+1.  An
// item only ever waits for items earlier in the queue, which running CTAs
// hold and which never wait, so the schedule cannot deadlock; the wait is
// bounded all the same.
//
// Band slicing is folded into the pooled layout: the pool items write the 128
// pooled dims in a permuted order [high-only | both | low-only | neither], so
// each band is a contiguous column range: high = [0, s2), low = [s1, s3).
#pragma once
#include "ptx.cuh"

namespace prism {

struct BandLayout {
  uint8_t perm[128];  // pooled column c holds original dim perm[c]
  int s1, s2, s3;     // segment boundaries (see above)
  int d_hi, d_lo;     // band sizes
};

constexpr int kEstThreads = 512;      // 16 warps, one CTA per SM
constexpr int kPoolTilesPerItem = 8;  // 8 x 32 KB of Q or K per pool item
constexpr uint32_t kTileBytes = 128 * 128 * 2;
constexpr int kMaxPoolStages = 6;     // bulk-copy ring depth (32 KB stages)
constexpr int kScoreRows = 64;        // (head, query block) rows per score item
constexpr int kColTile = 128;         // key blocks per product column tile
constexpr int kStageLD = kColTile + 1;
constexpr int kGemmSmemBytes = (128 * kScoreRows + 128 * kColTile + 2 * kScoreRows * kStageLD + 2 * kScoreRows) * 4;
constexpr int kMaxGroupHeads = 64;    // Q heads per KV head supported by the tau step
constexpr float kLog2e = 1.4426950408889634f;

struct EstParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  float* pool;    // [q_rows + kv_rows, nb, 128] band-ordered means
  float* part;    // [q_rows + kv_rows, nb, 4] sum(mean^2): hi, lo, all
  float* tau;     // [q_rows, 4]: tau_hi, tau_lo, 1/(tau_hi sqrt d_hi), 1/(tau_lo sqrt d_lo)
  float* scores;  // [q_rows, 2, nb(nb+1)/2] scaled band logits, packed rows
  uint32_t* mask;
  float* dbg_tau;
  uint32_t* sync;  // [0] queue head, [1 + g] pool items done, [1 + n_groups + g] group ready
  int hq, hkv, G, nb, W, q_rows, n_groups;
  int pool_items;      // per group
  int score_items;     // per group
  int pool_item_span;  // pool items per head row
  int topp_warps;
  int topp_stride;  // bytes of shared memory per Top-P warp
  int pool_stages;  // bulk-copy ring depth (<= kMaxPoolStages)
  float p;
  int explicit_tau;
  float tau_hi, tau_lo;
  BandLayout bl;
};

// ---------------------------------------------------------------------------
// warp / ordering helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// steps (1)-(3a): mean of one 128 x 128 bf16 tile, band-ordered fp32 write,
// energy partials.  Thread t holds 16-byte vectors of rows t/16 + 16 r at
// dims 8 (t % 16) .. +7: each warp reads two full 256-byte rows.
// ---------------------------------------------------------------------------
struct PoolSmem {
  float red[16][128];
  float mean[128];
  float wsum[4][3];
  float sums[kMaxGroupHeads + 1][3];
  uint64_t bars[kMaxPoolStages];
  int flag;
};

// Reduces one tile held in shared memory (128 rows x 256 bytes): thread t
// sums the 16 rows 8k + t/64 of the bf16 pair in 32-bit word t % 64
// (conflict-free), the 8 row groups are combined in a fixed order.  `refill`
// runs once every thread has read the stage (it may overwrite it).
template <class Refill>
__device__ __forceinline__ void pool_tile(const uint32_t* tile, const EstParams& P, int hr, int blk, PoolSmem& sm,
                                          Refill refill) {
  const int t = threadIdx.x;
  const int pw = t & 63, rg = t >> 6;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t w = tile[(rg + 8 * k) * 64 + pw];
    a0 += bf16lo(w);
    a1 += bf16hi(w);
  }
  sm.red[rg][2 * pw] = a0;
  sm.red[rg][2 * pw + 1] = a1;
  __syncthreads();
  refill();
  if (t < 128) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) s += sm.red[g][t];
    sm.mean[t] = s * (1.0f / 128.0f);
  }
  __syncthreads();
  if (t < 128) {
    const float m = sm.mean[P.bl.perm[t]];
    P.pool[((size_t)hr * P.nb + blk) * 128 + t] = m;
    const float sq = m * m;
    float hi = t < P.bl.s2 ? sq : 0.f;
    float lo = (t >= P.bl.s1 && t < P.bl.s3) ? sq : 0.f;
    float all = sq;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      hi += __shfl_xor_sync(0xffffffffu, hi, o);
      lo += __shfl_xor_sync(0xffffffffu, lo, o);
      all += __shfl_xor_sync(0xffffffffu, all, o);
    }
    if ((t & 31) == 0) {
      sm.wsum[t >> 5][0] = hi;
      sm.wsum[t >> 5][1] = lo;
      sm.wsum[t >> 5][2] = all;
    }
  }
  __syncthreads();
  if (t < 3)
    P.part[((size_t)hr * P.nb + blk) * 4 + t] =
        (sm.wsum[0][t] + sm.wsum[1][t]) + (sm.wsum[2][t] + sm.wsum[3][t]);
}

// steps (3b)-(4): RMS of every pooled band of the group's heads over all
// blocks and the temperatures of its Q heads (reading R1 of the pages: the
// band's pooled Q x K energy relative to the full spectrum's).
__device__ void group_temperatures(const EstParams& P, int g, PoolSmem& sm) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int bi = g / P.hkv, kv = g - bi * P.hkv;
  for (int slot = 0; slot <= P.G; ++slot) {  // slots 0..G-1: Q heads, G: the KV head
    const int hr = slot < P.G ? bi * P.hq + kv * P.G + slot : P.q_rows + g;
    float s[3] = {0.f, 0.f, 0.f};
    for (int i = t; i < P.nb; i += kEstThreads) {
      const float* pp = P.part + ((size_t)hr * P.nb + i) * 4;
      s[0] += pp[0];
      s[1] += pp[1];
      s[2] += pp[2];
    }
#pragma unroll
    for (int e = 0; e < 3; ++e) s[e] = warp_sum(s[e]);
    if (lane == 0)
#pragma unroll
      for (int e = 0; e < 3; ++e) sm.red[warp][e] = s[e];
    __syncthreads();
    if (t < 3) {
      float a = 0.f;
      for (int w = 0; w < kEstThreads / 32; ++w) a += sm.red[w][t];
      sm.sums[slot][t] = a;
    }
    __syncthreads();
  }
  if (t < P.G) {
    const int row = bi * P.hq + kv * P.G + t;
    float th, tl;
    if (P.explicit_tau) {
      th = P.tau_hi;
      tl = P.tau_lo;
    } else {
      const float n = (float)P.nb;
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
// group (its Q heads, then its KV head), the next tile's loads in flight
// while the current one is reduced.
__device__ void pool_item(const EstParams& P, int g, int y, PoolSmem& sm, unsigned char* ring, int stages,
                          uint32_t& phases) {
  const int slot = y / P.pool_item_span;
  const int blk0 = (y - slot * P.pool_item_span) * kPoolTilesPerItem;
  const int blk1 = min(blk0 + kPoolTilesPerItem, P.nb);
  const int bi = g / P.hkv, kv = g - bi * P.hkv;
  int hr;
  const __nv_bfloat16* base;
  if (slot < P.G) {
    hr = bi * P.hq + kv * P.G + slot;
    base = P.q + (size_t)hr * P.nb * (128 * 128);
  } else {
    hr = P.q_rows + g;
    base = P.k + (size_t)g * P.nb * (128 * 128);
  }
  // bulk-copy ring: up to `stages` tiles in flight, each stage refilled with
  // the tile `stages` ahead as soon as every thread has read it
  const int nt = blk1 - blk0;
  const uint32_t ring0 = smem_u32(ring);
  auto issue = [&](int tt) {
    const int slot = tt % stages;
    const uint32_t bar = smem_u32(&sm.bars[slot]);
    mbar_arrive_expect_tx(bar, kTileBytes);
    bulk_load(ring0 + slot * kTileBytes, base + (size_t)(blk0 + tt) * (128 * 128), kTileBytes, bar);
  };
  if (threadIdx.x == 0)
    for (int tt = 0; tt < min(stages, nt); ++tt) issue(tt);
  for (int tt = 0; tt < nt; ++tt) {
    const int slot = tt % stages;
    mbar_wait(smem_u32(&sm.bars[slot]), (phases >> slot) & 1u);  // a timeout is recorded on the device
    phases ^= 1u << slot;
    pool_tile(reinterpret_cast<const uint32_t*>(ring + (size_t)slot * kTileBytes), P, hr, blk0 + tt, sm, [&] {
      if (threadIdx.x == 0 && tt + stages < nt) {
        fence_proxy_async_smem();
        issue(tt + stages);
      }
    });
  }
  // publish: count the item; the CTA that completes the group computes tau
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t done = atomicAdd(&P.sync[1 + g], 1u);
    sm.flag = (done == (uint32_t)P.pool_items - 1u);
    if (sm.flag) __threadfence();
  }
  __syncthreads();
  if (sm.flag) {
    group_temperatures(P, g, sm);
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      st_release_gpu(&P.sync[1 + P.n_groups + g], 1u);
    }
  }
}

// ---------------------------------------------------------------------------
// step (6): exact Top-P of one band row
// ---------------------------------------------------------------------------
// Shared-memory scratch of one Top-P warp.
struct ToppScratch {
  uint32_t* d;            // [n] logits, then the rank keys d_j (below)
  float* L2;              // [n] the second band's logits, loaded with the first
  uint16_t* cand;         // [n] members of the crossing bin
  unsigned long long* h;  // [256] bin masses
  uint32_t* kb;           // [W] blocks of bins before the crossing bin
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

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exact crossing among `cnt` members (<= 32) listed in S.cand, all ranked
// behind mass `base`: returns the member c with ahead(c) < target <=
// ahead(c) + e_c, or -1 if none reaches the target.  The members are sorted
// across the warp by (d, j) with a bitonic network, then an inclusive scan of
// their masses in that order finds the crossing.
__device__ __forceinline__ int topp_exact32(const ToppScratch& S, int cnt, unsigned long long base,
                                            unsigned long long target, int lane) {
  unsigned long long key = ~0ull;  // (d << 32) | j; absent members sort last
  if (lane < cnt) {
    const int j = S.cand[lane];
    key = ((unsigned long long)S.d[j] << 32) | (uint32_t)j;
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

// 64-bit bin mass kept as two 32-bit words: the low word's atomic add returns
// the old value, and an add that wraps it carries one into the high word, so
// the final sum is exact and independent of the order of the adds.
__device__ __forceinline__ void bin_add(uint32_t* lo, uint32_t* hi, int b, uint32_t x) {
  const uint32_t old = atomicAdd(&lo[b], x);
  if (old > ~x) atomicAdd(&hi[b], 1u);
}

// Softmax (step 5) + Top-P (step 6) of one band row of n scaled logits held
// in shared memory; ORs the kept blocks into bits[].
//
// e_j = 2^((L_j - max) log2 e); blocks ranked by (-e_j, j) == (d_j, j) with
// the exact order-reversing key d_j.  Radix selection on the keys: bins of 16
// per octave of e (bin = d >> 19, the last one collecting everything below
// 2^-14) hold their mass exactly (e_j in 2^-31 fixed point, 64-bit exact
// sums), so one scan gives Z, the crossing bin and the mass ranked before it
// as exact integers.  Blocks of earlier bins are kept, of later bins dropped;
// the crossing bin's members are ranked exactly (pairwise when <= 32, else by
// refining on the lower key bits the same way).  A block is kept iff the
// mass ranked strictly ahead of it is < p Z.
__device__ void topp_band_row(const float* Lsm, int n, int W, float p, const ToppScratch& S, uint32_t* bits,
                              int lane) {
  const unsigned lt = (1u << lane) - 1u;
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 4
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    if (j < n) mx[(j0 >> 5) & 3] = fmaxf(mx[(j0 >> 5) & 3], Lsm[j]);
  }
  const int nw = (n + 31) >> 5;
  if (p >= 1.0f) {  // every causal block is kept
    for (int w = lane; w < nw; w += 32) {
      const int lo = w * 32;
      bits[w] |= lo + 32 <= n ? 0xffffffffu : ((1u << (n - lo)) - 1u);
    }
    __syncwarp();
    return;
  }
  const float m = warp_max(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]))) * kLog2e;
  uint32_t* hlo = reinterpret_cast<uint32_t*>(S.h);
  uint32_t* hhi = hlo + kTopPBins;
  for (int b = lane; b < kTopPBins; b += 32) {
    hlo[b] = 0u;
    hhi[b] = 0u;
  }
  __syncwarp();
  // e_j, keys, exact bin masses
#pragma unroll 4
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    if (j < n) {
      const float e = fast_exp2(fmaf(Lsm[j], kLog2e, -m));
      const uint32_t d = rank_key(e);
      S.d[j] = d;
      bin_add(hlo, hhi, (int)min(d >> 19, (uint32_t)(kTopPBins - 1)), fixmass(e));
    }
  }
  __syncwarp();
  unsigned long long hv[8], tot = 0ull;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    hv[u] = ((unsigned long long)hhi[lane * 8 + u] << 32) | hlo[lane * 8 + u];
    tot += hv[u];
  }
  unsigned long long incl = warp_scan_u64(tot, lane);
  const unsigned long long Z = __shfl_sync(0xffffffffu, incl, 31);
  const unsigned long long target = (unsigned long long)((double)p * (double)Z);
  // crossing bin: the first with (mass before it + its mass) >= target
  int xb;
  unsigned long long base;
  {
    unsigned long long run = incl - tot;
    int bin = -1;
    unsigned long long bb = 0ull;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (bin < 0 && run + hv[u] >= target && hv[u] > 0ull) {
        bin = lane * 8 + u;
        bb = run;
      }
      run += hv[u];
    }
    const unsigned found = __ballot_sync(0xffffffffu, bin >= 0);
    const int sl = found ? __ffs(found) - 1 : 31;
    xb = found ? __shfl_sync(0xffffffffu, bin, sl) : kTopPBins - 1;
    base = found ? __shfl_sync(0xffffffffu, bb, sl) : Z;
  }
  // one pass: keep the earlier bins, list the crossing bin's members
  int cnt = 0;
#pragma unroll 2
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    bool before = false, in = false;
    if (j < n) {
      const int b = (int)min(S.d[j] >> 19, (uint32_t)(kTopPBins - 1));
      before = b < xb;
      in = b == xb;
    }
    const unsigned mb = __ballot_sync(0xffffffffu, before), mi = __ballot_sync(0xffffffffu, in);
    if (in) S.cand[cnt + __popc(mi & lt)] = (uint16_t)j;
    cnt += __popc(mi);
    if (lane == 0) bits[j0 >> 5] |= mb;
  }
  __syncwarp();
  // rank the crossing bin's members
  int cross = -1;
  bool refined = false;
  if (cnt <= 32) {
    cross = topp_exact32(S, cnt, base, target, lane);
  } else {
    // refine on lower key bits, 8-bit digits: a regular bin spans 2^19 keys
    // (digits at shifts 11, 3, 0), the catch-all bin up to 2^30 (22, 14, 6, 0)
    refined = true;
    uint32_t lo_key = (uint32_t)xb << 19;
    const bool wide = xb == kTopPBins - 1;
    for (int level = 0;; ++level) {
      const int sh = wide ? (level == 0 ? 22 : level == 1 ? 14 : level == 2 ? 6 : 0)
                          : (level == 0 ? 11 : level == 1 ? 3 : 0);
      for (int b = lane; b < kTopPBins; b += 32) {
        hlo[b] = 0u;
        hhi[b] = 0u;
      }
      __syncwarp();
      for (int x0 = 0; x0 < cnt; x0 += 32) {
        const int x = x0 + lane;
        if (x < cnt) {
          const uint32_t d = S.d[S.cand[x]];
          bin_add(hlo, hhi, (int)min((d - lo_key) >> sh, (uint32_t)(kTopPBins - 1)), fixmass(key_value(d)));
        }
      }
      __syncwarp();
      unsigned long long h2[8], t2 = 0ull;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        h2[u] = ((unsigned long long)hhi[lane * 8 + u] << 32) | hlo[lane * 8 + u];
        t2 += h2[u];
      }
      const unsigned long long inc2 = warp_scan_u64(t2, lane);
      unsigned long long run = inc2 - t2;
      int bin2 = -1;
      unsigned long long bb = 0ull;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (bin2 < 0 && base + run + h2[u] >= target && h2[u] > 0ull) {
          bin2 = lane * 8 + u;
          bb = base + run;
        }
        run += h2[u];
      }
      const unsigned f2 = __ballot_sync(0xffffffffu, bin2 >= 0);
      if (f2 == 0u) {
        // (exact sums make this unreachable) the members' mass stays below
        // the target: all of them are kept -- the cut is the last member
        uint32_t bd = 0u;
        int bj = -1;
        for (int x = lane; x < cnt; x += 32) {
          const int jj = S.cand[x];
          const uint32_t dd = S.d[jj];
          if (bj < 0 || dd > bd || (dd == bd && jj > bj)) {
            bd = dd;
            bj = jj;
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
      const uint32_t blo = lo_key + ((uint32_t)xb2 << sh);
      const uint32_t bhi = sh == 0 ? blo : blo + ((1u << sh) - 1u);
      int c2 = 0;
      for (int x0 = 0; x0 < cnt; x0 += 32) {
        const int x = x0 + lane;
        int jj = 0;
        bool in = false;
        if (x < cnt) {
          jj = S.cand[x];
          const uint32_t d = S.d[jj];
          in = d >= blo && d <= bhi;
        }
        const unsigned mk = __ballot_sync(0xffffffffu, in);
        __syncwarp();
        if (in) S.cand[c2 + __popc(mk & lt)] = (uint16_t)jj;
        c2 += __popc(mk);
      }
      __syncwarp();
      cnt = c2;
      lo_key = blo;
      if (cnt <= 32) {
        cross = topp_exact32(S, cnt, base, target, lane);
        break;
      }
      if (sh == 0) {
        // equal keys: the first member (by index) whose cumulative mass
        // reaches the target
        const unsigned long long me = (unsigned long long)fixmass(key_value(blo));
        unsigned long long acc = base;
        for (int x0 = 0; x0 < cnt && cross < 0; x0 += 32) {
          const int x = x0 + lane;
          const bool ok = x < cnt;
          const unsigned mk = __ballot_sync(0xffffffffu, ok);
          const int pos = __popc(mk & lt);
          const bool hit = ok && acc + me * (unsigned long long)(pos + 1) >= target;
          const unsigned hm = __ballot_sync(0xffffffffu, hit);
          if (hm) cross = __shfl_sync(0xffffffffu, ok ? (int)S.cand[x] : 0, __ffs(hm) - 1);
          acc += me * (unsigned long long)__popc(mk);
        }
        break;
      }
    }
  }
  __syncwarp();
  if (!refined) {
    // the crossing bin's members ranked at or ahead of the crossing
    const uint32_t dc = cross >= 0 ? S.d[cross] : 0u;
    if (lane < cnt) {
      const int j = S.cand[lane];
      const uint32_t d = S.d[j];
      if (cross < 0 || d < dc || (d == dc && j <= cross)) atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
  } else {
    // general case: every block ranked at or ahead of the crossing
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
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// score item: kScoreRows (head, query block) rows of one group, enumerated
// from the last query block down and over the group's heads; the rows share
// the group's pooled K.  Step (5) logits for j <= i with an fp32 4x4
// register tile per thread (the dims accumulate segment by segment so the
// two bands share the products of their common dims), then steps (5)-(7)
// per row.
// ---------------------------------------------------------------------------
__device__ void score_item(const EstParams& P, int g, int y, unsigned char* smem) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int bi = g / P.hkv, kv = g - bi * P.hkv;
  const int rows_total = P.G * P.nb;
  const int idx0 = y * kScoreRows;
  float* qT = reinterpret_cast<float*>(smem);      // [128 dims][64 rows]
  float* kT = qT + 128 * kScoreRows;               // [128 dims][128 cols]
  float* stage = kT + 128 * kColTile;              // [2][64][129]
  float* scl = stage + 2 * kScoreRows * kStageLD;  // [64][2]
  const size_t tri = (size_t)P.nb * (P.nb + 1) / 2;
  const float* kbase = P.pool + (size_t)(P.q_rows + g) * P.nb * 128;
  const int max_i = P.nb - 1 - idx0 / P.G;

  // rows of this item: r -> (head h, block i); false past the group's end
  auto row_of = [&](int r, int& bh, int& i) -> bool {
    const int idx = idx0 + r;
    if (idx >= rows_total) return false;
    bh = bi * P.hq + kv * P.G + idx % P.G;
    i = P.nb - 1 - idx / P.G;
    return true;
  };

  if (t < kScoreRows) {
    int bh, i;
    if (row_of(t, bh, i)) {
      scl[2 * t] = P.tau[bh * 4 + 2];
      scl[2 * t + 1] = P.tau[bh * 4 + 3];
    } else {
      scl[2 * t] = scl[2 * t + 1] = 0.f;
    }
  }
  // Qbar rows, transposed: lane -> row, warp -> 4-dim chunks
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int r = rr * 32 + lane;
    int bh = 0, i = 0;
    const bool ok = row_of(r, bh, i);
    const float* src = P.pool + ((size_t)bh * P.nb + i) * 128;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int c = warp + 16 * cc;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ok) a = *reinterpret_cast<const float4*>(src + 4 * c);
      qT[(4 * c + 0) * kScoreRows + r] = a.x;
      qT[(4 * c + 1) * kScoreRows + r] = a.y;
      qT[(4 * c + 2) * kScoreRows + r] = a.z;
      qT[(4 * c + 3) * kScoreRows + r] = a.w;
    }
  }
  const int ty = t >> 5, tx = t & 31;  // 16 x 32 threads, 4 x 4 outputs each
  for (int j0 = 0; j0 <= max_i; j0 += kColTile) {
    __syncthreads();  // the previous tile's kT and stage reads are done
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = rr * 32 + lane;
      const bool ok = j0 + r <= max_i;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = warp + 16 * cc;
        float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ok) b = *reinterpret_cast<const float4*>(kbase + (size_t)(j0 + r) * 128 + 4 * c);
        kT[(4 * c + 0) * kColTile + r] = b.x;
        kT[(4 * c + 1) * kColTile + r] = b.y;
        kT[(4 * c + 2) * kColTile + r] = b.z;
        kT[(4 * c + 3) * kColTile + r] = b.w;
      }
    }
    __syncthreads();
    float a[4][4], b[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) a[u][w] = b[u][w] = 0.f;
    auto fma_range = [&](float(&acc)[4][4], int d0, int d1) {
#pragma unroll 4
      for (int d = d0; d < d1; ++d) {
        const float4 qa = *reinterpret_cast<const float4*>(&qT[d * kScoreRows + 4 * ty]);
        const float4 kb = *reinterpret_cast<const float4*>(&kT[d * kColTile + 4 * tx]);
        const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
        const float kvv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(qv[u], kvv[w], acc[u][w]);
      }
    };
    fma_range(a, 0, P.bl.s1);        // high-only dims
    fma_range(b, P.bl.s1, P.bl.s2);  // dims of both bands
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) a[u][w] += b[u][w];  // a = high band
    fma_range(b, P.bl.s2, P.bl.s3);  // b = low band
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int row = 4 * ty + u;
      const float sh = scl[2 * row], sl = scl[2 * row + 1];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        stage[row * kStageLD + 4 * tx + w] = a[u][w] * sh;
        stage[kScoreRows * kStageLD + row * kStageLD + 4 * tx + w] = b[u][w] * sl;
      }
    }
    __syncthreads();
    for (int r = warp; r < kScoreRows; r += kEstThreads / 32) {
      int bh, i;
      if (!row_of(r, bh, i)) continue;
      float* out_hi = P.scores + (size_t)bh * 2 * tri + (size_t)i * (i + 1) / 2;
      float* out_lo = out_hi + tri;
      for (int c = lane; c < kColTile; c += 32) {
        const int jj = j0 + c;
        if (jj <= i) {
          out_hi[jj] = stage[r * kStageLD + c];
          out_lo[jj] = stage[kScoreRows * kStageLD + r * kStageLD + c];
        }
      }
    }
  }
  __syncthreads();  // this CTA's score rows are visible to all its threads

  // steps (5)-(7): one warp per row, both bands, union, whole mask row
  if (warp < P.topp_warps) {
    unsigned char* wb = smem + (size_t)warp * P.topp_stride;
    const int nbp = (P.nb + 7) & ~7;
    ToppScratch S;
    S.d = reinterpret_cast<uint32_t*>(wb);
    S.L2 = reinterpret_cast<float*>(wb + (size_t)nbp * 4);
    S.cand = reinterpret_cast<uint16_t*>(wb + (size_t)nbp * 8);
    S.h = reinterpret_cast<unsigned long long*>(wb + (size_t)nbp * 10);
    S.kb = reinterpret_cast<uint32_t*>(wb + (size_t)nbp * 10 + kTopPBins * 8);
    uint32_t* bits = S.kb + P.W;
    for (int r = warp; r < kScoreRows; r += P.topp_warps) {
      int bh, i;
      if (!row_of(r, bh, i)) continue;
      for (int w = lane; w < P.W; w += 32) bits[w] = 0u;
      __syncwarp();
      // both bands' rows -> shared memory in one round trip (32 loads in flight per lane)
      const float* row_hi = P.scores + (size_t)bh * 2 * tri + (size_t)i * (i + 1) / 2;
      const float* row_lo = row_hi + tri;
      const int n = i + 1;
      float* Lhi = reinterpret_cast<float*>(S.d);
      for (int j0 = 0; j0 < n; j0 += 512) {
        float xh[16], xl[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j = j0 + u * 32 + lane;
          xh[u] = j < n ? row_hi[j] : 0.f;
          xl[u] = j < n ? row_lo[j] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j = j0 + u * 32 + lane;
          if (j < n) {
            Lhi[j] = xh[u];
            S.L2[j] = xl[u];
          }
        }
      }
      __syncwarp();
      topp_band_row(Lhi, n, P.W, P.p, S, bits, lane);
      topp_band_row(S.L2, n, P.W, P.p, S, bits, lane);
      uint32_t* dst = P.mask + ((size_t)bh * P.nb + i) * P.W;
      for (int w = lane; w < P.W; w += 32) dst[w] = bits[w];
      __syncwarp();
    }
  }
  __syncthreads();  // shared memory is reused by the next item
}

// ---------------------------------------------------------------------------
// the persistent kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kEstThreads)
estimator_kernel(const __grid_constant__ EstParams P) {
  extern __shared__ __align__(16) unsigned char est_smem[];
  __shared__ PoolSmem psm;
  __shared__ int s_item;
  __shared__ int s_ok;
  const int per_pair = P.pool_items + P.score_items;
  const int stages = P.pool_stages;
  uint32_t phases = 0u;  // parity to wait for next, one bit per ring stage
  if (threadIdx.x == 0) {
    for (int st = 0; st < stages; ++st) mbar_init(smem_u32(&psm.bars[st]), 1u);
    fence_mbar_init();
  }
  __syncthreads();
  const int total = P.n_groups * per_pair;
  for (;;) {
    if (threadIdx.x == 0) s_item = (int)atomicAdd(&P.sync[0], 1u);
    __syncthreads();
    const int x = s_item;
    __syncthreads();
    if (x >= total) return;
    // queue order: pool(0), then pairs (pool(g+1), score(g)), last pair score(n-1) only
    int g, y;
    bool is_pool;
    if (x < P.pool_items) {
      is_pool = true;
      g = 0;
      y = x;
    } else {
      const int x2 = x - P.pool_items;
      const int pair = x2 / per_pair;
      const int rem = x2 - pair * per_pair;
      if (pair < P.n_groups - 1 && rem < P.pool_items) {
        is_pool = true;
        g = pair + 1;
        y = rem;
      } else {
        is_pool = false;
        g = pair;
        y = pair < P.n_groups - 1 ? rem - P.pool_items : rem;
      }
    }
    if (is_pool) {
      pool_item(P, g, y, psm, est_smem, stages, phases);
      continue;
    }
    // wait until the group's pooling and temperatures are published
    if (threadIdx.x == 0) {
      const uint32_t* ready = &P.sync[1 + P.n_groups + g];
      int ok = 1;
      if (ld_acquire_gpu(ready) == 0u) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(ready) == 0u) {
          if (globaltimer_ns() - t0 > 2000000000ull) {
            set_device_error(kDevErrTimeout);
            ok = 0;
            break;
          }
        }
      }
      s_ok = ok;
    }
    __syncthreads();
    if (s_ok) score_item(P, g, y, est_smem);
    __syncthreads();
  }
}

}  // namespace prism
