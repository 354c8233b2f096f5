// Causal block-sparse attention prefill on the 5th-generation tensor cores.
//
// "Prism: Spectral-Aware Block-Sparse Attention", gist.science Technical
// Summary section 1: block-sparse attention computes only a subset of the
// attention blocks; here the subset is the estimator's mask M (one bit per
// (query block i, key block j)), token-causal inside the diagonal block.
//
// One CTA per (batch, Q head, query block i) of 128 queries, 192 threads:
//   warp 5        TMA producer: Q once, then K_j / V_j of every kept block j
//                 into a 2-stage ring (128-byte swizzled, 2 x 16 KB halves)
//   warp 4        MMA issuer (one thread): S = Q K_j^T, then O += P V_j,
//                 tcgen05.mma kind::f16 (bf16 in, fp32 accumulate in tensor
//                 memory: S in columns 0-127, O in columns 128-255)
//   warps 0-3     softmax: thread r owns query row r (tensor-memory lane r),
//                 reads its S row, keeps the running max / sum (base-2
//                 exponent), rescales its O row when the max grows, writes
//                 P (bf16) into shared memory in the MMA operand layout, and
//                 at the end normalises O and stores it as bf16.
// Grid order runs query blocks from the last (most key blocks) to the first,
// so long rows start early.
#pragma once
#include "ptx.cuh"

namespace prism {
namespace attn {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kHalfBytes = 128 * 64 * 2;     // 128 rows x 64 bf16 (one swizzle span)
constexpr uint32_t kTileBytes = 2 * kHalfBytes;   // 128 x 128 bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffP = kOffV + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffP + kTileBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 256;

// Iterates the kept key blocks j <= i of one mask row in ascending order.
struct KeptIter {
  const uint32_t* row;
  int last_word;
  uint32_t last_mask;
  int w;
  uint32_t bits;
  __device__ __forceinline__ void init(const uint32_t* r, int i) {
    row = r;
    last_word = i >> 5;
    last_mask = ((i & 31) == 31) ? 0xffffffffu : ((2u << (i & 31)) - 1u);
    w = 0;
    bits = load(0);
  }
  __device__ __forceinline__ uint32_t load(int ww) const {
    uint32_t b = row[ww];
    return ww == last_word ? (b & last_mask) : b;
  }
  __device__ __forceinline__ int next() {
    while (bits == 0u) {
      if (++w > last_word) return -1;
      bits = load(w);
    }
    const int b = __ffs(bits) - 1;
    bits &= bits - 1u;
    return (w << 5) + b;
  }
};

__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const uint32_t* __restrict__ mask,
                   __nv_bfloat16* __restrict__ out, int batch, int hq, int hkv, int seqlen, int nb,
                   float scale_log2) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sgen = smem_raw + (sbase - raw);
  const uint32_t bar_q = sbase + kOffBar;
  const uint32_t bar_kv_full = bar_q + 8;    // [2]
  const uint32_t bar_kv_empty = bar_q + 24;  // [2]
  const uint32_t bar_s_full = bar_q + 40;
  const uint32_t bar_p_full = bar_q + 48;
  const uint32_t bar_o_full = bar_q + 56;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sgen + kOffBar + 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = batch * hq;
  const int i = nb - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
  const int bi = bh / hq, h = bh - bi * hq;
  const int kvh = bi * hkv + h / (hq / hkv);
  const int W = (nb + 31) >> 5;
  const uint32_t* mrow = mask + ((size_t)bh * nb + i) * W;

  // number of kept blocks j <= i (same value in every thread)
  int n_kept = 0;
  {
    KeptIter it;
    it.init(mrow, i);
    n_kept = __popc(it.bits);
    for (int ww = 1; ww <= it.last_word; ++ww) n_kept += __popc(it.load(ww));
  }

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_kv_full, 1);
    mbar_init(bar_kv_full + 8, 1);
    mbar_init(bar_kv_empty, 1);
    mbar_init(bar_kv_empty + 8, 1);
    mbar_init(bar_s_full, 1);
    mbar_init(bar_p_full, 128);
    mbar_init(bar_o_full, 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 5) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_kept > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int q_row = bh * seqlen + i * 128;
      mbar_arrive_expect_tx(bar_q, kTileBytes);
      tma_load_2d(sbase + kOffQ, &tmQ, 0, q_row, bar_q);
      tma_load_2d(sbase + kOffQ + kHalfBytes, &tmQ, 64, q_row, bar_q);
      KeptIter it;
      it.init(mrow, i);
      for (int t = 0;; ++t) {
        const int j = it.next();
        if (j < 0) break;
        const int s = t & 1;
        if (t >= kStages && !mbar_wait(bar_kv_empty + 8 * s, ((t >> 1) - 1) & 1)) break;
        const uint32_t full = bar_kv_full + 8 * s;
        mbar_arrive_expect_tx(full, 2 * kTileBytes);
        const int kr = kvh * seqlen + j * 128;
        const uint32_t kd = sbase + kOffK + s * kTileBytes, vd = sbase + kOffV + s * kTileBytes;
        tma_load_2d(kd, &tmK, 0, kr, full);
        tma_load_2d(kd + kHalfBytes, &tmK, 64, kr, full);
        tma_load_2d(vd, &tmV, 0, kr, full);
        tma_load_2d(vd + kHalfBytes, &tmV, 64, kr, full);
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kept > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);  // Q K-major, K K-major
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);  // P K-major, V MN-major
      if (mbar_wait(bar_q, 0)) {
        for (int t = 0; t < n_kept; ++t) {
          const int s = t & 1;
          if (!mbar_wait(bar_kv_full + 8 * s, (t >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t kb = sbase + kOffK + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            mma_bf16_ss(tS, smem_desc_sw128(sbase + kOffQ + off, 16, 1024),
                        smem_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0);
          }
          mma_commit(bar_s_full);
          if (!mbar_wait(bar_p_full, t & 1)) break;
          tc_fence_after();
          const uint32_t vb = sbase + kOffV + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            mma_bf16_ss(tO, smem_desc_sw128(sbase + kOffP + aoff, 16, 1024),
                        smem_desc_sw128(vb + kk * 2048, kHalfBytes, 1024), idesc_pv,
                        (t > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar_kv_empty + 8 * s);
          mma_commit(bar_o_full);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;  // query row within the block == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    __nv_bfloat16* orow = out + ((size_t)bh * seqlen + (size_t)i * 128 + r) * 128;
    bool ok = true;
    float m_run = -INFINITY, l_run = 0.f;
    KeptIter it;
    it.init(mrow, i);
    for (int t = 0; t < n_kept; ++t) {
      const int j = it.next();
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full, t & 1));
      if (!ok) break;
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t v[32];
        tmem_ld32(tS + lane_base + c4 * 32, v);
        tmem_wait_ld_dep(v);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c4 * 32 + e] = __uint_as_float(v[e]) * scale_log2;
      }
      if (j == i) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > r) x[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, x[c]);
      const float m_new = fmaxf(m_run, mx);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        x[c] = exp2f(x[c] - m_new);
        rs += x[c];
      }
      if (t > 0) {
        // the previous P V must be done before O is rescaled and P is rewritten
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_full, (t - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        const float alpha = exp2f(m_run - m_new);
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t v[32];
            tmem_ld32(tO + lane_base + c4 * 32, v);
            tmem_wait_ld_dep(v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(tO + lane_base + c4 * 32, v);
          }
          tmem_wait_st();
        }
        l_run = l_run * alpha + rs;
      } else {
        l_run = rs;
      }
      m_run = m_new;
      // P row r -> shared memory, 128-byte swizzled K-major layout:
      // half ch holds keys 64ch..64ch+63; row r at (r/8)*1024 + (r%8)*128;
      // 16-byte chunk u stored at chunk position u ^ (r % 8).
      unsigned char* prow = sgen + kOffP + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c0 = ch * 64 + u * 8;
          uint4 pk;
          pk.x = pack_bf16x2(x[c0 + 0], x[c0 + 1]);
          pk.y = pack_bf16x2(x[c0 + 2], x[c0 + 3]);
          pk.z = pack_bf16x2(x[c0 + 4], x[c0 + 5]);
          pk.w = pack_bf16x2(x[c0 + 6], x[c0 + 7]);
          *reinterpret_cast<uint4*>(prow + ch * kHalfBytes + ((u ^ (r & 7)) << 4)) = pk;
        }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p_full);
    }
    // ------------------------------------------------------------ epilogue
    if (n_kept == 0) {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int c = 0; c < 16; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
    } else if (ok && __all_sync(0xffffffffu, mbar_wait(bar_o_full, (n_kept - 1) & 1))) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t v[32];
        tmem_ld32(tO + lane_base + c4 * 32, v);
        tmem_wait_ld_dep(v);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 pk;
          pk.x = pack_bf16x2(__uint_as_float(v[q4 * 8 + 0]) * inv, __uint_as_float(v[q4 * 8 + 1]) * inv);
          pk.y = pack_bf16x2(__uint_as_float(v[q4 * 8 + 2]) * inv, __uint_as_float(v[q4 * 8 + 3]) * inv);
          pk.z = pack_bf16x2(__uint_as_float(v[q4 * 8 + 4]) * inv, __uint_as_float(v[q4 * 8 + 5]) * inv);
          pk.w = pack_bf16x2(__uint_as_float(v[q4 * 8 + 6]) * inv, __uint_as_float(v[q4 * 8 + 7]) * inv);
          reinterpret_cast<uint4*>(orow)[c4 * 4 + q4] = pk;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn
}  // namespace prism
