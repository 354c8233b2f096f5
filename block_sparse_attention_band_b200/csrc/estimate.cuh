// Prism block-importance estimator, steps (1)-(7) of the method paragraph of
// the paper.rainbus.top review of "Prism: Spectral-Aware Block-Sparse
// Attention": band slicing, mean pooling per block of B = 128 tokens, RMS of
// each pooled band, temperatures tau_z, dual-band pooled softmax, Top-P per
// query-block row and band, union of the two masks.
//
// Four kernels, all on CUDA cores (the work is HBM-bound or small):
//   pool_kernel    (1)+(2)+(3 partials)  reads Q and K once (the HBM-bound part)
//   tau_kernel     (3)+(4)               one CTA per (batch, Q head)
//   scores_kernel  (5, logits)           fp32 register-tiled pooled Q K^T, both bands
//   topp_kernel    (5 softmax)+(6)+(7)   one warp per (batch, Q head, query block)
//
// Band slicing is folded into the pooled layout: the pooling kernel writes the
// 128 pooled dims in a permuted order [high-only | both | low-only | neither],
// so each band is a contiguous column range: high = [0, s2), low = [s1, s3).
#pragma once
#include "ptx.cuh"

namespace prism {

struct BandLayout {
  uint8_t perm[128];  // pooled column c holds original dim perm[c]
  int s1, s2, s3;     // segment boundaries (see above)
  int d_hi, d_lo;     // band sizes
};

// ---------------------------------------------------------------------------
// (1)+(2)+(3a): mean pool each 128x128 bf16 tile, write fp32 means in band
// order, and per-block energy partials sum(mean^2) over hi / lo / all dims.
// One CTA per (head row, block); 256 threads; thread t reads 16-byte vectors
// of rows t/16, t/16+16, ... at dims 8*(t%16) .. +7 (fully coalesced).
// ---------------------------------------------------------------------------
constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int q_rows,
            int nb, float* __restrict__ pool, float* __restrict__ part, const BandLayout bl) {
  __shared__ float red[16][128];
  __shared__ float mean[128];
  __shared__ float wsum[4][3];
  const int unit = blockIdx.x;
  const int hr = unit / nb;  // head row: q heads first, then k heads
  const int blk = unit - hr * nb;
  const __nv_bfloat16* src = hr < q_rows ? q + ((size_t)hr * nb + blk) * (128 * 128)
                                         : k + ((size_t)(hr - q_rows) * nb + blk) * (128 * 128);
  const int t = threadIdx.x;
  const int c8 = t & 15;
  const int rg = t >> 4;
  uint4 v[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) v[r] = ldg_nc_v4(src + (size_t)(rg + 16 * r) * 128 + c8 * 8);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    acc[0] += bf16lo(v[r].x); acc[1] += bf16hi(v[r].x);
    acc[2] += bf16lo(v[r].y); acc[3] += bf16hi(v[r].y);
    acc[4] += bf16lo(v[r].z); acc[5] += bf16hi(v[r].z);
    acc[6] += bf16lo(v[r].w); acc[7] += bf16hi(v[r].w);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][c8 * 8 + e] = acc[e];
  __syncthreads();
  if (t < 128) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < 16; ++g) s += red[g][t];
    mean[t] = s * (1.0f / 128.0f);
  }
  __syncthreads();
  if (t < 128) {
    const float m = mean[bl.perm[t]];
    pool[((size_t)hr * nb + blk) * 128 + t] = m;
    const float sq = m * m;
    float hi = t < bl.s2 ? sq : 0.f;
    float lo = (t >= bl.s1 && t < bl.s3) ? sq : 0.f;
    float all = sq;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      hi += __shfl_xor_sync(0xffffffffu, hi, o);
      lo += __shfl_xor_sync(0xffffffffu, lo, o);
      all += __shfl_xor_sync(0xffffffffu, all, o);
    }
    if ((t & 31) == 0) {
      wsum[t >> 5][0] = hi;
      wsum[t >> 5][1] = lo;
      wsum[t >> 5][2] = all;
    }
  }
  __syncthreads();
  if (t < 3) {
    const float s = (wsum[0][t] + wsum[1][t]) + (wsum[2][t] + wsum[3][t]);
    part[((size_t)hr * nb + blk) * 4 + t] = s;
  }
}

// ---------------------------------------------------------------------------
// (3)+(4): RMS of each pooled band over all blocks and the temperatures.
// One CTA (256 threads) per (batch, Q head).  Output tau[row] =
// (tau_hi, tau_lo, 1/(tau_hi sqrt d_hi), 1/(tau_lo sqrt d_lo)).
// ---------------------------------------------------------------------------
constexpr int kTauThreads = 256;

__global__ void __launch_bounds__(kTauThreads)
tau_kernel(const float* __restrict__ part, int q_rows, int hq, int hkv, int nb, int d_hi, int d_lo,
           int explicit_tau, float tau_hi_x, float tau_lo_x, float* __restrict__ tau,
           float* __restrict__ dbg_tau) {
  __shared__ float red[kTauThreads / 32][6];
  const int row = blockIdx.x;  // batch * hq + h
  const int bi = row / hq;
  const int h = row - bi * hq;
  const int kvrow = q_rows + bi * hkv + h / (hq / hkv);
  float s[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (!explicit_tau) {
    for (int i = threadIdx.x; i < nb; i += kTauThreads) {
      const float* pq = part + ((size_t)row * nb + i) * 4;
      const float* pk = part + ((size_t)kvrow * nb + i) * 4;
      s[0] += pq[0]; s[1] += pq[1]; s[2] += pq[2];
      s[3] += pk[0]; s[4] += pk[1]; s[5] += pk[2];
    }
  }
#pragma unroll
  for (int e = 0; e < 6; ++e)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s[e] += __shfl_xor_sync(0xffffffffu, s[e], o);
  if ((threadIdx.x & 31) == 0)
#pragma unroll
    for (int e = 0; e < 6; ++e) red[threadIdx.x >> 5][e] = s[e];
  __syncthreads();
  if (threadIdx.x == 0) {
    float th, tl;
    if (explicit_tau) {
      th = tau_hi_x;
      tl = tau_lo_x;
    } else {
      float S[6];
      for (int e = 0; e < 6; ++e) {
        float a = 0.f;
        for (int w = 0; w < kTauThreads / 32; ++w) a += red[w][e];
        S[e] = a;
      }
      const float n = (float)nb;
      const float rq_hi = sqrtf(S[0] / (n * d_hi)), rq_lo = sqrtf(S[1] / (n * d_lo));
      const float rq_f = sqrtf(S[2] / (n * 128.f));
      const float rk_hi = sqrtf(S[3] / (n * d_hi)), rk_lo = sqrtf(S[4] / (n * d_lo));
      const float rk_f = sqrtf(S[5] / (n * 128.f));
      const float den = rq_f * rk_f;
      const float nh = rq_hi * rk_hi, nl = rq_lo * rk_lo;
      th = (den > 0.f && nh > 0.f) ? nh / den : 1.f;
      tl = (den > 0.f && nl > 0.f) ? nl / den : 1.f;
    }
    tau[row * 4 + 0] = th;
    tau[row * 4 + 1] = tl;
    tau[row * 4 + 2] = 1.0f / (th * sqrtf((float)d_hi));
    tau[row * 4 + 3] = 1.0f / (tl * sqrtf((float)d_lo));
    if (dbg_tau) {
      dbg_tau[row * 2 + 0] = th;
      dbg_tau[row * 2 + 1] = tl;
    }
  }
}

// ---------------------------------------------------------------------------
// (5) band logits: L_z[i][j] = Qbar_z[i] . Kbar_z[j] * scale_z for j <= i.
// 64 x 64 output tiles over the lower triangle of each (batch, Q head);
// 256 threads, each a 4 x 4 register tile; the dims are accumulated segment
// by segment so the two bands share the overlapping dims' products.
// Output: packed lower-triangular rows, [row][band][i(i+1)/2 + j].
// ---------------------------------------------------------------------------
constexpr int kScoreTile = 64;
constexpr int kScoreThreads = 256;
constexpr int kScoreSmemBytes = 2 * 128 * kScoreTile * 4;

__global__ void __launch_bounds__(kScoreThreads)
scores_kernel(const float* __restrict__ pool, int q_rows, int hq, int hkv, int nb,
              const float* __restrict__ tau, int s1, int s2, int s3, float* __restrict__ scores) {
  extern __shared__ __align__(16) float score_smem[];
  float(*qT)[kScoreTile] = reinterpret_cast<float(*)[kScoreTile]>(score_smem);
  float(*kT)[kScoreTile] = reinterpret_cast<float(*)[kScoreTile]>(score_smem + 128 * kScoreTile);
  const int row = blockIdx.y;  // batch * hq + h
  const int bi = row / hq;
  const int h = row - bi * hq;
  const int kvrow = q_rows + bi * hkv + h / (hq / hkv);
  // lower-triangle tile index -> (ti, tj), tj <= ti
  const int tid = blockIdx.x;
  int ti = (int)((sqrtf(8.f * tid + 1.f) - 1.f) * 0.5f);
  while ((ti + 1) * (ti + 2) / 2 <= tid) ++ti;
  while (ti * (ti + 1) / 2 > tid) --ti;
  const int tj = tid - ti * (ti + 1) / 2;
  const int i0 = ti * kScoreTile, j0 = tj * kScoreTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* qsrc = pool + (size_t)row * nb * 128;
  const float* ksrc = pool + (size_t)kvrow * nb * 128;
  // transposed staging: lane -> row, warp -> 4-dim chunks
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int r = rr * 32 + lane;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c = warp + 8 * cc;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (i0 + r < nb) a = *reinterpret_cast<const float4*>(qsrc + (size_t)(i0 + r) * 128 + 4 * c);
      if (j0 + r < nb) b = *reinterpret_cast<const float4*>(ksrc + (size_t)(j0 + r) * 128 + 4 * c);
      qT[4 * c + 0][r] = a.x; qT[4 * c + 1][r] = a.y; qT[4 * c + 2][r] = a.z; qT[4 * c + 3][r] = a.w;
      kT[4 * c + 0][r] = b.x; kT[4 * c + 1][r] = b.y; kT[4 * c + 2][r] = b.z; kT[4 * c + 3][r] = b.w;
    }
  }
  __syncthreads();
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float a[4][4], b[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) a[u][w] = b[u][w] = 0.f;
  auto fma_range = [&](float(&acc)[4][4], int d0, int d1) {
#pragma unroll 4
    for (int d = d0; d < d1; ++d) {
      const float4 qa = *reinterpret_cast<const float4*>(&qT[d][4 * ty]);
      const float4 kb = *reinterpret_cast<const float4*>(&kT[d][4 * tx]);
      const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
      const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(qv[u], kv[w], acc[u][w]);
    }
  };
  fma_range(a, 0, s1);   // high-only dims
  fma_range(b, s1, s2);  // dims in both bands
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) a[u][w] += b[u][w];  // a = high band
  fma_range(b, s2, s3);  // b = low band
  const float sc_hi = tau[row * 4 + 2], sc_lo = tau[row * 4 + 3];
  __syncthreads();
  // stage the two 64 x 64 tiles through shared memory for coalesced row writes
  float* stage = &qT[0][0];  // 2 * 64 * 65 floats fit in qT + kT (16384 floats)
  constexpr int LD = kScoreTile + 1;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      stage[(4 * ty + u) * LD + 4 * tx + w] = a[u][w] * sc_hi;
      stage[kScoreTile * LD + (4 * ty + u) * LD + 4 * tx + w] = b[u][w] * sc_lo;
    }
  __syncthreads();
  const size_t tri = (size_t)nb * (nb + 1) / 2;
  float* out_hi = scores + (size_t)row * 2 * tri;
  float* out_lo = out_hi + tri;
  for (int r = warp; r < kScoreTile; r += kScoreThreads / 32) {
    const int i = i0 + r;
    if (i >= nb) break;
    const size_t base = (size_t)i * (i + 1) / 2;
    for (int c = lane; c < kScoreTile; c += 32) {
      const int j = j0 + c;
      if (j <= i) {
        out_hi[base + j] = stage[r * LD + c];
        out_lo[base + j] = stage[kScoreTile * LD + r * LD + c];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// (5 softmax)+(6)+(7): one warp per (batch, Q head, query block i).
// For each band: e_j = exp(L_j - max), Z = sum e_j; rank j by (-e_j, j);
// the crossing block c is the one with mass(ahead of c) < p Z <= mass(ahead)
// + e_c; keep every block ranked at or ahead of c.  The crossing block is
// found by a warp quickselect over candidate lists in shared memory (median
// of three pivots, stable ballot compaction), so the cost is O(n) per row.
// All sums run in a fixed order: the result is deterministic.
// ---------------------------------------------------------------------------
constexpr int kTopPWarps = 4;

__device__ __forceinline__ bool ranks_before(const float* e, int a, int b) {
  const float ea = e[a], eb = e[b];
  return ea > eb || (ea == eb && a < b);
}

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
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Returns the crossing block index, or -1 when every block is kept.
__device__ int topp_crossing(const float* e, uint16_t* bufA, uint16_t* bufB, int n, float target,
                             int lane) {
  const uint16_t* cur = nullptr;  // nullptr: candidates are 0..cnt-1
  uint16_t* nxt = bufA;
  int cnt = n;
  float base = 0.f;  // mass of blocks known to rank ahead of every candidate
#define CAND(x) (cur ? (int)cur[(x)] : (x))
  while (cnt > 32) {
    int p1 = CAND(cnt >> 2), p2 = CAND(cnt >> 1), p3 = CAND((3 * cnt) >> 2);
    // median of three by rank
    if (ranks_before(e, p2, p1)) { int t = p1; p1 = p2; p2 = t; }
    if (ranks_before(e, p3, p2)) { int t = p2; p2 = p3; p3 = t; }
    if (ranks_before(e, p2, p1)) { int t = p1; p1 = p2; p2 = t; }
    const int piv = p2;
    const float ep = e[piv];
    float s = 0.f;
    int c = 0;
    for (int x = lane; x < cnt; x += 32) {
      const int j = CAND(x);
      if (ranks_before(e, j, piv)) { s += e[j]; ++c; }
    }
    s = warp_sum(s);
    c = warp_sum_i(c);
    bool take_ahead;
    if (base + s >= target) {
      take_ahead = true;
    } else if (base + s + ep >= target) {
      return piv;
    } else {
      base = base + s + ep;
      take_ahead = false;
    }
    int out = 0;
    for (int x0 = 0; x0 < cnt; x0 += 32) {
      const int x = x0 + lane;
      bool sel = false;
      int j = 0;
      if (x < cnt) {
        j = CAND(x);
        sel = take_ahead ? ranks_before(e, j, piv) : ranks_before(e, piv, j);
      }
      const unsigned m = __ballot_sync(0xffffffffu, sel);
      if (sel) nxt[out + __popc(m & ((1u << lane) - 1u))] = (uint16_t)j;
      out += __popc(m);
    }
    __syncwarp();
    cur = nxt;
    nxt = (nxt == bufA) ? bufB : bufA;
    cnt = take_ahead ? c : cnt - c - 1;
  }
  // at most 32 candidates left: each lane holds one and sums the mass ahead of it
  int j = -1;
  float ej = 0.f;
  if (lane < cnt) {
    j = CAND(lane);
    ej = e[j];
  }
#undef CAND
  float ahead = 0.f;
  int rank = 0;
  for (int l = 0; l < cnt; ++l) {
    const int jl = __shfl_sync(0xffffffffu, j, l);
    const float el = __shfl_sync(0xffffffffu, ej, l);
    if (lane < cnt && (el > ej || (el == ej && jl < j))) {
      ahead += el;
      ++rank;
    }
  }
  const bool crosses = lane < cnt && (base + ahead + ej >= target);
  // first crossing in rank order (ranks are distinct integers)
  int best = crosses ? rank : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
  if (best != 0x7fffffff) {
    const unsigned m = __ballot_sync(0xffffffffu, crosses && rank == best);
    return __shfl_sync(0xffffffffu, j, __ffs(m) - 1);
  }
  // no candidate reaches the target (rounding with p close to 1): keep all of
  // them -- the lowest-ranked candidate becomes the cut, or everything if none
  if (cnt == 0) return -1;
  int worst = lane < cnt ? rank : -1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) worst = max(worst, __shfl_xor_sync(0xffffffffu, worst, o));
  const unsigned m = __ballot_sync(0xffffffffu, lane < cnt && rank == worst);
  return __shfl_sync(0xffffffffu, j, __ffs(m) - 1);
}

__global__ void __launch_bounds__(kTopPWarps * 32)
topp_kernel(const float* __restrict__ scores, int rows_total /* b*hq*nb */, int nb, float p,
            uint32_t* __restrict__ mask) {
  extern __shared__ __align__(16) unsigned char topp_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = (nb + 31) >> 5;
  const int nbp = (nb + 3) & ~3;
  const size_t per_warp = (size_t)nbp * 4 + (size_t)nbp * 2 * 2 + (size_t)W * 4;
  unsigned char* base = topp_smem + warp * ((per_warp + 15) & ~(size_t)15);
  float* e = reinterpret_cast<float*>(base);
  uint16_t* bufA = reinterpret_cast<uint16_t*>(base + (size_t)nbp * 4);
  uint16_t* bufB = bufA + nbp;
  uint32_t* bits = reinterpret_cast<uint32_t*>(base + (size_t)nbp * 8);
  const int gr = blockIdx.x * (blockDim.x >> 5) + warp;  // (batch*hq) * nb + i
  if (gr >= rows_total) return;
  const int row = gr / nb;
  const int i = gr - row * nb;
  const int n = i + 1;
  const size_t tri = (size_t)nb * (nb + 1) / 2;
  for (int w = lane; w < W; w += 32) bits[w] = 0u;
  __syncwarp();
  for (int band = 0; band < 2; ++band) {
    const float* src = scores + ((size_t)row * 2 + band) * tri + (size_t)i * (i + 1) / 2;
    float m = -INFINITY;
    for (int j = lane; j < n; j += 32) {
      const float x = src[j];
      e[j] = x;
      m = fmaxf(m, x);
    }
    m = warp_max(m);
    float z = 0.f;
    for (int j = lane; j < n; j += 32) {
      const float x = expf(e[j] - m);
      e[j] = x;
      z += x;
    }
    z = warp_sum(z);
    __syncwarp();
    int cross = -1;
    if (p < 1.0f) cross = topp_crossing(e, bufA, bufB, n, p * z, lane);
    __syncwarp();
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      bool keep = false;
      if (j < n) keep = (cross < 0) || j == cross || ranks_before(e, j, cross);
      const unsigned word = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) bits[j0 >> 5] |= word;
    }
    __syncwarp();
  }
  uint32_t* dst = mask + (size_t)gr * W;
  for (int w = lane; w < W; w += 32) dst[w] = bits[w];
}

}  // namespace prism
