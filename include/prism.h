/*
 * prism.h -- C ABI of the B200 (sm_100a) implementation of Prism's
 * spectral-aware block-importance estimator and the causal block-sparse
 * attention prefill that consumes its mask.
 *
 * Method: "Prism: Spectral-Aware Block-Sparse Attention" (Wang et al., 2026,
 * arXiv 2602.08426).  Passages cited below:
 *   [review:method]  paper.rainbus.top review, the paragraph listing the full
 *                    pipeline, steps (1)-(7);
 *   [review:repro]   the same page, reproducibility paragraph (B = 128,
 *                    d_high = 64, d_low = 96, p = 0.95 / 0.93);
 *   [summary:1], [summary:2A], [summary:2B]  gist.science Technical Summary,
 *                    sections 1 (mean pooling as coarse proxy, block-sparse
 *                    attention computes a subset of blocks), 2A (dual band),
 *                    2B (RMS-based temperature calibration).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor arguments are DEVICE pointers owned by the caller, contiguous,
 *   16-byte aligned (the mask: 4-byte aligned, so the rows of any group of
 *   heads can be addressed inside a larger mask).  The library never
 *   allocates device memory, never synchronises, and enqueues all work on
 *   the caller's `stream` (0 = the legacy default stream).  Calls are asynchronous: a 0 return means the work
 *   was enqueued, not that it finished.
 * - Layouts (b = batch, hq / hkv = query / key-value heads, N = seqlen (the
 *   padded length when per-sequence lengths are given), D = head_dim = 128,
 *   nb = ceil(N / 128), W = ceil(nb / 32)):
 *     q, o        bf16 [b, hq,  N, D]     (Q after RoPE; output O)
 *     k, v        bf16 [b, hkv, N, D]     (K after RoPE)
 *     mask        uint32 [b, hq, nb, W]:  bit (j % 32) of word j / 32 of row i
 *                 set <=> key block j is kept for query block i.  The
 *                 estimator writes every word (bits j > i are 0).
 * - GQA: query head h reads key/value head h / (hq / hkv).
 * - Return value: PRISM_OK (0) or a negative PRISM_ERR_* code.  Argument
 *   checks run on the host before anything is enqueued; on an error nothing
 *   is enqueued and no output is touched.  The library never aborts or traps.
 */
#ifndef PRISM_B200_H
#define PRISM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* prism_stream_t; /* == cudaStream_t */

enum {
  PRISM_OK = 0,
  PRISM_ERR_NULL = -1,        /* a required pointer is NULL                        */
  PRISM_ERR_SHAPE = -2,       /* batch/heads/seqlen non-positive, hq % hkv != 0,
                                 or sizes overflow                                 */
  PRISM_ERR_ALIGN = -3,       /* a tensor pointer is not 16-byte aligned (mask: 4)  */
  PRISM_ERR_BAND = -4,        /* band index out of [0, head_dim), duplicated, or an
                                 empty band                                        */
  PRISM_ERR_P = -5,           /* p is not in (0, 1] (p > 1 is treated as 1), or NaN */
  PRISM_ERR_UNSUPPORTED = -6, /* head_dim != 128, block != 128, causal != 1, or an
                                 unknown tau_mode                                  */
  PRISM_ERR_WORKSPACE = -7,   /* workspace NULL or smaller than prism_workspace_size */
  PRISM_ERR_CUDA = -8,        /* a CUDA runtime call failed (launch, attribute)     */
  PRISM_ERR_DEVICE = -9,      /* the device is not sm_100 (B200-class)              */
  PRISM_ERR_TIMEOUT = -10,    /* a kernel gave up a bounded wait (device error word) */
  PRISM_ERR_TAU = -11,        /* PRISM_TAU_EXPLICIT with a temperature that is not
                                 finite and > 0                                    */
  PRISM_ERR_SCRATCH_LIMIT = -12 /* prism_estimate_noalloc: the problem needs more
                                 scratch than prism_noalloc_scratch_bytes()        */
};

enum {
  PRISM_TAU_RMS = 0,      /* tau_z from the pooled RMS energies (reading R1 below) */
  PRISM_TAU_EXPLICIT = 1  /* tau_hi / tau_lo taken from the config (tests, ablations) */
};

/*
 * Problem statement of one attention layer ([review:method]; [review:repro]).
 * Band sets are HOST arrays of distinct dimension indices in [0, head_dim);
 * the default Prism split for the half-split RoPE layout is
 *   band_hi = {0..31} u {64..95}   (d_high = 64: the 32 fastest RoPE pairs)
 *   band_lo = {16..63} u {80..127} (d_low  = 96: the 48 slowest RoPE pairs)
 * The library copies what it needs during the call; the arrays may be freed
 * when the call returns.
 *
 * tau (step 4 of [review:method]) -- reading R1:
 *   tau_z = RMS(Qbar_z) * RMS(Kbar_z) / (RMS(Qbar_full) * RMS(Kbar_full)),
 *   per (batch, query head), RMS over all pooled blocks and the band's dims,
 *   Kbar of the head's KV head; tau_z = 1 if any RMS is 0.
 * Scores (step 5): L_z[i][j] = Qbar_z[i] . Kbar_z[j] / (tau_z sqrt(d_z)), j <= i.
 * Top-P (step 6): per row and band, keys ranked by (-prob, j); block j kept iff
 *   the mass ranked strictly ahead of it is < p (the crossing block is kept);
 *   p >= 1 keeps every causal block.  Union (step 7): M = M_hi | M_lo.
 */
typedef struct prism_config {
  int batch;
  int hq;
  int hkv;
  int seqlen;
  int head_dim;          /* must be 128 */
  int block;             /* B; must be 128.  seqlen need not be a multiple of B:
                            nb = ceil(seqlen / B) blocks, the last one short; its
                            pooled value is the mean over the tokens it has, and
                            attention sees only real tokens (causal) */
  const int32_t* band_hi;
  int n_hi;
  const int32_t* band_lo;
  int n_lo;
  float p;               /* Top-P threshold, 0 < p; p >= 1 keeps all causal blocks */
  int causal;            /* must be 1 */
  int tau_mode;          /* PRISM_TAU_RMS or PRISM_TAU_EXPLICIT */
  float tau_hi;          /* used only with PRISM_TAU_EXPLICIT; must be > 0 */
  float tau_lo;
  float softmax_scale;   /* attention scale; <= 0 selects 1/sqrt(head_dim) */
  int force_blocks;      /* 0: the mask is exactly M_high | M_low (the method).
                            Optional additions, OR-ed bit flags:
                            PRISM_FORCE_SINK keeps key block 0 in every row,
                            PRISM_FORCE_DIAG keeps the diagonal block j = i.
                            Other bits: PRISM_ERR_UNSUPPORTED. */
  const int32_t* seqlens;  /* NULL: every batch element holds seqlen tokens.
                            Else a host array of batch lengths, 1 <= seqlens[b]
                            <= seqlen (batch <= 256, else
                            PRISM_ERR_UNSUPPORTED; out of range:
                            PRISM_ERR_SHAPE): batch element b holds seqlens[b]
                            tokens at positions 0 .. seqlens[b]-1 of the
                            [.., seqlen, 128] layout, the rest is padding that
                            must hold zeros in q and k and finite values in v.
                            Each sequence has its own ceil(seqlens[b] / B)
                            blocks, pooling, temperatures and Top-P rows; mask
                            rows past them are written as zeros, o rows past
                            them are not written.  Read during the call only. */
} prism_config;

enum { PRISM_FORCE_SINK = 1, PRISM_FORCE_DIAG = 2 };

/*
 * Device workspace, in bytes, that prism_estimate / prism_prefill need for
 * `cfg` (prism_sparse_attn needs none).  Host-only; enqueues nothing.
 * Writes the size to *bytes.  The workspace holds the pooled Q/K means (three
 * bf16 terms per value),
 * per-block energy partials, the temperatures, the fp32 band scores
 * (b * hq * 2 * nb(nb+1)/2 floats) and the estimator's work-queue counters,
 * which each call clears with a memset on its stream; its contents on return
 * are unspecified.
 */
int prism_workspace_size(const prism_config* cfg, size_t* bytes);

/*
 * Optional copies of the estimator's intermediate values, for checking each
 * step on its own (the paper has no counterpart: these are test outputs).
 * Every member may be NULL (not written); all are DEVICE pointers, fp32,
 * owned by the caller, 16-byte aligned (tau: 4-byte).  nb(nb+1)/2 = T.
 *   scores   [b, hq, 2 (hi, lo), T]: the scaled band logits of step (5),
 *            L_z[i][j] = Qbar_z[i] . Kbar_z[j] / (tau_z sqrt(d_z)), in packed
 *            lower-triangular rows (row i starts at i(i+1)/2, j = 0..i).
 *   weights  [b, hq, 2, T], same packing: the unnormalised softmax weights
 *            e_j = 2^((L_j - max_k L_k) log2 e) in (0, 1] exactly as the Top-P
 *            step ranks and sums them (step (6): block j is kept iff the sum
 *            of round(e_k 2^31) over the blocks ranked ahead of it, by (-e, k),
 *            is below max(floor(p Z), 1), Z the row's sum of round(e_k 2^31)).
 *            Written only when p < 1.
 *   tau      [b, hq, 2] = (tau_hi, tau_lo) of step (4).
 *   pooled   [b hq + b hkv, nb, 128]: the block means of step (2) over all
 *            128 dims (rows: the b hq query heads batch-major, then the b hkv
 *            key heads batch-major); a short last block is the mean over its
 *            tokens; blocks past a sequence (per-sequence lengths) are not
 *            written.
 */
typedef struct prism_debug {
  float* scores;
  float* weights;
  float* tau;
  float* pooled;
} prism_debug;

/*
 * Estimator, steps (1)-(7) of [review:method]: band slicing and mean pooling
 * per block of B = 128 tokens, RMS energy of each pooled band, temperatures,
 * dual-band pooled softmax scores, Top-P per query-block row and band, union.
 *   q, k        inputs (layouts above)
 *   mask        output, uint32 [b, hq, nb, W]; every word written
 *   workspace   >= prism_workspace_size(cfg) bytes, 256-byte aligned
 *   dbg         optional (NULL: none) debug outputs, see prism_debug; the
 *               struct is read during the call only
 */
int prism_estimate(const prism_config* cfg, const void* q, const void* k, uint32_t* mask,
                   void* workspace, size_t workspace_bytes, prism_stream_t stream,
                   const prism_debug* dbg);

/*
 * Causal block-sparse attention ([summary:1]: only the selected blocks are
 * computed).  For a query token t in block i it attends to all keys of the
 * kept blocks j < i and to keys s <= t of block i if block i is kept;
 * O_t = sum_s softmax_s(q_t . k_s * scale) v_s, fp32 accumulation, bf16 out.
 * Bits of j > i are ignored; a query block with no kept block gets O = 0.
 * Runs on the tensor cores (tcgen05 MMA, accumulators in tensor memory).
 */
int prism_sparse_attn(const prism_config* cfg, const void* q, const void* k, const void* v,
                      const uint32_t* mask, void* o, prism_stream_t stream);

/*
 * One prefill layer: prism_estimate followed by prism_sparse_attn on the same
 * stream, no host synchronisation in between.  mask_out may be NULL, in which
 * case the mask lives in the workspace (the size then includes it).  The
 * attention is launched with programmatic serialization: its thread blocks
 * may start on SMs the estimator has left, each waiting (bounded, then
 * PRISM_ERR_TIMEOUT through prism_get_last_device_error) until the estimator
 * has published the mask rows it reads, so attention on finished rows
 * overlaps the end of the estimator (Prism: Spectral-Aware Block-Sparse
 * Attention, gist.science Technical Summary, introduction: the cost of
 * finding the relevant blocks is what such methods must keep small).  The
 * outputs equal those of the two separate calls.
 */
int prism_prefill(const prism_config* cfg, const void* q, const void* k, const void* v,
                  uint32_t* mask_out, void* o, void* workspace, size_t workspace_bytes,
                  prism_stream_t stream);

/*
 * Allocation-free estimator.  The paper has no counterpart to this entry
 * point: it exists for callers that cannot allocate device memory -- for
 * example a plugin inside a host framework that hands out no workspace, or a
 * serving loop that forbids cudaMalloc after start-up because it can
 * synchronise the device and fail under memory pressure.
 *
 * Computes exactly what prism_estimate computes (same kernels, same mask,
 * bit for bit) but uses scratch built into the library: a fixed device array
 * of prism_noalloc_scratch_bytes() = 32 MiB that every GPU loading the library
 * holds until the process exits.  The caller still passes q, k and mask
 * (device pointers, layouts as above); no dbg outputs.
 *   - Problems whose estimator workspace (prism_workspace_size less the
 *     mask slot only prism_prefill uses) exceeds 32 MiB are rejected with
 *     PRISM_ERR_SCRATCH_LIMIT before anything is enqueued (the Llama-3-8B
 *     shape, 32 Q / 8 KV heads, batch 1, fits up to 265 blocks = 33,920
 *     tokens).
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress while that device is current; make that first call
 *     before any stream capture.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; the few counters that must start at zero are cleared
 *     on `stream` at the start of each call.  Calls whose work overlaps on
 *     the GPU (different streams, or host threads, without ordering between
 *     them) race on the array.  Order them on one stream, or synchronise
 *     between them.
 */
int prism_estimate_noalloc(const prism_config* cfg, const void* q, const void* k, uint32_t* mask,
                           prism_stream_t stream);

/* Size in bytes of the scratch built into prism_estimate_noalloc. */
size_t prism_noalloc_scratch_bytes(void);

/*
 * Reads and clears the device error word that kernels set when a bounded
 * wait gives up (PRISM_ERR_TIMEOUT) -- synchronises `stream` first.  Returns
 * PRISM_OK when no kernel reported an error, a PRISM_ERR_* code otherwise.
 */
int prism_get_last_device_error(prism_stream_t stream);

/*
 * Diagnostic for the failure path (the paper has no counterpart): enqueues a
 * one-warp kernel on `stream` that waits, with the same bounded-wait helpers
 * the estimator and attention kernels use but a limit of `timeout_us`
 * microseconds (1 .. 2,000,000), on a device word nothing writes and on an
 * mbarrier phase nothing completes.  Both waits give up and record
 * PRISM_ERR_TIMEOUT; the kernel returns normally, so the context stays usable.
 * Read the result with prism_get_last_device_error(stream), which then returns
 * PRISM_ERR_TIMEOUT (and clears it).  Returns PRISM_OK once enqueued,
 * PRISM_ERR_SHAPE for a timeout out of range, PRISM_ERR_DEVICE / _CUDA.
 */
int prism_selftest_wait_timeout(prism_stream_t stream, unsigned timeout_us);

/* Static description of a status code; never NULL. */
const char* prism_status_str(int status);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int prism_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_B200_H */
