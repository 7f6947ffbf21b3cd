/*
 * sfa.h - C ABI of the B200 (sm_100a) importance-scored block-sparse attention library.
 *
 * The library computes, on one GPU, the two stages described in
 * "Prism: Spectral-Aware Block-Sparse Attention":
 *   1. a block-importance estimate from RoPE-applied Q/K that are mean-pooled
 *      per block, split into a high- and a low-frequency band and calibrated
 *      by an energy (RMS) temperature, followed by a block-level score matrix
 *      and a per-query-block selection (§1, §2, §3.1, §3.2, §5);
 *   2. exact softmax attention over the kept key blocks only (§1);
 * and the decode-side analogue of "FASA: Frequency-aware Sparse Attention"
 * (§2B): token importance of a KV cache from dominant rotary pairs, the top-k
 * tokens, and exact attention of one query token over them (sfa_decode_*).
 *
 * Conventions shared by every entry point:
 *   - Tensors are contiguous, row-major, layout [B, H, L, d] (batch, head,
 *     token, head dim).  Q has heads_q heads, K and V have heads_kv heads;
 *     Q head h reads KV head h / (heads_q / heads_kv) (grouped-query attention).
 *   - All tensor pointers are DEVICE pointers owned by the caller, into the
 *     memory of the calling thread's current CUDA device: every kernel is
 *     launched there.  The library never allocates or frees device memory and
 *     never synchronises the stream; every launch goes on `stream` (a
 *     cudaStream_t of that device passed as void*, NULL = legacy default
 *     stream).
 *   - Arguments are validated on the host before anything is launched; a
 *     validation failure returns an error status and launches nothing.  A
 *     failed launch returns SFA_ERR_CUDA.  Faults detected on the device
 *     (bounded waits that ran out, bad index lists) are written into the
 *     optional `status_word` (a device int, first error wins; 0 = ok) and the
 *     kernel returns without hanging.  No C++ exception crosses this ABI.
 *   - Sizes (prefill calls): L % block == 0; block in {64, 128}; d in {64, 128};
 *     heads_q % heads_kv == 0 (SFA_ERR_SHAPE otherwise); nb = L / block <= 2048
 *     and batch * heads_q * L < 2^31, so that every row of the [B*H*L, d] views
 *     has an int32 index (SFA_ERR_UNSUPPORTED otherwise).  The decode calls
 *     state their own rules below.
 */
#ifndef SFA_H_
#define SFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SFA_OK = 0,
  SFA_ERR_INVALID_ARG = 1,  /* null pointer, bad k / mass / flags / scale */
  SFA_ERR_SHAPE = 2,        /* sizes violate the rules above */
  SFA_ERR_DTYPE = 3,        /* unknown dtype code */
  SFA_ERR_UNSUPPORTED = 4,  /* valid but not implemented (e.g. nb > 2048) */
  SFA_ERR_WORKSPACE = 5,    /* workspace missing or too small */
  SFA_ERR_CUDA = 6,         /* a CUDA runtime / driver call failed */
  SFA_ERR_TIMEOUT = 7,      /* device: a bounded wait ran out (status_word only) */
  SFA_ERR_INDEX = 8         /* device: an index list entry out of range / not ascending */
} sfa_status;

typedef enum { SFA_F32 = 0, SFA_BF16 = 1 } sfa_dtype;

/* Problem shape.  dtype is the element type of Q, K, V, Q_rot, K_rot and O. */
typedef struct {
  int32_t batch, heads_q, heads_kv, seq_len, head_dim;
  int32_t dtype; /* sfa_dtype */
} sfa_shape;

/* RoPE tables: cos/sin of angle p * base^(-2m/d), [L, d/2] float32, device.
 * apply = 0 means Q and K are already rotated (tables ignored, may be NULL). */
typedef struct {
  const float* cos;
  const float* sin;
  int32_t apply;
} sfa_rope;

/* Flags for sfa_block_scores / sfa_select. */
enum {
  SFA_KEEP_SINK = 1,   /* select: also force key block 0 into every row */
  SFA_NO_CALIB = 2,    /* scores: temperature tau = 1 (plain mean pooling) */
  SFA_SINGLE_BAND = 4, /* scores: all d dims form one band (one tau) */
  SFA_RELATIVE_CALIB = 8, /* scores: restore band H relative to band L only: tau^H <- tau^H / tau^L, tau^L <- 1 */
  SFA_BAND_MAX = 16,      /* scores: one causal softmax per band, combined by the renormalised elementwise max */
  SFA_BLOCK_TAU = 32      /* scores: per-block temperature rho^b_i(Q) rho^b_j(K) (excludes NO_CALIB, RELATIVE_CALIB) */
};

/* Library version: major * 10000 + minor * 100 + patch. */
int sfa_version(void);

/* Human-readable text for a status code (static storage, never NULL). */
const char* sfa_status_string(sfa_status status);

/*
 * RoPE tables (Prism §2 names RoPE; the rotate-half convention of the Llama
 * and Qwen models of §5).  cos[p, m] = cos(p * base^(-2m/d)) and likewise
 * sin, computed on the host in double precision and rounded to float32, then
 * copied to the device arrays `cos` and `sin` ([seq_len, head_dim/2] each,
 * caller-owned) on `stream`.  Uses a temporary host buffer; returns after the
 * copies are enqueued.  Errors: SFA_ERR_INVALID_ARG for null pointers or
 * base <= 0; SFA_ERR_SHAPE for seq_len < 1 or an odd / non-positive head_dim.
 */
sfa_status sfa_rope_table(double base, int seq_len, int head_dim, float* cos, float* sin,
                          void* stream);

/*
 * Bytes of workspace sfa_block_scores needs for this shape and block size
 * (0 if the shape is invalid).  The workspace holds, each at a 256-byte
 * aligned offset given by sfa_workspace_layout:
 *   [0] Qbar   [B, heads_q,  nb, d] float64  block means of rotated Q
 *   [1] Kbar   [B, heads_kv, nb, d] float64  block means of rotated K
 *   [2] energy [B, heads_q + heads_kv, nb, 4] float64 per block:
 *              sum_t ||x_t^H||^2, sum_t ||x_t^L||^2, ||xbar^H||^2, ||xbar^L||^2
 *              (Q heads first, then KV heads)
 *   [3] tau    [B, heads_q, 2] float64  (band H, band L)
 */
size_t sfa_block_scores_workspace(const sfa_shape* shape, int block);

/* Byte offsets of the four workspace arrays above.  Errors as sfa_block_scores. */
sfa_status sfa_workspace_layout(const sfa_shape* shape, int block, size_t offsets[4]);

/*
 * Block-importance estimate (Prism §2, §3.1, §3.2, §5).
 *
 * Q [B, heads_q, L, d], K [B, heads_kv, L, d] (dtype of shape): pre-RoPE values
 * when rope->apply, else already rotated.  With rope->apply the rotated
 * tensors are written to Q_rot / K_rot (same shape and dtype, rounded to
 * nearest even); they are the Q and K the attention call should read.
 * Q_rot may be NULL: the rotated Q is then not stored, and the attention runs
 * through sfa_block_sparse_attn_rope, which rotates Q tiles as it loads them.
 *
 * Per (batch, Q head, band b in {H, L}), with band H = rotary pairs
 * m < band_split (dims m and m + d/2), band L = the other dims:
 *   xbar_j  = mean of the rotated vectors of block j
 *   rho^b   = sqrt(mean_j ||xbar_j^b||^2 / mean_t ||x_t^b||^2)   (1 if the band has no energy)
 *   tau^b   = max(rho^b(Q_h) * rho^b(K_g), 1e-6)   (1 with SFA_NO_CALIB)
 *   s_ij    = sum_b (qbar_i^b . kbar_j^b) / (tau^b * sqrt(d)),  j <= i
 *   probs_ij = exp(s_ij) / sum_{j' <= i} exp(s_ij'), and 0 for j > i.
 * probs [B, heads_q, nb, nb] float32.  SFA_SINGLE_BAND puts all dims in band H.
 * SFA_RELATIVE_CALIB (an alternative reading of the temperature) divides
 * tau^H by tau^L and sets tau^L = 1 (1 for both with a single band).
 * SFA_BLOCK_TAU (alternative reading, Prism §3.2): band b of s_ij is divided by
 * rho^b_i(Q_h) rho^b_j(K_g) instead of tau^b, where a block's own retained
 * amplitude is rho^b_j = sqrt(||xbar_j^b||^2 * block / sum_{t in j} ||x_t^b||^2),
 * floored at 1e-3, 1 if the block's band energy is 0 (the workspace tau still
 * holds the global values).  Combined with SFA_NO_CALIB or
 * SFA_RELATIVE_CALIB it is SFA_ERR_INVALID_ARG.
 * SFA_BAND_MAX (alternative reading, Prism §3 "two parallel branches"): each
 * band's part of s_ij gets its own causal softmax p^b; then
 * probs_ij = max_b p^b_ij / sum_{j' <= i} max_b p^b_ij'.  With one band (band
 * H or L empty, or SFA_SINGLE_BAND) it changes nothing.
 * RoPE is applied in float32; block means, energies, temperatures, logits and
 * the softmax are float64 (the 1/tau calibration amplifies pooled logits, so
 * float32 sums would move probabilities by ~1e-6), rounded once to float32.
 *
 * workspace: device buffer of at least sfa_block_scores_workspace() bytes,
 * 256-byte aligned; its contents are documented above and may be read back.
 * Errors: SFA_ERR_INVALID_ARG (null pointers, band_split outside [0, d/2],
 * unknown flags), SFA_ERR_SHAPE, SFA_ERR_DTYPE, SFA_ERR_UNSUPPORTED,
 * SFA_ERR_WORKSPACE, SFA_ERR_CUDA.  Launches 3 kernels.
 */
sfa_status sfa_block_scores(const sfa_shape* shape, const void* Q, const void* K,
                            const sfa_rope* rope, int band_split, int block, unsigned flags,
                            void* Q_rot, void* K_rot, float* probs, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * sfa_block_scores_select: sfa_block_scores followed by sfa_select in one
 * pass, the selection running on each row of block probabilities while it is
 * still in shared memory (the same float32 values, so the same index lists as
 * the two calls), so the probabilities need not be written to device memory:
 * `probs` may be NULL.  Arguments as in sfa_block_scores and sfa_select (k >= 0
 * top-k, else cumulative mass; counts [B, heads_q, nb], idx [B, heads_q, nb,
 * kmax]).  Errors: the union of both calls' errors.
 */
sfa_status sfa_block_scores_select(const sfa_shape* shape, const void* Q, const void* K,
                                   const sfa_rope* rope, int band_split, int block, unsigned flags,
                                   int k, float mass, void* Q_rot, void* K_rot, float* probs,
                                   int* counts, int* idx, int kmax, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * sfa_block_scores_noalloc - the same computation and outputs as
 * sfa_block_scores, for callers that cannot allocate device memory.
 * (The paper has no counterpart: this is a deployment convenience.)
 *
 * Some callers cannot call cudaMalloc or hand out scratch buffers at call
 * time: plugin or callback code run by a host runtime that owns all device
 * memory and passes in only the input and output buffers, processes whose
 * device memory is already reserved by another framework's allocator, and
 * latency-bound loops that must not risk the implicit device synchronisation
 * an allocation can cause.  This entry point takes the same arguments minus
 * the workspace; it uses a fixed scratch array of SFA_NOALLOC_SCRATCH_BYTES
 * (16 MiB) that the library declares in device memory, so every GPU that
 * loads the library holds those 16 MiB until the process exits.  It calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *
 * Limit: shapes whose sfa_block_scores_workspace() exceeds
 * SFA_NOALLOC_SCRATCH_BYTES are rejected with SFA_ERR_WORKSPACE (e.g. the
 * 32 query / 8 KV head, d = 128, block = 128 layer fits up to L = 32768 per
 * batch element).  The caller still passes Q, K, Q_rot, K_rot and probs.
 *
 * The first call on a device looks up the scratch array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it once the
 * lookup succeeds; make that first call before any stream capture (a first
 * call on a stream that is being captured returns SFA_ERR_CUDA and launches
 * nothing; the lookup is tried again by the next call).  All calls on a device share the one
 * scratch array and it keeps the last call's contents: calls whose kernels
 * overlap on the GPU (different streams, no ordering between them) race on it
 * and give wrong results.  Serialise such calls, e.g. issue them on one stream.
 * Every scratch region is fully rewritten by each call, so nothing needs
 * clearing between calls.  Errors: as sfa_block_scores, plus SFA_ERR_WORKSPACE
 * for shapes over the limit and SFA_ERR_UNSUPPORTED for device ordinals >= 64.
 */
#define SFA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
sfa_status sfa_block_scores_noalloc(const sfa_shape* shape, const void* Q, const void* K,
                                    const sfa_rope* rope, int band_split, int block, unsigned flags,
                                    void* Q_rot, void* K_rot, float* probs, void* stream);

/*
 * Block selection (Prism §1: attention runs over a chosen subset of key blocks).
 * For every row (b, h, i) of probs [B, heads_q, nb, nb]:
 *   forced F_i = {i}, plus {0} with SFA_KEEP_SINK;
 *   candidates {0..i} \ F_i ordered by (probability desc, index asc);
 *   top-k (k >= 0, mass ignored): keep F_i and the first min(k, |C_i|);
 *   mass (k < 0, 0 < mass <= 1): keep F_i, then add candidates in order while
 *     the running sum of kept probabilities (forced blocks included,
 *     accumulated in float64) is below mass.
 * Writes counts [B, heads_q, nb] int32 and idx [B, heads_q, nb, kmax] int32:
 * the kept indices ascending, padded with -1.  kmax must be >= the largest
 * possible count: min(nb, k + |F|) for top-k, nb for mass.
 * Errors: SFA_ERR_INVALID_ARG (nulls, mass outside (0, 1], kmax too small,
 * unknown flags), SFA_ERR_SHAPE, SFA_ERR_UNSUPPORTED, SFA_ERR_CUDA.
 */
sfa_status sfa_select(const sfa_shape* shape, int block, const float* probs, int k, float mass,
                      unsigned flags, int* counts, int* idx, int kmax, void* stream);

/*
 * Exact attention over the kept blocks (Prism §1).  For each query token t
 * of query block i, over the tokens s of the blocks idx[b, h, i, 0..count)
 * (with s <= t when causal):
 *   O_t = sum_s softmax_s(scale * q_t . k_s) v_s,   lse_t = log sum_s exp(scale * q_t . k_s)
 * Q [B, heads_q, L, d]; K, V [B, heads_kv, L, d]; O like Q; lse [B, heads_q, L]
 * float32 (natural log; optional, may be NULL).  An empty row gives O = 0 and
 * lse = -inf.  Each idx row must be ascending with entries in [0, nb) (and
 * <= i when causal); a violation found on the device sets status_word to
 * SFA_ERR_INDEX and that tile is skipped.
 * scale <= 0 selects 1/sqrt(d).
 * bf16 with block = 128 and d = 128 runs on the tcgen05 tensor cores (TMA
 * tiles fetched through the index list, accumulators in tensor memory);
 * every other case (float32, block 64, d 64) runs a float32 CUDA-core kernel.
 * Errors: SFA_ERR_INVALID_ARG, SFA_ERR_SHAPE, SFA_ERR_DTYPE, SFA_ERR_CUDA.
 */
sfa_status sfa_block_sparse_attn(const sfa_shape* shape, int block, const void* Q, const void* K,
                                 const void* V, const int* counts, const int* idx, int kmax,
                                 int causal, float scale, void* O, float* lse, int* status_word,
                                 void* stream);

/*
 * sfa_block_sparse_attn with RoPE applied to Q on load (Prism §5: the rotated
 * Q is used only by this call, so it need not make a round trip through
 * device memory).  Q is the pre-RoPE query tensor; rope->cos / rope->sin the
 * [L, d/2] float32 tables of sfa_rope_table (rope->apply must be nonzero);
 * K_rot the rotated keys written by sfa_block_scores.  Each Q tile is rotated
 * with the same float32 arithmetic and rounding to the storage dtype as
 * sfa_block_scores' Q_rot, so O and lse equal those of
 * sfa_block_sparse_attn(Q_rot, K_rot, V) bit for bit.  Other arguments,
 * layouts and errors as sfa_block_sparse_attn; SFA_ERR_INVALID_ARG also for a
 * missing or misaligned table.
 */
sfa_status sfa_block_sparse_attn_rope(const sfa_shape* shape, int block, const void* Q,
                                      const sfa_rope* rope, const void* K_rot, const void* V,
                                      const int* counts, const int* idx, int kmax, int causal,
                                      float scale, void* O, float* lse, int* status_word,
                                      void* stream);

/*
 * ---------------------------------------------------------------------------
 * Decode step ("FASA: Frequency-aware Sparse Attention" §2B): one query token
 * per (batch, Q head) against a KV cache.  shape->seq_len is the cache length
 * L; shape->dtype must be SFA_BF16 (SFA_ERR_DTYPE otherwise).  heads_q /
 * heads_kv in {1, 2, 4, 8}, and L at most 512 chunks of the selection kernel
 * (4096 tokens each, fewer for long pair lists: L <= 2^21 when 2 nfc <= 32),
 * else SFA_ERR_UNSUPPORTED.  q [B, heads_q, d] is the newest token's query,
 * already rotated at its position; K_cache, V_cache [B, heads_kv, L, d] hold
 * the rotated keys and the values at their original positions.
 *
 * fc: HOST array [heads_kv][nfc] of each KV head's dominant rotary pairs
 * (pair m = dims m and m + d/2; found by an offline calibration that this
 * library does not perform), distinct entries in [0, d/2); 4 <= nfc <= d/2,
 * nfc % 4 == 0, heads_kv * nfc <= 1024.  The Q heads of a group share their
 * KV head's list.  Violations: SFA_ERR_INVALID_ARG.
 * ---------------------------------------------------------------------------
 */

/*
 * Compact dominant-pair key copy (§2C, FASA-C reads only this part of the
 * keys for the estimate): K_fc [B, heads_kv, L, 2 nfc] bf16, column c < nfc =
 * dim fc[g][c], column nfc + c = dim fc[g][c] + d/2.  Writes the rows of
 * positions [pos0, pos0 + npos) only (the whole cache once, then each
 * appended range).  K_cache and K_fc 16-byte aligned.
 */
sfa_status sfa_decode_fc_gather(const sfa_shape* shape, const void* K_cache, const int* fc, int nfc,
                                int pos0, int npos, void* K_fc, void* stream);

/* Workspace bytes sfa_decode_select needs for a budget of k tokens (0 if invalid). */
size_t sfa_decode_workspace(const sfa_shape* shape, int k);

/*
 * Token Importance Predictor (§2B.1): for Q head h of KV group g,
 *   s_t = sum_{m in fc[g]} q_m k_{t,m} + q_{m+d/2} k_{t,m+d/2}
 * from K_fc, ranked by its float64 value (each bf16 x bf16 product is exact
 * in float64), then the first min(k, L) tokens by (s desc, index asc).  A
 * float32 copy of s serves only as a filter, with a margin of twice its
 * rounding bound, so it never drops a token of the top k (finite inputs).
 * idx [B, heads_q, k] int32: the kept token indices ascending, padded with -1.
 * k >= 1.  workspace: device, at least sfa_decode_workspace() bytes, 256-byte
 * aligned (SFA_ERR_WORKSPACE).  status_word (device, nullable):
 * SFA_ERR_TIMEOUT if a copy of the compact keys did not land within about 2 s
 * (that chunk then contributes no tokens).  Launches 2 kernels: a persistent
 * one (per chunk of the cache: float32 filter scores, a lower bound of the
 * row's k-th largest score found in the chunk or carried from an earlier
 * chunk of the same rows, the tokens above it with their 16-bit filter keys
 * and the chunk's filter error bound) and a merge per row (a tighter bound
 * from the candidates' filter keys, float64 scores of the survivors, exact top
 * k).  The calls of one step may be captured in a CUDA graph (all buffers
 * fixed at capture), as FasaDecode.step does.
 */
sfa_status sfa_decode_select(const sfa_shape* shape, const void* q, const void* K_fc, const int* fc,
                             int nfc, int k, int* idx, void* workspace, size_t workspace_bytes,
                             int* status_word, void* stream);

/*
 * Focused Attention Computation (§2B.2): full-dimension attention of q over
 * the tokens listed in idx [B, heads_q, k] (-1 entries skipped; the cached
 * keys keep their original positions):
 *   o = sum_t softmax_t(scale * q . k_t) v_t,  lse = log sum_t exp(scale * q . k_t)
 * o [B, heads_q, d] bf16; lse [B, heads_q] float32 (nullable; natural log).
 * scale <= 0 selects 1/sqrt(d).  An entry outside [-1, L) sets status_word to
 * SFA_ERR_INDEX and that row's o = 0, lse = -inf; an empty row likewise.
 */
sfa_status sfa_decode_attn(const sfa_shape* shape, const void* q, const void* K_cache,
                           const void* V_cache, const int* idx, int k, float scale, void* o,
                           float* lse, int* status_word, void* stream);

/*
 * Diagnostics (no counterpart in the pages): exercises the bounded wait that
 * every kernel of this library uses on its mbarriers.  One CTA waits on a
 * barrier phase that nothing completes (complete == 0) or that it completes
 * itself (complete != 0), giving up after limit_ms (1 .. 10000) milliseconds;
 * writes SFA_ERR_TIMEOUT or SFA_OK to *status_word (device).  Returns
 * SFA_ERR_INVALID_ARG for a NULL status word or a limit out of range.
 */
sfa_status sfa_selftest_bounded_wait(int* status_word, unsigned limit_ms, int complete, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SFA_H_ */
