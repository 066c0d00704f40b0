/*
 * libspectra -- C ABI of a SPECTRA-style spectral latent KV-cache codec for
 * NVIDIA B200 (sm_100a).
 *
 * What it computes follows "SPECTRA: Pushing the KV Cache Beyond the 2-Bit Cliff
 * via Spectral Transform Coding" (technical summary):
 *   - "SPECTRA pipeline", stage 1 (G-weighted transform): the activation Gram
 *     G = E[h^T h] (observation 3) whitens W_K / W_V; the SVD of G^{1/2} W gives
 *     an energy-ordered, second-moment-orthogonal latent basis; W_down = W V_r
 *     projects a token down, W_up = V_r^T rebuilds it;
 *   - stage 2 (rate-distortion quantisation): reverse water-filling on the
 *     latent second moments decides bits; adjacent coordinates share one width
 *     ("grouping"); zero bits drop a group (observation 2);
 *   - stage 3 (system integration): every new token is projected down,
 *     quantised per token and appended to an append-only latent cache;
 *   - "Significance and claims": attention computed directly in the latent
 *     space (the query is folded with W_up, W_up^V is applied once per head).
 *
 * Conventions
 *   - Every entry point returns a spectra_status and never throws.  On failure,
 *     spectra_last_error() returns a thread-local message.
 *   - "device" pointers are CUDA global-memory addresses on the current device;
 *     "host" pointers are ordinary CPU memory.  `stream` is a cudaStream_t passed
 *     as void* (NULL = legacy default stream).  Device-side work is enqueued on
 *     `stream` and the call returns without synchronising, except where stated.
 *   - The caller owns every large device buffer (activations, queries,
 *     outputs, the cache pool, page table, lengths, workspaces); sizes come
 *     from the *_bytes helpers.  A codec owns only its small device tables and
 *     factors and is released by spectra_codec_destroy.
 *   - Conditions found on the device (capacity overflow, unsorted seq_ids, a
 *     bounded wait that gave up) set the codec's device error word; read and
 *     clear it with spectra_device_status.
 *   - No function here calls into a CPU fallback: without a usable CUDA device
 *     the device entry points fail with SPECTRA_ERR_CUDA.
 *
 * Canonical page layout (this library's definition; the pages only fix that
 * codes are appended per token with one width per group):
 *   A page holds P = page_tokens tokens of one sequence for every KV head.
 *   page = head sections a = 0..n_kv_heads-1; head section = K side then V side;
 *   side section = for each group j with b_j > 0, ascending: its code blocks
 *   (P*g*b_j/8 bytes), then its P/2 scale/zero records of 8 bytes.
 *   Code blocks: one block per 256/g consecutive tokens, 8*b_j little-endian
 *   uint32 words.  Entry (token tau of the block, coordinate k of the group) has
 *   a fragment position (gid, t4, slot), gid 0..7, t4 0..3, slot 0..7:
 *     g = 16: K side row = tau/2 (tau even) or 8 + tau/2 (tau odd), col = k;
 *             V side row = k, col = tau;
 *             gid = row % 8, t4 = (col % 8)/2, slot = row/8 + 2*(col/8) + 4*(col % 2);
 *     g = 8 (32-token blocks; mi = tau/16, tl = tau%16):
 *             K side row from tl as above, gid = row % 8, t4 = k/2,
 *                    slot = row/8 + 2*mi + 4*(k % 2);
 *             V side gid = k, t4 = (tl % 8)/2, slot = mi + 2*(tl/8) + 4*(tl % 2).
 *   Code bit p of the entry sits at (word, bit):
 *     b = 4: word 4*gid + t4, bit 4*slot + p;
 *     b = 2: word 2*gid + t4/2, bit 4*slot + 2*(t4 % 2) + p;
 *     b = 1: word gid, bit 4*slot + t4;
 *     b = 3: bits 0-1 as for b = 2 (words 0..15), bit 2 as for b = 1 in word 16 + gid;
 *     b = 8: word 2*(4*gid + t4) + (slot/2) % 2, bit 8*((slot % 2) + 2*(slot/4)) + p.
 *   (Lane gid*4 + t4 of an mma.sync A fragment thus finds its 8 codes in one or
 *   two words; slot r and r+4 form fragment register r.)
 *   Records: fp16 {s[2u], s[2u+1], z[2u], z[2u+1]} (little-endian) of the token
 *   pair u (tokens 2u, 2u+1 of the page) at record index (u % 8)*(P/16) + u/8.
 *   A page therefore takes exactly P * sum over kept groups of (g*b_j + 32)/8
 *   bytes; all offsets are multiples of 16 bytes.
 *
 * Quantiser (per token, per kept group of g fp32 latents, every step one IEEE
 * fp32 operation): s = fp16_rn(sat((max - min) / (2^b - 1))), z = fp16_rn(sat(min)),
 * code = clamp(rint_half_even((x - z) / s), 0, 2^b - 1); s == 0 gives codes 0;
 * sat clamps to +-65504.  Dequantised value: code*s + z.
 */
#ifndef SPECTRA_H
#define SPECTRA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPECTRA_ABI_VERSION 1

#if defined(__GNUC__)
#define SPECTRA_API __attribute__((visibility("default")))
#else
#define SPECTRA_API
#endif

typedef enum spectra_status {
  SPECTRA_OK = 0,
  SPECTRA_ERR_INVALID = 1,     /* bad argument: null pointer, size, alignment or shape */
  SPECTRA_ERR_CUDA = 2,        /* a CUDA runtime or driver call failed */
  SPECTRA_ERR_CAPACITY = 3,    /* page table / pool too small; nothing was written */
  SPECTRA_ERR_NUMERIC = 4,     /* non-finite data, Gram not positive definite, eigen failure */
  SPECTRA_ERR_UNSUPPORTED = 5, /* a shape outside what the kernels implement */
  SPECTRA_ERR_TIMEOUT = 6,     /* a bounded device wait gave up; the kernel returned early */
  SPECTRA_ERR_ORDER = 7        /* seq_ids of an append were not non-decreasing; nothing written */
} spectra_status;

typedef enum spectra_dtype { SPECTRA_F32 = 0, SPECTRA_BF16 = 1 } spectra_dtype;

/* Shapes and budget of one attention layer's codec. */
typedef struct spectra_config {
  int32_t d_model;        /* width of the layer input h */
  int32_t n_q_heads;      /* query heads */
  int32_t n_kv_heads;     /* KV heads; n_q_heads % n_kv_heads == 0, ratio (GQA) <= 8 */
  int32_t d_head;         /* head dimension (<= 256) */
  int32_t rank;           /* latent coordinates kept before allocation, <= d_head, multiple of group */
  int32_t group;          /* coordinates per group: 8 or 16 */
  int32_t budget_bits;    /* bits per token, per KV head, per side (K or V) */
  int32_t count_overhead; /* nonzero: a kept group costs group*b + 32 bits (fp16 s and z) */
  int32_t page_tokens;    /* P, tokens per cache page: multiple of 32, 32..1024 */
} spectra_config;

typedef struct spectra_codec spectra_codec; /* opaque, library-owned */

/* A paged, append-only latent cache.  All pointers are device memory owned by
 * the caller.  Page i occupies pool[i*page_bytes, (i+1)*page_bytes); the pool
 * must be 16-byte aligned.  page_table[b*max_pages_per_seq + k] is the page that
 * holds tokens [k*P, (k+1)*P) of sequence b.  lengths[b] is the number of
 * tokens of sequence b in the cache; encode advances it. */
typedef struct spectra_cache {
  void* pool;
  int64_t n_pages;
  const int32_t* page_table;
  int32_t* lengths;
  int32_t batch;
  int32_t max_pages_per_seq;
} spectra_cache;

/* Summary of a codec. */
typedef struct spectra_codec_info {
  spectra_config config;
  int32_t n_groups;          /* rank / group */
  int32_t n_eff;             /* latent columns of W_down: kept coordinates over all heads and sides */
  int64_t page_bytes;        /* bytes per cache page */
  int64_t bits_per_token;    /* sum over heads and sides of the spent bits (incl. overhead) */
  int32_t max_kept;          /* largest kept-coordinate count of one (head, side) */
} spectra_codec_info;

/* ------------------------------------------------------------------------- */
/* Calibration (once per layer, off the hot path)                             */
/* ------------------------------------------------------------------------- */

/* spectra_calibrate -- SPECTRA pipeline stages 1-2.
 *   H        device [n_tokens][d_model], dtype `dtype`: calibration activations.
 *   W_K, W_V device [d_model][n_kv_heads*d_head], dtype `dtype`: head a uses
 *            columns [a*d_head, (a+1)*d_head).
 * Accumulates G = sum_t h_t^T h_t on the GPU (tcgen05 tensor cores for bf16),
 * forms M = W^T G W per head and side on the GPU, and on the host (fp64)
 * eigen-decomposes M (Jacobi), sorts by decreasing eigenvalue, fixes signs
 * (largest-magnitude entry of each vector positive), allocates group widths
 * (spectra_allocate_widths) and folds W_down = W V_r (bf16) and W_up = V_r^T
 * (fp32).  Synchronises `stream`.  Allocates and frees its own temporary device
 * memory (O(d_model^2) bytes).  On success *out receives a new codec. */
SPECTRA_API spectra_status spectra_calibrate(const spectra_config* cfg, int32_t dtype, const void* H,
                                 int64_t n_tokens, const void* W_K, const void* W_V,
                                 spectra_codec** out, void* stream);

/* Width allocation of spectra_calibrate_ex. */
typedef enum spectra_allocation {
  SPECTRA_ALLOC_WATERFILL = 0, /* spectra_allocate_widths (stage 2 reverse water-filling, grouped) */
  SPECTRA_ALLOC_UNIFORM = 1    /* spectra_allocate_widths_uniform (one width for all kept groups) */
} spectra_allocation;

/* spectra_calibrate_ex -- spectra_calibrate with a choice of allocation and an
 * optional energy threshold on the rank.
 *   allocation        SPECTRA_ALLOC_WATERFILL (what spectra_calibrate does) or
 *                     SPECTRA_ALLOC_UNIFORM.
 *   energy_threshold  0: every group may get bits; in (0, 1]: per head and side
 *                     only the groups holding the leading spectra_energy_rank
 *                     coordinates (rounded up to whole groups) may get bits
 *                     ("Spectral-KV: SVD-projection KV cache compression
 *                     (28x)", technical principle 1; e.g. 0.95).
 * Otherwise as spectra_calibrate; SPECTRA_ERR_INVALID for other values. */
SPECTRA_API spectra_status spectra_calibrate_ex(const spectra_config* cfg, int32_t dtype, const void* H,
                                                int64_t n_tokens, const void* W_K, const void* W_V,
                                                int32_t allocation, double energy_threshold,
                                                spectra_codec** out, void* stream);

/* spectra_codec_create -- build a codec from given factors (no calibration).
 *   widths   host [n_kv_heads][2][rank/group], each in {0,1,2,3,4,8}.
 *   W_down   host fp32 [d_model][n_eff]; columns head-major, K then V, kept
 *            coordinates ascending (n_eff = number of kept coordinates over all
 *            heads and sides); rounded to bf16 (nearest, ties to even).
 *   W_up     host fp32 [n_kv_heads][2][rank][d_head] (rows of V_r^T; rows of
 *            dropped groups are ignored).
 *   sigma2   host [n_kv_heads][2][rank] or NULL (stored for info/serialisation). */
SPECTRA_API spectra_status spectra_codec_create(const spectra_config* cfg, const int32_t* widths,
                                    const float* W_down, const float* W_up,
                                    const double* sigma2, spectra_codec** out);

SPECTRA_API void spectra_codec_destroy(spectra_codec* codec);

SPECTRA_API spectra_status spectra_codec_get_info(const spectra_codec* codec, spectra_codec_info* out);

/* Host copies of the codec state.  Any output pointer may be NULL.
 *   widths [n_kv_heads][2][n_groups]; sigma2 [n_kv_heads][2][rank];
 *   theta [n_kv_heads][2] (continuous water level for the spent payload bits);
 *   W_down [d_model][n_eff] (the bf16 values as fp32); W_up [n_kv_heads][2][rank][d_head]. */
SPECTRA_API spectra_status spectra_codec_get_state(const spectra_codec* codec, int32_t* widths,
                                       double* sigma2, double* theta, float* W_down,
                                       float* W_up);

/* Versioned binary blob of the codec (config, widths, sigma2, theta, W_down
 * bf16, W_up fp32).  Call with buf == NULL to get the size in *bytes. */
SPECTRA_API spectra_status spectra_codec_serialize(const spectra_codec* codec, void* buf, size_t* bytes);
SPECTRA_API spectra_status spectra_codec_deserialize(const void* buf, size_t bytes, spectra_codec** out);

/* spectra_wo_correction -- SPECTRA pipeline stage 1, "Refinement": a closed-form,
 * training-free correction of W_O for the rank truncation.  Reading used here
 * (the pages give no formula): treat the calibration tokens as one causal
 * sequence; for each q head h (KV head a = h / (n_q/n_kv)) let O_h be the
 * attention output with exact K, V and L_h the latent output of attention with
 * the rank-truncated, unquantised K and the values projected on the kept value
 * directions U_a (kept coordinates only).  M'_h = (L_h^T L_h + eps I)^-1 L_h^T O_h
 * with eps = 1e-8 tr(L_h^T L_h)/n_kept, M_h = U_a M'_h, W_O' = blockdiag(M_h) W_O
 * (the minimum-norm least-squares map from the truncated output to the exact one).
 *   H device [n_tokens][d_model]; W_Q device [d_model][n_q_heads*d_head];
 *   W_K, W_V as for calibrate; W_O device [n_q_heads*d_head][d_model];
 *   W_O_out device fp32 [n_q_heads*d_head][d_model].  All inputs in `dtype`.
 * Synchronises `stream`; n_tokens <= 4096. */
SPECTRA_API spectra_status spectra_wo_correction(const spectra_codec* codec, int32_t dtype, const void* H,
                                     int64_t n_tokens, const void* W_Q, const void* W_K,
                                     const void* W_V, const void* W_O, float* W_O_out,
                                     void* stream);

/* ------------------------------------------------------------------------- */
/* Hot path                                                                   */
/* ------------------------------------------------------------------------- */

/* Workspace bytes for spectra_encode_append with up to max_tokens tokens. */
SPECTRA_API spectra_status spectra_encode_workspace_bytes(const spectra_codec* codec, int64_t max_tokens,
                                              size_t* bytes);
/* Workspace bytes for spectra_decode_attend with `batch` sequences of up to
 * max_len tokens. */
SPECTRA_API spectra_status spectra_decode_workspace_bytes(const spectra_codec* codec, int32_t batch,
                                              int64_t max_len, size_t* bytes);

/* spectra_project -- stage 3 "projected down": latents = H W_down.
 *   H device bf16 [T][d_model]; latents device fp32 [T][n_eff].
 * bf16 x bf16 products accumulated in fp32: tcgen05 tensor cores for T >= 64,
 * a bandwidth-bound CUDA-core kernel for smaller T. */
SPECTRA_API spectra_status spectra_project(const spectra_codec* codec, const void* H, int64_t T,
                               float* latents, void* stream);

/* spectra_quantize_append -- stage 3 "quantised per token, appended": quantise
 * fp32 latents (layout of spectra_project's output) and write them into the
 * cache at lengths[seq]; then advance lengths.
 *   latents device fp32 [T][n_eff]; seq_ids device int32 [T], non-decreasing,
 *   each in [0, batch).  Token i goes to position lengths[seq_ids[i]] + (i minus
 *   the first index of its sequence in this call).  If any token would not fit
 *   (position >= max_pages_per_seq*P, or a needed page id outside [0, n_pages))
 *   or seq_ids are not sorted, nothing is written and the device error word is
 *   set (SPECTRA_ERR_CAPACITY / SPECTRA_ERR_ORDER).  workspace: device,
 *   >= spectra_encode_workspace_bytes(T), 256-byte aligned (per-token positions). */
SPECTRA_API spectra_status spectra_quantize_append(const spectra_codec* codec, const spectra_cache* cache,
                                       const float* latents, const int32_t* seq_ids, int64_t T,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* spectra_encode_append -- spectra_project followed by spectra_quantize_append.
 *   H device bf16 [T][d_model]; seq_ids as above; latents_out device fp32
 *   [T][n_eff] or NULL (when given, the latents are kept there);
 *   workspace device, >= spectra_encode_workspace_bytes(T), 256-byte aligned;
 *   its first 8448 bytes hold arrival counters that must be zero when a call
 *   starts: zero the workspace once before its first use; every call leaves
 *   the counters at zero.  Calls that share a workspace must not overlap.
 * For T <= 16 (decode steps) the projection, quantisation and packing run fused
 * in one kernel: CTAs per (kept group, d_model chunk) write partial sums, the
 * last chunk of a group adds them in chunk order and quantises the group
 * (latents summed in a different order than spectra_project's, so they may
 * differ from it in the last bits; the codes are those
 * spectra_quantize_append gives for these latents).  The lengths advance as
 * soon as every CTA holds its positions, while the page writes may still be
 * in flight: a kernel of this library that starts before this one completes
 * (spectra_decode_attend) reads the lengths before its dependency wait only as
 * a hint, 16 tokens short.  For T >= 64 with latents_out
 * NULL (prefill) the positions are planned and checked first, then the
 * tcgen05 projection GEMM quantises and packs each output tile in its
 * epilogue, so no fp32 latents are written; its accumulators equal
 * spectra_project's, so the pages equal those of spectra_project followed by
 * spectra_quantize_append.  Otherwise (16 < T < 64, or latents_out given) the
 * latents go through memory.  The same checks apply on every route and a
 * failure writes nothing.  The decode-step encode stages W_down rows in shared
 * memory behind a bounded wait (200 ms); if it gives up, the call records
 * SPECTRA_ERR_TIMEOUT, the lengths may already have advanced and the step's
 * codes are undefined.  Test hooks, read from the environment at every launch
 * and meant for tests only: SPECTRA_ENCODE_TEST_DROP_STAGE (the first CTA never
 * issues its first staged copy, so its wait gives up) and
 * SPECTRA_ENCODE_TEST_WAIT_NS (the wait's limit). */
SPECTRA_API spectra_status spectra_encode_append(const spectra_codec* codec, const spectra_cache* cache,
                                     const void* H, const int32_t* seq_ids, int64_t T,
                                     float* latents_out, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* spectra_decode_attend -- one decode step of attention for every sequence of
 * the cache, in the latent space: q_lat = q W_up^K^T, scores against the
 * dequantised latent keys of all lengths[b] tokens, exact (online) softmax,
 * sum_t p_t c_V,t, then W_up^V once per head.  Split-K over the context; no
 * masking beyond lengths[b].  One kernel launch; the split-K partition and the
 * merge order depend only on the lengths, so the result is deterministic.
 *   q   device fp32 [batch][n_q_heads][d_head]
 *   out device fp32 [batch][n_q_heads][d_head] (attention output before W_O)
 *   workspace device, >= spectra_decode_workspace_bytes, 256-byte aligned.  It
 *       holds the split-K records and per-(sequence, KV head) arrival counters
 *       that must be zero when a call starts: zero the workspace once before
 *       its first use; every call leaves the counters at zero again.  Calls
 *       that share a workspace must not overlap on the GPU.
 * q must not be written by a kernel of this library still running in the
 * same stream (q is read before the dependency on earlier launches resolves).
 * A length outside [0, max_pages_per_seq * page_tokens] (that sequence is then
 * read as empty) or a page id outside [0, n_pages) (that context split's pages
 * are skipped) records SPECTRA_ERR_INVALID in the device error word.  The cache
 * may come straight from spectra_encode_append or spectra_quantize_append on
 * the same stream, with no synchronisation in between.  Needs d_head a
 * multiple of 16 and at most 256, at most 8 kept groups per head and side and
 * at most 8 q heads per KV head (else SPECTRA_ERR_UNSUPPORTED).
 * Test hooks, read from the environment at every launch and meant for tests
 * only: SPECTRA_DECODE_HINT_LAG (tokens taken off the early length hint beyond
 * the built-in 16; the result does not change), SPECTRA_DECODE_TEST_DROP_PAGE
 * (the first CTA never issues the copy of that page of its list, so its
 * bounded wait gives up and the call reports SPECTRA_ERR_TIMEOUT) and
 * SPECTRA_DECODE_TEST_WAIT_NS (the limit of every bounded wait, default
 * 200 ms). */
SPECTRA_API spectra_status spectra_decode_attend(const spectra_codec* codec, const spectra_cache* cache,
                                     const float* q, float* out, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* spectra_decode_attend_noalloc -- the decode attention of spectra_decode_attend
 * for callers that cannot allocate device memory while they decode (a runtime
 * that plans all of its buffers ahead of time, a process whose device allocator
 * belongs to another framework, code running where an allocation would stall
 * or be refused).  No counterpart on the SPECTRA pages: an interface of this
 * library only.  Arguments as for spectra_decode_attend minus the workspace.
 * The scratch (split-K records and arrival counters) lives in one static 4 MiB
 * device array per GPU, kept until the process exits.  The first call on a
 * device looks up that array's device address (cudaGetSymbolAddress), so make
 * the first call on each device before any stream capture.  Every call shares
 * the array and leaves its contents behind: the counters, which must start at
 * zero, are zero when the library loads and every completed call leaves them
 * at zero; the records are rewritten by each call before they are read.
 * Calls whose kernels can overlap on the GPU (other streams, other codecs at
 * the same time) race on the array: serialise them.  A batch/context
 * whose scratch would exceed 4 MiB fails with SPECTRA_ERR_CAPACITY.  Calls no
 * cudaMalloc, cudaFree or allocating library routine. */
SPECTRA_API spectra_status spectra_decode_attend_noalloc(const spectra_codec* codec,
                                                         const spectra_cache* cache, const float* q,
                                                         float* out, void* stream);

/* spectra_reconstruct -- rebuild the keys and values of cached tokens (stage 3:
 * the dequantised latents lifted back with W_up for standard attention):
 *   k^ = c^_K W_up^K, v^ = c^_V W_up^V, c^ = code * s + z (fp32), zero-width
 *   groups contributing 0, for tokens [t0, t0 + n) of sequence `seq`.
 *   K_out, V_out device fp32 [n][n_kv_heads][d_head], caller-owned.
 * Any group count and width.  A range beyond lengths[seq] (known only on the
 * device) or a page id outside [0, n_pages) records SPECTRA_ERR_INVALID in the
 * device error word and leaves the outputs unspecified. */
SPECTRA_API spectra_status spectra_reconstruct(const spectra_codec* codec, const spectra_cache* cache,
                                               int32_t seq, int64_t t0, int64_t n, float* K_out, float* V_out,
                                               void* stream);

/* Workspace bytes for spectra_decode_attend_reconstruct with `batch` sequences
 * of up to max_len tokens (a cache whose max_pages_per_seq * page_tokens is at
 * most max_len). */
SPECTRA_API spectra_status spectra_decode_reconstruct_workspace_bytes(const spectra_codec* codec, int32_t batch,
                                                                      int64_t max_len, size_t* bytes);

/* spectra_decode_attend_reconstruct -- one decode step of attention with the
 * keys rebuilt from the cache ("SPECTRA pipeline" stage 3 as the pages
 * integrate it: latents dequantised and lifted back with W_up, then standard
 * attention), with optional rotary position embedding:
 *   k^_t = R(t) (c^_K,t W_up^K) for t in [0, lengths[b]),  q' = R(lengths[b]-1) q,
 *   out = softmax(q' k^^T / sqrt(d_head)) (c^_V W_up^V)
 * where R(p) turns the pair (i, i + d_head/2) by p * rope_theta^(-2i/d_head)
 * (the rotate-half form) and rope_theta = 0 means no rotation (then the result
 * equals spectra_decode_attend's up to rounding).  The values are summed in the
 * latent space and lifted once per head (the same result by linearity).
 *   q   device fp32 [batch][n_q_heads][d_head] (before rotation)
 *   out device fp32 [batch][n_q_heads][d_head]; a sequence of length 0 gives 0
 *   workspace device, >= spectra_decode_reconstruct_workspace_bytes, 256-byte aligned.
 * Needs d_head a multiple of 16 and <= 128, <= 128 kept coordinates per side and
 * <= 8 q heads per KV head (else SPECTRA_ERR_UNSUPPORTED).  rope_theta must be
 * 0 or a finite value above 1 (else SPECTRA_ERR_INVALID).  A page id outside
 * [0, n_pages) or a length outside [0, max_pages_per_seq * page_tokens] records
 * SPECTRA_ERR_INVALID in the device error word (that part reads as zero). */
SPECTRA_API spectra_status spectra_decode_attend_reconstruct(const spectra_codec* codec, const spectra_cache* cache,
                                                             const float* q, double rope_theta, float* out,
                                                             void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the codec's device error word.
 * Returns the recorded device-side status (SPECTRA_OK if none). */
SPECTRA_API spectra_status spectra_device_status(const spectra_codec* codec, void* stream);

/* ------------------------------------------------------------------------- */
/* Host-only helpers (no GPU needed)                                          */
/* ------------------------------------------------------------------------- */

/* Grouped widths for one (head, side): b_j in {0,1,2,3,4,8} minimising
 * sum_j S_j 4^-b_j (S_j = sum of sigma2 over group j, summed in ascending order;
 * b = 0 leaves S_j) subject to sum_j cost(b_j) <= budget_bits, cost(b) =
 * group*b (+32 with count_overhead) for b > 0.  Exact backward dynamic programme
 * over groups; ties go to the smaller width.  This is the discrete, grouped form
 * of reverse water-filling (stage 2).  widths_out [rank/group]; distortion_out
 * may be NULL. */
SPECTRA_API spectra_status spectra_allocate_widths(const double* sigma2, int32_t rank, int32_t group,
                                       int32_t budget_bits, int32_t count_overhead,
                                       int32_t* widths_out, double* distortion_out);

/* Uniform allocation (SpectralQuant with uniform allocation, "Ablation,
 * Statistical Inference, and Validation for KV-Cache Compression", practical
 * recommendations): the leading k of the first n_eligible_groups groups all get
 * one width b in {1,2,3,4,8}, the others 0; (k, b) minimises the model
 * sum_j S_j 4^-b_j of spectra_allocate_widths under the same budget (ties: fewer
 * bits, then fewer groups; k = 0 when nothing fits).  widths_out [rank/group];
 * distortion_out may be NULL. */
SPECTRA_API spectra_status spectra_allocate_widths_uniform(const double* sigma2, int32_t rank, int32_t group,
                                                           int32_t n_eligible_groups, int32_t budget_bits,
                                                           int32_t count_overhead, int32_t* widths_out,
                                                           double* distortion_out);

/* Effective rank: the smallest r with sigma2_0 + .. + sigma2_{r-1} >= threshold *
 * (sigma2_0 + .. + sigma2_{n-1}), sigma2 in decreasing order, threshold in
 * (0, 1] ("Spectral-KV: SVD-projection KV cache compression (28x)", technical
 * principle 1, spectral profiling). */
SPECTRA_API spectra_status spectra_energy_rank(const double* sigma2, int32_t n, double threshold,
                                               int32_t* rank_out);

/* Continuous reverse water-filling: theta with sum_i max(0, 1/2 log2(sigma2_i/theta))
 * = rate_bits; rates_out [n] (may be NULL). */
SPECTRA_API spectra_status spectra_water_fill(const double* sigma2, int32_t n, double rate_bits,
                                  double* theta_out, double* rates_out);

/* Symmetric eigen-decomposition (cyclic Jacobi, fp64) of the row-major n x n
 * matrix M (n <= 512): eigenvalues decreasing, eigenvectors as columns of the
 * row-major n x n `vecs`, each with its largest-magnitude entry positive. */
SPECTRA_API spectra_status spectra_sym_eigen(const double* M, int32_t n, double* vals, double* vecs);

/* Page size and group placement for given widths ([n_kv_heads][2][rank/group]).
 * offsets (may be NULL) receives, per (head, side, group), the byte offset of
 * the group's first code block in the page (-1 for dropped groups), followed by
 * the same count of record offsets. */
SPECTRA_API spectra_status spectra_page_layout(const spectra_config* cfg, const int32_t* widths,
                                   int64_t* page_bytes, int64_t* offsets);

SPECTRA_API const char* spectra_last_error(void);
SPECTRA_API int32_t spectra_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SPECTRA_H */
