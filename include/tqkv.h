/*
 * libtqkv -- TurboQuant compressed KV cache on one NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only; no C++ or CUDA types cross it.
 * Streams are passed as `void*` holding a cudaStream_t (NULL = default
 * stream).  Every call that launches GPU work is asynchronous on that stream
 * and returns a status code (tq_status); no exception crosses the ABI.
 *
 * Method, by page title and section:
 *  - "What is TurboQuant? mechanism, measured accuracy, status as of July
 *    2026": stage 1 rotates with a randomized Hadamard transform and applies
 *    per-coordinate Lloyd-Max quantization ("Stage 1: rotation and scalar
 *    quantization by PolarQuant"); stage 2 applies a 1-bit QJL projection to
 *    the residual so inner-product estimates are unbiased ("Stage 2");
 *    no calibration data ("Where calibration-free pays off"); presets chosen
 *    as a KV-cache dtype, k8v4 = FP8 keys + 4-bit values ("vLLM: available by
 *    switching --kv-cache-dtype").
 *  - "TurboQuant and RotorQuant on DGX Spark", "Two-stage compression:
 *    PolarQuant + QJL": no per-block scale values, one norm per vector.
 *  - "TurboQuant" overview (ai-work-lab.com), "QJL": +1/-1 sign bits of a
 *    random projection; the same codec serves inner-product vector search.
 *
 * Notation: d = head dimension (power of two, 8..1024); bits b; m = d QJL
 * rows; R = H D / sqrt(d) (H natural-order Sylvester Hadamard, D = diag of
 * random signs); S = m x d Gaussian matrix rounded to bf16; c = Lloyd-Max
 * levels for the coordinate law of a random unit vector in R^d.
 *
 * Memory ownership: the caller owns every buffer passed in (device memory
 * allocated by the caller, e.g. through torch).  The library owns only
 * tq_params objects (a host copy and a device copy).  Apart from
 * tq_make_params, no call allocates device memory: ops that need scratch
 * take a caller-allocated workspace whose size the matching
 * tq_*_workspace_bytes call returns.  Every workspace starts with a 256-byte
 * header holding a device status word (tq_read_status).
 */
#ifndef TQKV_H
#define TQKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
enum tq_status {
    TQ_OK = 0,
    TQ_EINVAL = 1,        /* bad argument (null pointer, size, alignment)   */
    TQ_EUNSUPPORTED = 2,  /* valid but unsupported (e.g. d not a power of 2) */
    TQ_ECUDA = 3,         /* a CUDA runtime call or launch failed            */
    TQ_EDEVICE = 4,       /* a kernel reported an error in the status word   */
    TQ_ENOMEM = 5,        /* tq_make_params could not allocate               */
    TQ_ESCRATCH = 6       /* problem needs more scratch than
                             tq_decode_attn_noalloc's static array holds     */
};

/* Bits of the device status word written by kernels (see tq_read_status). */
#define TQ_DEV_SLOT_RANGE   0x1u  /* slot_mapping entry beyond the cache; token skipped  */
#define TQ_DEV_BLOCK_RANGE  0x2u  /* block_table entry beyond the cache; page skipped    */
#define TQ_DEV_WAIT_TIMEOUT 0x4u  /* a bounded on-chip wait gave up; results invalid    */

/* Input dtypes for tq_encode. */
#define TQ_DTYPE_BF16 0
#define TQ_DTYPE_F32  1

/* Code widths: 1..4 = Lloyd-Max bits per coordinate; 8 = FP8 E4M3 (keys);
 * TQ_BITS_HALF | b (b in 1..3) = the fractional rate b + 1/2: coordinates
 * 0 .. d/2-1 of the rotated vector take b + 1 bits and coordinates
 * d/2 .. d-1 take b bits, each half with the Lloyd-Max codebook of its width
 * for the same coordinate law (the rotation makes every coordinate follow
 * that law, so the split needs no calibration).  Rates 1.5, 2.5 and 3.5
 * ("What is TurboQuant?": quality-neutral at 3.5 bits per channel, a minor
 * loss at 2.5; community forks ship turboquant25 / turboquant35 presets);
 * the split rule is not on the pages.  16 <= d <= 256; the general kernels
 * serve these rates. */
#define TQ_BITS_FP8 8
#define TQ_BITS_HALF 16
/* TQ_BITS_POLAR: the polar-coordinate angle quantizer of the standalone
 * PolarQuant ("What is TurboQuant?", "Stage 1": vectors mapped to polar
 * coordinates, the angles quantized, no per-vector scale beyond one radius;
 * ai-work-lab overview, PolarQuant section).  After the rotation, level 1
 * turns coordinate pairs (y_2p, y_2p+1) into radii and angles atan2 in
 * [0, 2 pi); each level l = 2 .. log2 d turns pairs of radii (a, b) into
 * sqrt(a^2 + b^2) and psi = atan2(b, a) in [0, pi/2]; the last radius is the
 * stored norm.  Level-1 angles take 4 bits on 16 uniform cells (centres as
 * levels); level-l angles take 2 bits from the Lloyd-Max quantizer of their
 * law for a random direction, density proportional to (sin psi cos psi)^(k-1)
 * with k = 2^(l-1).  The bit allocation (4, 2) is our reading.  Layout: the
 * d/2 level-1 codes as 4-bit fields, then d/2 slots of 2-bit fields holding
 * level 2's d/4 codes, level 3's d/8, ..., level log2 d's one (last slot
 * zero): 3d/8 bytes.  Keys may add QJL on the residual y - y_hat.
 * 8 <= d <= 256; the general kernels serve it (no vector search). */
#define TQ_BITS_POLAR 32

/* ------------------------------------------------------------------------ */
/* Parameters                                                               */
/* ------------------------------------------------------------------------ */
typedef struct tq_params tq_params;   /* opaque, library-owned */

/* Build the data-independent parameters for (d, bits, seed) on the current
 * CUDA device: the sign diagonal D (top bit of SplitMix64 draws, stream 0),
 * the Gaussian matrix S (Box-Muller of SplitMix64 draws, stream 1, rounded
 * to bf16, row-major m x d) and, for bits 1..4, the Lloyd-Max levels and
 * decision boundaries (fp32).  Page: "What is TurboQuant?", "Stage 1" and
 * "Where calibration-free pays off" (the parameters depend on nothing but
 * (d, bits, seed)).
 * d: power of two in [8, 1024]; bits in {1,2,3,4,8} or TQ_BITS_HALF | b
 * (b in 1..3, then 16 <= d <= 256; levels and bounds of the (b + 1)-bit
 * codebook come first, then those of the b-bit one).  *out receives the
 * handle.  Returns TQ_EINVAL / TQ_EUNSUPPORTED on bad arguments, TQ_ENOMEM /
 * TQ_ECUDA on allocation or copy failure.  Synchronous. */
int tq_make_params(int d, int bits, uint64_t seed, tq_params **out);

/* The same parameters computed on the host only (no CUDA call): signs [d],
 * S [d*d] (fp32 holding bf16-exact values), levels [2^bits] and bounds
 * [2^bits - 1] in ascending bucket order (not written for bits = 8).  Any
 * output pointer may be NULL.  Returns TQ_EUNSUPPORTED for bad (d, bits). */
int tq_compute_params_host(int d, int bits, uint64_t seed, int8_t *signs, float *S, float *levels,
                           float *bounds);

/* Rotations.  TQ_ROT_HADAMARD: R = H D / sqrt(d) (tq_make_params).
 * TQ_ROT_DENSE: the dense random rotation ("TurboQuant and RotorQuant on DGX
 * Spark", section on compression quality: TurboQuant's 128 x 128 = 16,384
 * rotation parameters): the d x d matrix of iid N(0,1) entries (Box-Muller of
 * SplitMix64 draws, stream 2) with its rows orthonormalised in order (the Q
 * of the QR factorisation of its transpose with a positive diagonal,
 * transposed), stored in float32 (round to nearest even); under it the norm
 * is n = ||R x|| and the inverse applied to outputs is R^T.  d <= 256.  The
 * cache layout is the same for both. */
#define TQ_ROT_HADAMARD 0
#define TQ_ROT_DENSE 1

/* tq_make_params with a choice of rotation (TQ_ROT_*).  TQ_EUNSUPPORTED for
 * an unknown rotation or TQ_ROT_DENSE with d > 256. */
int tq_make_params_rot(int d, int bits, uint64_t seed, int rotation, tq_params **out);

/* The same matrix computed on the host only (no CUDA call). */
int tq_compute_rotation_host(int d, uint64_t seed, int rotation, float *R);

/* Copy the rotation matrix R (row-major d x d, y = R x) of a handle to R:
 * H D / sqrt(d) in float32 for TQ_ROT_HADAMARD, the stored matrix for
 * TQ_ROT_DENSE. */
int tq_params_export_rotation(const tq_params *p, float *R);

/* Release a handle (NULL is a no-op).  Synchronous. */
void tq_free_params(tq_params *p);

/* Copy the host-side parameters out: signs [d] (+1/-1), S [d*d] (fp32
 * holding bf16-exact values), levels [2^bits] and bounds [2^bits - 1] (fp32;
 * not written for bits = 8).  Any pointer may be NULL. */
int tq_params_export(const tq_params *p, int8_t *signs, float *S, float *levels, float *bounds);

/* ------------------------------------------------------------------------ */
/* Paged compressed cache                                                   */
/* ------------------------------------------------------------------------ */
/* One page holds page_tokens consecutive token slots of one KV head, as a
 * structure of arrays (each array padded to 16 bytes), in this order:
 *   K codes   b-bit fields for kbits in {1,2,4}; a 2-bit array then a 1-bit
 *             array for kbits = 3; d bytes of E4M3 for kbits = 8
 *   K signs   d/8 bytes of QJL sign bits (only if kqjl)
 *   K norm    fp16 ||k||
 *   K rho     fp16 ||residual|| (only if kqjl)
 *   V codes   as K codes with vbits (absent if vbits = 0)
 *   V norm    fp16 ||v|| (absent if vbits = 0)
 * Code fields of one token: coordinate i at bit offset i*w of the token's
 * little-endian byte string.  A fractional rate stores the first half of
 * the coordinates as a (b + 1)-bit code of d/2 coordinates, then the second
 * half as a b-bit code of d/2 coordinates (each by the rules above).  A Lloyd-Max code is stored sign-magnitude:
 * top bit set for the negative half of the levels, low bits the rank of the
 * level's magnitude (0 = smallest).  QJL bit j is 1 iff (S r)_j >= 0.
 * The cache is an array [num_blocks][n_kv_heads] of pages; token slot s lives
 * in block s / page_tokens at position s % page_tokens.
 * Page: "TurboQuant and RotorQuant on DGX Spark", "Two-stage compression"
 * (no per-block scales); the byte layout itself is not on the pages. */
typedef struct {
    int d;            /* head dim, power of two in [8, 1024]              */
    int kbits;        /* 1..4 Lloyd-Max, 8 = FP8 E4M3, or TQ_BITS_HALF|b   */
    int kqjl;         /* 1: QJL sign bits + residual norm (not FP8 keys)   */
    int vbits;        /* 1..4, TQ_BITS_HALF|b, or 0 = no value fields      */
    int page_tokens;  /* multiple of 8, 8..256                             */
    int n_kv_heads;   /* >= 1                                              */
} tq_cache_desc;

/* Bytes of one page (one block of one KV head) under *desc. */
int tq_cache_bytes(const tq_cache_desc *desc, size_t *page_bytes);

/* ------------------------------------------------------------------------ */
/* Encode (write path)                                                      */
/* ------------------------------------------------------------------------ */
/* Compress n_tokens new tokens into the cache.  K, V: device
 * [n_tokens][n_kv_heads][d] of in_dtype (V ignored and may be NULL when
 * vbits = 0).  slot_mapping: device int32 [n_tokens]; a negative slot skips
 * the token; a slot >= num_blocks * page_tokens skips it and sets
 * TQ_DEV_SLOT_RANGE.  kp / vp: parameters with kp->bits == kbits,
 * vp->bits == vbits (vp may be NULL when vbits = 0), both of dimension d.
 * Per vector: n = ||x||, y = R x, codes = bucket(y / n), nhat = fp16(n);
 * QJL keys additionally rho = fp16(||y - nhat c[code]||) and signs of S r;
 * FP8 keys store e4m3(sqrt(d) y / n).  Pages: "What is TurboQuant?",
 * "Stage 1", "Stage 2", vLLM presets; ai-work-lab "QJL".
 * workspace: device, >= tq_encode_workspace_bytes(desc, n_tokens) bytes,
 * 256-byte aligned. */
size_t tq_encode_workspace_bytes(const tq_cache_desc *desc, int64_t n_tokens);
int tq_encode(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc,
              const void *K, const void *V, int in_dtype, int64_t n_tokens,
              const int32_t *slot_mapping, void *cache, int64_t num_blocks,
              void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* Decode attention (one new query token per sequence, GQA)                 */
/* ------------------------------------------------------------------------ */
/* Q: device bf16 [B][Hq][d]; q-head h reads kv-head h / (Hq / n_kv_heads).
 * block_table: device int32 [B][max_blocks]; seq_lens: device int32 [B]
 * (the cache already holds the current token).  out: device bf16 [B][Hq][d].
 * lse (optional, device fp32 [B][Hq]): natural-log softmax denominator of
 * the scaled logits.  logits (optional, device fp32 [B][Hq][logits_stride]):
 * the scaled logits of positions < seq_len.  Logit of key t:
 *   (nhat_t <Rq, c[code_t]> + rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1>) / sqrt(d)
 * then softmax and o = R_v^T sum_t p_t nhat_v,t c_v[code_v,t], bf16 (RNE).
 * Pages: "What is TurboQuant?" ("Stage 2": unbiased inner products; the 8x
 * attention-logit figure), ai-work-lab overview (attention on compressed
 * keys).  FP8 keys (kbits = 8, preset k8v4) score nhat <Rq, e4m3(code)> / sqrt(d)
 * ("What is TurboQuant?", vLLM presets: k8v4 = FP8 keys + 4-bit values).
 * workspace: >= tq_decode_workspace_bytes(desc, B, Hq, max_seq_len). */
size_t tq_decode_workspace_bytes(const tq_cache_desc *desc, int B, int Hq, int max_seq_len);
int tq_decode_attn(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc,
                   const void *Q, int B, int Hq, const int32_t *block_table, int max_blocks,
                   const int32_t *seq_lens, int max_seq_len, const void *cache,
                   int64_t num_blocks, void *out, float *lse, float *logits,
                   int64_t logits_stride, void *workspace, size_t workspace_bytes,
                   void *stream);

/* One decode step with the new token's write fused in: for every sequence b,
 * K_new/V_new [B][n_kv_heads][d] (device, bf16) are compressed into cache
 * slot slot_mapping[b] (< 0 skips the write; >= num_blocks * page_tokens
 * skips it and sets TQ_DEV_SLOT_RANGE), exactly as tq_encode would, and then
 * the queries Q attend over seq_lens[b] tokens that include it, exactly as
 * tq_decode_attn.  The write shares the launch that prepares the queries
 * (a warp per vector; QJL signs from an fp32 projection by S), so the step
 * takes the same three launches as tq_decode_attn alone.  Pages: "What is
 * TurboQuant?" (the cache dtype is chosen per vLLM preset and the serving
 * engine writes each new token as it decodes; "vLLM: available by switching
 * --kv-cache-dtype").  Workspace: tq_decode_workspace_bytes(desc, B, Hq,
 * max_seq_len). */
int tq_decode_step(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc, const void *K_new,
                   const void *V_new, const int32_t *slot_mapping, const void *Q, int B, int Hq,
                   const int32_t *block_table, int max_blocks, const int32_t *seq_lens, int max_seq_len,
                   void *cache, int64_t num_blocks, void *out, float *lse, float *logits,
                   int64_t logits_stride, void *workspace, size_t workspace_bytes, void *stream);

/* Decode attention without any device allocation, for callers that cannot
 * allocate device memory (an engine that keeps all device memory in its own
 * pool and forbids other allocations, a plug-in handed only one call's
 * tensors, a latency-critical path that cannot afford a blocking cudaMalloc).
 * The pages describe no counterpart: this is a library convenience.  Same
 * arguments and results as tq_decode_attn minus the workspace, which is
 * replaced by a file-scope device array of TQ_NOALLOC_SCRATCH_BYTES bytes
 * that every GPU loading the library holds until the process exits.
 * - Sizes whose tq_decode_workspace_bytes exceeds TQ_NOALLOC_SCRATCH_BYTES
 *   are rejected with TQ_ESCRATCH before anything is launched.
 * - No cudaMalloc, cudaFree or allocating library routine is called.
 * - The first call on a device looks up the array's device address with that
 *   device current (cudaGetSymbolAddress) and caches it; make that first call
 *   before any stream capture.
 * - All calls on a device share the array, which keeps the last call's
 *   contents; the status word at its start is cleared at the start of every
 *   call and read back by tq_noalloc_read_status.  Calls whose execution
 *   overlaps on the GPU (different streams, or streams without an ordering
 *   between them) race on the array and give undefined results. */
#define TQ_NOALLOC_SCRATCH_BYTES (16u << 20)
int tq_decode_attn_noalloc(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc,
                           const void *Q, int B, int Hq, const int32_t *block_table, int max_blocks,
                           const int32_t *seq_lens, int max_seq_len, const void *cache,
                           int64_t num_blocks, void *out, float *lse, float *logits,
                           int64_t logits_stride, void *stream);

/* The device status word (TQ_DEV_* bits) left by the last
 * tq_decode_attn_noalloc on the current device, copied to *flags and
 * cleared, as tq_read_status does for a workspace (a slot or block out of
 * range, a wait that timed out: results invalid).  Orders after the work on
 * `stream` and synchronizes it.  Allocates nothing; like the entry point it
 * follows, it looks up the array's device address on first use. */
int tq_noalloc_read_status(void *stream, uint32_t *flags);

/* ------------------------------------------------------------------------ */
/* Chunked prefill over the compressed cache (one sequence)                 */
/* ------------------------------------------------------------------------ */
/* The sequence's cache (block_table: device int32 [max_blocks]) holds
 * seq_len tokens whose last C are the chunk.  Q: device bf16 [C][Hq][d];
 * chunk query j sees positions < seq_len - C + j + 1 (causal inside the
 * chunk, the whole earlier cache).  out: device bf16 [C][Hq][d]; lse
 * optional fp32 [C][Hq].  Logits as tq_decode_attn.  Page: "What is
 * TurboQuant?" (long-prefill workloads bound vLLM's throughput range). */
size_t tq_prefill_workspace_bytes(const tq_cache_desc *desc, int C, int Hq, int seq_len);
int tq_prefill_attn(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc,
                    const void *Q, int C, int Hq, const int32_t *block_table, int max_blocks,
                    int seq_len, const void *cache, int64_t num_blocks, void *out, float *lse,
                    void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* Compressed inner-product search                                          */
/* ------------------------------------------------------------------------ */
/* The database is a cache with n_kv_heads = 1 and vbits = 0 whose slots
 * 0..n_db-1 hold the vectors (written by tq_encode with slots 0..n_db-1).
 * Q: device fp32 [n_q][d].  For every query, the k largest estimates
 *   nhat_t <Rq, c[code_t]> (+ rho_t sqrt(pi/2)/m <S R q, 2 s_t - 1>)
 * over t < n_db, sorted descending, ties to the lower index: top_scores fp32
 * [n_q][k], top_idx int64 [n_q][k].  k in 1..64.  Page: ai-work-lab
 * overview ("also applies to vector search; no index preprocessing").
 * workspace: >= tq_score_workspace_bytes(desc, n_db, n_q, k). */
size_t tq_score_workspace_bytes(const tq_cache_desc *desc, int64_t n_db, int n_q, int k);
int tq_score(const tq_params *p, const tq_cache_desc *desc, const void *db_cache, int64_t n_db,
             const float *Q, int n_q, int k, float *top_scores, int64_t *top_idx,
             void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* Status                                                                   */
/* ------------------------------------------------------------------------ */
/* Copy the device status word of a workspace to *flags (TQ_DEV_* bits) and
 * clear it.  Synchronizes the stream. */
int tq_read_status(void *workspace, void *stream, uint32_t *flags);

/* Static description of a status code. */
const char *tq_status_string(int status);

/* ------------------------------------------------------------------------ */
/* Testing aid                                                              */
/* ------------------------------------------------------------------------ */
/* Make the next tq_decode_attn launch of the tensor-core decode kernel
 * (d = 128, 64-token pages, Lloyd-Max keys with QJL) start every block with a
 * wait of `polls` polls on an on-chip barrier that nothing completes.  The
 * wait runs out before any copy or tensor-core operation is issued, the
 * blocks take their time-out path (no further copies, results written as
 * empty) and the workspace status word gets TQ_DEV_WAIT_TIMEOUT.  It exists
 * so that the time-out path can be exercised without a fault; polls = 0
 * cancels a pending request.  The pages describe no counterpart. */
int tq_test_stall_next_decode(uint32_t polls);

#ifdef __cplusplus
}
#endif
#endif /* TQKV_H */
