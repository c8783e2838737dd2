/*
 * fp8vit.h -- C ABI of libfp8vit.so, the B200 (sm_100a) FP8 vision-encoder
 * attention path.
 *
 * What the path computes (web sources cited by title and section):
 *   - vLLM docs "FP8 ViT Encoder Attention", intro and Usage: BF16 Q/K/V are
 *     quantized to FP8 e4m3 with one scale per tensor right before the
 *     attention call.  Without a scale file the scale is dynamic: a 16-entry
 *     circular buffer of the observed Q/K/V amax drives the per-forward
 *     scale.  With a scale file (section "Scale File Format", saved with the
 *     --mm-encoder-fp8-scale-save-margin of 1.5) the scales are static.
 *     Packed variable-length image batches attend without crossing images.
 *   - vLLM issue "[Feature]: Add support for fused fp8 output to FlashAttention
 *     3", Description: an output_scale argument makes attention write FP8.
 *   - atrex-bench "#025 per_token_group_quant_fp8", Reference Implementation:
 *     the per-token-group quantizer that feeds an FP8 o-proj.
 *
 * Conventions (every entry point):
 *   - A pointer named d_* is DEVICE memory, allocated and owned by the caller.
 *     The library allocates device memory only in fp8vit_create (its context
 *     scratch) and nothing per call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Device work is enqueued asynchronously on it; the call returns
 *     after the launch.
 *   - BF16 tensors are uint16_t bit patterns; FP8 tensors are uint8_t e4m3fn
 *     codes (OCP E4M3: bias 7, max +-448, no infinities, NaN = S.1111.111).
 *   - Activation layout: packed [T, H, D] row-major (== [T, H*D]); T counts
 *     the tokens of all images.
 *   - "descale" is the dequantisation multiplier of a per-tensor FP8 tensor:
 *     value ~= code * descale, descale = max(amax / 448, 1e-10) (the group
 *     quantizer page calls the same quantity "scales").
 *   - Host-side argument checks return at once with FP8VIT_EINVAL (null or
 *     misaligned pointer, negative or overflowing size) or
 *     FP8VIT_EUNSUPPORTED (a shape the kernels do not implement).  Faults the
 *     GPU detects (bad cu_seqlens, a bounded wait that timed out) are
 *     recorded in the context's device status word; fp8vit_check() returns
 *     the first one.
 */
#ifndef FP8VIT_H
#define FP8VIT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8VIT_OK = 0,
    FP8VIT_EINVAL = 1,       /* bad argument (host) or bad cu_seqlens (device)      */
    FP8VIT_EUNSUPPORTED = 2, /* shape/mode not implemented (e.g. head_dim not 72/128) */
    FP8VIT_ECUDA = 3,        /* a CUDA runtime/driver call failed                    */
    FP8VIT_EIO = 4,          /* scale file could not be opened/written               */
    FP8VIT_EPARSE = 5,       /* scale file is not the documented JSON format          */
    FP8VIT_ENOTFOUND = 6,    /* layer name absent from the scale file                */
    FP8VIT_ETIMEOUT = 7      /* a bounded wait inside a kernel gave up                */
} fp8vit_status;

typedef struct fp8vit_ctx fp8vit_ctx;

/* ---- context ------------------------------------------------------------ */

/* Create a context on CUDA device `device` (made current by the call).  The
 * context owns a device status word and the amax reduction scratch used by
 * fp8_amax_ring_update.  One context must not be used by two streams at the
 * same time (the scratch is shared).  *out is NULL on failure. */
fp8vit_status fp8vit_create(int32_t device, fp8vit_ctx** out);

/* Free the context's device memory.  NULL is accepted. */
fp8vit_status fp8vit_destroy(fp8vit_ctx* ctx);

/* Synchronize `stream`, then return and clear the first fault recorded on the
 * device since the last check (FP8VIT_OK if none).  *site, if not NULL,
 * receives a kernel-specific location code of that fault (0 if none).  After
 * a fault it also resets the context's amax reduction state, which a launch
 * that gave up can leave half-updated. */
fp8vit_status fp8vit_check(fp8vit_ctx* ctx, void* stream, int32_t* site);

const char* fp8vit_status_string(fp8vit_status s);

/* Failure injection for tests, on the host side: record on the context an
 * arrival that never happens, so that the next fp8_amax_ring_quantize_qkv on
 * it cannot complete its grid barrier.  Each of that launch's blocks gives up
 * after its bounded 2 s wait and returns; fp8vit_check then reports
 * FP8VIT_ETIMEOUT (site 200) and resets the context's reduction state, after
 * which the context works normally.  No GPU fault is involved.  Synchronizes
 * `stream`.  Not for production use. */
fp8vit_status fp8vit_inject_lost_arrival(fp8vit_ctx* ctx, void* stream);

/* Failure injection for tests: attention launches on this context
 * (fp8_varlen_attn_fwd and its variants) never announce their first tile of
 * scores, so each CTA's softmax warps give up after their bounded 2 s wait;
 * the kernel then stops its other roles, drains its copies and MMAs, frees
 * TMEM and returns.  The injection stays set until fp8vit_check returns the
 * fault it causes: FP8VIT_ETIMEOUT (site 113, the softmax wait for the
 * scores, or the issuer's wait that starves with it: 114, the FP8 kernel's
 * wait for the first tile's P, 119, the BF16 kernel's wait for the score
 * buffer to be released; whichever gives up first); that check clears it together with the status
 * word.  A check with no attention launch in between leaves it set.  No GPU
 * fault is involved.  Synchronizes `stream`.  Not for production use. */
fp8vit_status fp8vit_inject_attn_timeout(fp8vit_ctx* ctx, void* stream);

/* The context keeps the TMA tensor maps its attention launches encode
 * (keyed by base pointer, rows, row bytes and box rows; 12 entries, replaced
 * round-robin), so a layer that reuses its buffers encodes them once.  The
 * counts of launches' map lookups served from the cache and encoded anew.
 * Host only. */
fp8vit_status fp8vit_tmap_cache_stats(fp8vit_ctx* ctx, uint64_t* hits, uint64_t* misses);

/* How many e4m3 terms the probabilities P of fp8_varlen_attn_fwd are kept in
 * for the PV product on this context (both run on the FP8 tensor cores):
 *   2 (the default): P = hi + lo, hi = e4m3(p), lo = e4m3(p - hi), two PV
 *     MMAs into one fp32 accumulator; about 8 significant bits of P.  This is
 *     the mode that meets the attention tolerance (max-abs 3e-2 over the BF16
 *     rounding, mean-abs 3e-3, cosine 0.999) on inputs with x8 outlier
 *     channels.
 *   1: P = e4m3(p) alone, 3 significant bits; one PV MMA and a cheaper
 *     softmax (12-18 % less attention time).  On the same inputs its max-abs
 *     error is 3-4x the 3e-2 tolerance on images of a few hundred tokens and
 *     just inside it on images of 8192 and more (mean-abs and cosine stay
 *     inside the tolerance).
 * Other values: FP8VIT_EINVAL.  Host only; affects later launches. */
fp8vit_status fp8vit_set_attn_p_terms(fp8vit_ctx* ctx, int32_t terms);

/* Library ABI version (major * 100 + minor). */
int32_t fp8vit_version(void);

/* ---- dynamic scaling: amax ring (vLLM "FP8 ViT Encoder Attention", Usage) --- */

/* Size in bytes of one ring state: float hist[3][16] (rows q, k, v), then an
 * int32 write position shared by the three rows, padded to 256 bytes. */
#define FP8VIT_RING_BYTES 256

/* Zero a ring state (all slots 0, position 0) on `stream`. */
fp8vit_status fp8vit_ring_init(void* d_ring, void* stream);

/* One forward of dynamic scaling for q, k and v in a single launch:
 *   amax_t = max |x_t| over all n_elems elements of tensor t (exact);
 *   hist[t][pos] = amax_t for t = q, k, v;  pos = (pos + 1) mod 16;
 *   d_descale3[t] = max(max_j hist[t][j] / 448, 1e-10)   (fp32 division).
 * The current forward's amax is in the ring before its scale is taken.
 * d_q, d_k, d_v: BF16 [n_elems], 16-byte aligned.  d_ring: FP8VIT_RING_BYTES
 * bytes, 16-byte aligned.  d_descale3: float[3] written.  Nothing returns to
 * the host (no synchronisation). */
fp8vit_status fp8_amax_ring_update(fp8vit_ctx* ctx, const uint16_t* d_q, const uint16_t* d_k,
                                   const uint16_t* d_v, int64_t n_elems, void* d_ring,
                                   float* d_descale3, void* stream);

/* The two halves of fp8_amax_ring_update, for a packed batch split across
 * GPUs (each GPU holds some of the images): every rank runs fp8_amax3 on its
 * share, the ranks all-reduce the three values with max (e.g. NCCL), and each
 * runs fp8_ring_push with the result, so all ranks quantize with the same
 * per-tensor descales.  fp8_amax3 followed by fp8_ring_push on one GPU gives
 * bit for bit what fp8_amax_ring_update gives.
 *   fp8_amax3: d_amax3[t] = max |x_t| over n_elems BF16 elements (fp32,
 *     exact), t = q, k, v.  Same argument rules as fp8_amax_ring_update.
 *   fp8_ring_push: the ring rule of fp8_amax_ring_update applied to the
 *     three device values d_amax3 (one thread; writes d_ring and d_descale3). */
fp8vit_status fp8_amax3(fp8vit_ctx* ctx, const uint16_t* d_q, const uint16_t* d_k,
                        const uint16_t* d_v, int64_t n_elems, float* d_amax3, void* stream);
fp8vit_status fp8_ring_push(const float* d_amax3, void* d_ring, float* d_descale3,
                            void* stream);

/* Same computation and arguments as fp8_amax_ring_update, for callers that
 * cannot allocate device memory where they run (for example a process whose
 * memory pool already holds nearly all free HBM, code that must avoid
 * cudaMalloc's device-wide synchronisation, or a caller with no place to keep
 * a context, since fp8vit_create allocates).  The pages describe no such
 * entry point; it has no counterpart there.
 *   - Takes no context and allocates nothing: its 128 bytes of scratch come
 *     from a 256-byte array built into the library's device image, which
 *     every GPU that loads the library keeps until the process exits.  The
 *     scratch need does not grow with n_elems; that it fits the array is
 *     checked when the library is compiled.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it for the life of the process; make
 *     that first call before any stream capture on the device.  The cached
 *     address must not outlive the device's primary context: after
 *     cudaDeviceReset on a device, do not call this entry point on it again
 *     in the same process.
 *   - Devices numbered 64 or above are refused with FP8VIT_EUNSUPPORTED (the
 *     per-device address cache has 64 slots).
 *   - Every call on a device shares the one array: each call clears it with
 *     a 128-byte memset on `stream` before its kernel.  Calls whose work
 *     overlaps on the GPU (different streams, no ordering) race on it and
 *     give wrong maxima; order such calls, or use the context entry point.
 * Returns FP8VIT_EINVAL for the same argument errors as fp8_amax_ring_update. */
fp8vit_status fp8_amax_ring_update_noalloc(const uint16_t* d_q, const uint16_t* d_k,
                                           const uint16_t* d_v, int64_t n_elems, void* d_ring,
                                           float* d_descale3, void* stream);

/* Host helper for the calibrate-once workflow (vLLM "FP8 ViT Encoder
 * Attention", "Calibrate-Once, Reuse Workflow"): synchronize `stream`, copy
 * the ring state to the host and return max_j hist[t][j] for t = q, k, v. */
fp8vit_status fp8_ring_read_amax(const void* d_ring, float out_amax3[3], void* stream);

/* ---- per-tensor quantization (vLLM "FP8 ViT Encoder Attention", intro) ---- */

/* x8 = e4m3_rn_satfinite(float(x) / descale_t) for t = q, k, v, with an IEEE
 * fp32 division, round-to-nearest-even and saturation to +-448.  d_descale3:
 * float[3] (q, k, v) in device memory, e.g. from fp8_amax_ring_update or the
 * static scales.  Inputs BF16 [n_elems] 16-byte aligned; outputs e4m3 codes
 * [n_elems], 8-byte aligned.  d_q8 may be NULL: Q's codes are then not
 * written (fp8_varlen_attn_fwd_qbf16 quantizes Q in its prologue). */
fp8vit_status fp8_quantize_qkv_per_tensor(fp8vit_ctx* ctx, const uint16_t* d_q,
                                          const uint16_t* d_k, const uint16_t* d_v,
                                          int64_t n_elems, const float* d_descale3, uint8_t* d_q8,
                                          uint8_t* d_k8, uint8_t* d_v8, void* stream);

/* The dynamic-scale path in one launch (vLLM "FP8 ViT Encoder Attention":
 * Usage, dynamic scaling; intro: Q/K/V quantized right before attention):
 * exactly fp8_amax_ring_update(d_q, d_k, d_v, n_elems, d_ring, d_descale3)
 * followed by fp8_quantize_qkv_per_tensor(..., d_descale3, d_q8, d_k8,
 * d_v8): the same ring update, descales and codes, bit for bit.  Up to
 * about twice the L2 size of BF16 inputs, one kernel is launched
 * cooperatively (all its blocks resident at once) and meets at a grid
 * barrier between the amax and the quantization, so the scale stages cost no
 * extra launch and part of the second read of the inputs comes from L2;
 * larger tensors take those two calls' kernels, which stream HBM faster
 * without the barrier.  A barrier wait that exceeds 2 s records
 * FP8VIT_ETIMEOUT (read it with fp8vit_check) and leaves the codes unwritten.
 * Alignment and ownership as the two calls; uses the context's scratch (one
 * stream per context at a time).  d_q8 may be NULL (Q's amax still enters
 * the ring; its codes are left to fp8_varlen_attn_fwd_qbf16). */
fp8vit_status fp8_amax_ring_quantize_qkv(fp8vit_ctx* ctx, const uint16_t* d_q,
                                         const uint16_t* d_k, const uint16_t* d_v,
                                         int64_t n_elems, void* d_ring, float* d_descale3,
                                         uint8_t* d_q8, uint8_t* d_k8, uint8_t* d_v8,
                                         void* stream);

/* ---- varlen FP8 attention (vLLM "FP8 ViT Encoder Attention"; vLLM issue
 *      "fused fp8 output for FlashAttention 3") ------------------------------ */

/* Non-causal attention over cu_seqlens-packed images, FP8 QK^T and PV on the
 * tensor cores with fp32 accumulation and online softmax:
 *   for each image i, head h and query row r of image i:
 *     s_j = softmax_scale * dq * dk * <q8[r,h,:], k8[j,h,:]>   (keys j of image i)
 *     o[r,h,:] = sum_j softmax(s)_j * dv * v8[j,h,:]
 * d_q8, d_k8, d_v8: e4m3 [total_tokens, num_heads, head_dim], 16-byte aligned.
 * d_q_descale, d_k_descale, d_v_descale: one float each, device memory.
 * d_cu_seqlens: int32 [num_seqs + 1], non-decreasing, cu[num_seqs] <=
 *   total_tokens, every image length <= max_seqlen (checked on the device;
 *   a violation records FP8VIT_EINVAL and skips that image).  Images of
 *   length 0 are allowed.
 * head_dim: 72 or 128 (others: FP8VIT_EUNSUPPORTED).  Any num_heads >= 1.
 * out_dtype 0: d_out is BF16 [total_tokens, num_heads, head_dim] and
 *   d_output_scale must be NULL.
 * out_dtype 1: d_out is e4m3 [same shape], out = e4m3_rn_satfinite(o /
 *   *d_output_scale), d_output_scale a device float.
 * Rows of d_out outside [cu[0], cu[num_seqs]) are not written. */
fp8vit_status fp8_varlen_attn_fwd(fp8vit_ctx* ctx, const uint8_t* d_q8, const uint8_t* d_k8,
                                  const uint8_t* d_v8, const float* d_q_descale,
                                  const float* d_k_descale, const float* d_v_descale,
                                  const int32_t* d_cu_seqlens, int32_t num_seqs,
                                  int32_t max_seqlen, int64_t total_tokens, int32_t num_heads,
                                  int32_t head_dim, float softmax_scale, void* d_out,
                                  int32_t out_dtype, const float* d_output_scale, void* stream);

/* The BF16 attention that the pages compare FP8 against (vLLM "FP8 ViT
 * Encoder Attention", Performance: BF16 vs FP8 attention time), on the same
 * kernel skeleton as fp8_varlen_attn_fwd: QK^T and PV as kind::f16 tcgen05
 * MMAs with fp32 accumulation, P rounded to BF16, online softmax.
 *   o[r,h,:] = sum_j softmax_j(softmax_scale * <q[r,h,:], k[j,h,:]>) v[j,h,:]
 * over the keys j of r's image.  d_q, d_k, d_v, d_out: BF16
 * [total_tokens, num_heads, head_dim], 16-byte aligned; no scales.
 * head_dim 72 or 128 (else FP8VIT_EUNSUPPORTED).  cu_seqlens, checks and
 * faults as fp8_varlen_attn_fwd.  A comparator for the FP8 path; the
 * library's FP8 path does not call it. */
fp8vit_status bf16_varlen_attn_fwd(fp8vit_ctx* ctx, const uint16_t* d_q, const uint16_t* d_k,
                                   const uint16_t* d_v, const int32_t* d_cu_seqlens,
                                   int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
                                   int32_t num_heads, int32_t head_dim, float softmax_scale,
                                   uint16_t* d_out, void* stream);

/* fp8_varlen_attn_fwd with Q given as BF16 d_q [T, H, D] (16-byte aligned):
 * the kernel's prologue divides each query row by *d_q_descale (IEEE fp32)
 * and rounds it to e4m3 (RNE, satfinite) -- the same bytes
 * fp8_quantize_qkv_per_tensor writes -- straight into its shared-memory Q
 * tile, so Q's codes are neither written nor read through memory (vLLM docs
 * "FP8 ViT Encoder Attention": Q/K/V are quantized right before attention;
 * the small-image overhead of separate quantization passes).  Pair it with
 * fp8_quantize_qkv_per_tensor or fp8_amax_ring_quantize_qkv called with
 * d_q8 = NULL (K and V codes only; the amax still covers Q).  Other
 * arguments, checks and faults as fp8_varlen_attn_fwd. */
fp8vit_status fp8_varlen_attn_fwd_qbf16(fp8vit_ctx* ctx, const uint16_t* d_q,
                                        const uint8_t* d_k8, const uint8_t* d_v8,
                                        const float* d_q_descale, const float* d_k_descale,
                                        const float* d_v_descale, const int32_t* d_cu_seqlens,
                                        int32_t num_seqs, int32_t max_seqlen,
                                        int64_t total_tokens, int32_t num_heads,
                                        int32_t head_dim, float softmax_scale, void* d_out,
                                        int32_t out_dtype, const float* d_output_scale,
                                        void* stream);

/* fp8_varlen_attn_fwd with the per-token-group quantizer fused into its
 * epilogue (vLLM issue "fused fp8 output for FlashAttention 3": the output
 * quantization moves into the attention kernel; atrex-bench "#025
 * per_token_group_quant_fp8": group 128, fp32 scales, the o-proj input).
 * head_dim must be 128, so that each 128-column group of a token row of
 * [total_tokens, num_heads * 128] is exactly one head (head_dim 72 groups
 * straddle heads: FP8VIT_EUNSUPPORTED; use
 * fp8_varlen_attn_fwd_bf16_group_quant).  The attention output is rounded to BF16 as
 * fp8_varlen_attn_fwd's out_dtype 0 stores it, then quantized exactly as
 * per_token_group_quant_fp8(group = 128) does: the bytes of d_xq and the bits
 * of d_scales equal those two calls' results, and no BF16 output is written.
 * d_xq: e4m3 [total_tokens, num_heads * 128], 16-byte aligned.
 * d_scales: fp32 [total_tokens, num_heads], 4-byte aligned.
 * Other arguments, checks and faults as fp8_varlen_attn_fwd. */
fp8vit_status fp8_varlen_attn_fwd_group_quant(
    fp8vit_ctx* ctx, const uint8_t* d_q8, const uint8_t* d_k8, const uint8_t* d_v8,
    const float* d_q_descale, const float* d_k_descale, const float* d_v_descale,
    const int32_t* d_cu_seqlens, int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
    int32_t num_heads, int32_t head_dim, float softmax_scale, uint8_t* d_xq, float* d_scales,
    void* stream);

/* fp8_varlen_attn_fwd (BF16 output) and per_token_group_quant_fp8(group =
 * 128) of that output in one launch, for any supported head_dim (72 or 128)
 * with num_heads * head_dim a multiple of 128 (vLLM issue "fused fp8 output
 * for FlashAttention 3": the output quantization moves into the attention
 * call; atrex-bench "#025 per_token_group_quant_fp8": 128-wide groups of a
 * token row, fp32 scales, the o-proj input).  At head_dim 72 a group spans
 * two or three heads, so no single head's CTA holds a group: every CTA
 * stores its BF16 head slice to d_out and counts itself in on the groups its
 * columns touch; the CTA that completes a group (the last of its heads to
 * finish on that query tile) quantizes it for the tile's token rows.  The
 * counters only elect; no CTA waits for another.
 * d_out: BF16 [total_tokens, num_heads * head_dim], 16-byte aligned; holds
 *   fp8_varlen_attn_fwd's out_dtype 0 result on return.
 * d_xq: e4m3 [total_tokens, num_heads * head_dim], 16-byte aligned, and
 * d_scales: fp32 [total_tokens, num_heads * head_dim / 128], 4-byte aligned:
 *   byte for byte and bit for bit what per_token_group_quant_fp8(d_out, 128)
 *   writes.
 * d_tile_counters: uint32 workspace of at least
 *   ((total_tokens + 127) / 128 + num_seqs) * (num_heads * head_dim / 128)
 *   entries, all zero before the first call; a completed call leaves them
 *   zero again (the caller zeroes it once, e.g. with cudaMemsetAsync, and
 *   reuses it).  Calls that share a counter buffer must not run concurrently.
 * Returns FP8VIT_EINVAL when num_heads * head_dim is not a multiple of 128
 * or a pointer is null or misaligned, FP8VIT_EUNSUPPORTED for another
 * head_dim.  Other arguments, checks and faults as fp8_varlen_attn_fwd. */
fp8vit_status fp8_varlen_attn_fwd_bf16_group_quant(
    fp8vit_ctx* ctx, const uint8_t* d_q8, const uint8_t* d_k8, const uint8_t* d_v8,
    const float* d_q_descale, const float* d_k_descale, const float* d_v_descale,
    const int32_t* d_cu_seqlens, int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
    int32_t num_heads, int32_t head_dim, float softmax_scale, uint16_t* d_out, uint8_t* d_xq,
    float* d_scales, uint32_t* d_tile_counters, void* stream);

/* ---- per-token-group quantizer (atrex-bench "#025 per_token_group_quant_fp8",
 *      Reference Implementation) --------------------------------------------- */

/* For each row r < m and each group g of `group` consecutive columns of the
 * row-major BF16 matrix d_x [m, n]:
 *   amax = max |x|;  scale = max(amax / 448, 1e-10)  (fp32 division)
 *   d_xq[r, c] = e4m3_rn_satfinite(x[r, c] / scale)  (fp32 division)
 *   d_scales[r, g] = scale                            (fp32, [m, n/group])
 * group in {16, 32, 64, 128, 256}; n % group == 0 (else FP8VIT_EINVAL).
 * d_x 16-byte aligned, d_xq 8-byte aligned, d_scales 4-byte aligned. */
fp8vit_status per_token_group_quant_fp8(fp8vit_ctx* ctx, const uint16_t* d_x, int64_t m,
                                        int64_t n, int32_t group, uint8_t* d_xq,
                                        float* d_scales, void* stream);

/* ---- static scales (vLLM "FP8 ViT Encoder Attention", "Scale File Format"
 *      and the 1.5 save margin) -------------------------------------------- */

/* Read the q, k, v numbers of `layer` from the JSON scale file at `path`:
 *   { "<layer>": {"q": a, "k": b, "v": c}, ... }
 * with "q_scale"/"k_scale"/"v_scale" accepted as aliases (both spellings
 * with different values is FP8VIT_EPARSE).  The numbers are in the amax
 * domain (margin x observed amax); fp8_descale_from_amax turns one into a
 * descale.  A negative value, or one that is not finite as fp32, is
 * FP8VIT_EPARSE.  Host only; no CUDA call. */
fp8vit_status fp8_static_scales_load(const char* path, const char* layer, float out_qkv[3]);

/* Write the scale file for n_layers layers: layer i gets
 * {"q": margin*qkv_amax[3i], "k": margin*qkv_amax[3i+1], "v": margin*qkv_amax[3i+2]}
 * (fp32 products, printed so they read back exactly).  Host only. */
fp8vit_status fp8_static_scales_save(const char* path, int32_t n_layers,
                                     const char* const* layers, const float* qkv_amax,
                                     float margin);

/* max(v / 448, 1e-10) in fp32: the descale for a value v of the amax domain. */
float fp8_descale_from_amax(float v);

/* The descale of an observed amax with the save margin applied here
 * (vLLM "FP8 ViT Encoder Attention": the margin multiplies the calibrated
 * amax when the scales are saved): fp8_descale_from_amax(fp32(margin *
 * amax)), the same fp32 product fp8_static_scales_save writes, so that
 * scales taken this way equal those of a saved and reloaded file. */
float fp8_descale_from_amax_margin(float amax, float margin);

#ifdef __cplusplus
}
#endif

#endif /* FP8VIT_H */
