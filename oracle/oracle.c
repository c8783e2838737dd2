/*
 * oracle.c -- the CPU oracle for the FP8 vision-encoder attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
 * statement of what the path computes.  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark may load it.  It shares no code,
 * header, table or constant generator with the CUDA library, and it includes
 * nothing from it.
 *
 * Sources (web pages; cited by title and section):
 *   [vLLM-FP8ViT]  vLLM docs, "FP8 ViT Encoder Attention":
 *                  intro (Q/K/V quantized to FP8 right before the attention
 *                  call), Usage (dynamic scaling: a 16-entry circular buffer
 *                  of observed Q/K/V amax drives the per-forward scale),
 *                  Calibrate-Once workflow + save margin (default 1.5),
 *                  Scale File Format.
 *   [atrex-025]    atrex-bench operator #025 "per_token_group_quant_fp8",
 *                  Reference Implementation.
 *   [vLLM-29920]   vLLM issue "[Feature]: Add support for fused fp8 output to
 *                  FlashAttention 3", Description (output_scale parameter).
 *
 * Readings of points the pages leave open (each one is also listed with its
 * reasoning in the design notes):
 *   R1  e4m3 = OCP FP8 E4M3 "fn" (torch.float8_e4m3fn, whose finfo max 448 the
 *       group quantizer uses); conversion rounds to nearest, ties to even.
 *   R2  finite values beyond +-448 saturate to +-448 (the group quantizer
 *       clamps to +-fp8_max before the cast; the per-tensor path does the same).
 *   R3  x / scale is an IEEE fp32 division (the group quantizer divides in
 *       fp32 after x.float()).
 *   R4  ring: the current forward's amax is written into the ring first, then
 *       the scale is taken from the max over all 16 slots; empty slots are 0.
 *   R5  scale floor 1e-10 (the group quantizer's clamp) is reused for the
 *       per-tensor scale.
 *   R6  scale-file numbers are in the amax domain (margin x amax); the
 *       dequantisation scale is value / 448.
 *   R7  attention is non-causal and confined to one cu_seqlens segment.
 *   Nomenclature: "descale" = the dequantisation multiplier = amax / 448, the
 *   quantity [atrex-025] calls "scales".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_E4M3_MAX 448.0
#define ORC_SCALE_FLOOR 1e-10f
#define ORC_RING_SLOTS 16

/* ------------------------------------------------------------------------ */
/* e4m3 codec (R1, R2)                                                       */
/* ------------------------------------------------------------------------ */

/* Decode one e4m3fn code from the format definition: 1 sign bit, 4 exponent
 * bits (bias 7), 3 mantissa bits; exponent field 0 is subnormal
 * (mantissa/8 * 2^-6); S.1111.111 is NaN; there is no infinity. */
double orc_e4m3_decode(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return sign ? -NAN : NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round a float onto the e4m3 grid: nearest value, ties to the even code,
 * finite magnitudes above 448 saturate to 448, the sign is kept (so -0 and
 * negative values that round to zero give 0x80).  NaN gives 0x7F/0xFF. */
uint8_t orc_e4m3_encode(float f) {
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (isnan(f)) return (uint8_t)(sign | 0x7F);
    if (a >= ORC_E4M3_MAX) return (uint8_t)(sign | 0x7E); /* saturate */
    if (a < 0.015625) {                                   /* below 2^-6   */
        /* subnormal grid: multiples of 2^-9; 8 * 2^-9 is the smallest normal
         * (code 0x08), so rounding up into it needs no special case. */
        double k = rint(a * 512.0); /* exact scaling; rint is ties-to-even */
        return (uint8_t)(sign | (uint8_t)k);
    }
    int e2;
    double fr = frexp(a, &e2); /* a = fr * 2^e2, fr in [0.5, 1) */
    int ex = e2 - 1;           /* a = s * 2^ex, s in [1, 2)      */
    double s = fr * 2.0;
    double mant = rint((s - 1.0) * 8.0); /* exact; ties to even */
    if (mant == 8.0) {
        mant = 0.0;
        ex += 1;
    }
    /* a < 448 and the carry above keep (ex, mant) <= (8, 6) == 448. */
    return (uint8_t)(sign | (uint8_t)(((ex + 7) << 3) | (int)mant));
}

void orc_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}

void orc_e4m3_decode_array(const uint8_t* codes, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(codes[i]);
}

/* ------------------------------------------------------------------------ */
/* bf16                                                                      */
/* ------------------------------------------------------------------------ */

float orc_bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to bfloat16 (nearest, ties to even) in one step; used only
 * to express the reference output in the kernel's output type when a test
 * wants the bf16 rounding floor of the exact result. */
uint16_t orc_double_to_bf16(double d) {
    if (isnan(d)) return 0x7FC0;
    if (d == 0.0) return signbit(d) ? 0x8000 : 0x0000;
    int e2;
    double fr = frexp(fabs(d), &e2);           /* |d| = fr * 2^e2 */
    double r = ldexp(rint(ldexp(fr, 8)), e2 - 8); /* 8 significant bits */
    float f = (float)r;                        /* exact unless out of range */
    if (signbit(d)) f = -f;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* amax, ring buffer and scale rules   [vLLM-FP8ViT] Usage; R4, R5, R6       */
/* ------------------------------------------------------------------------ */

/* amax(x) = max |x| over the whole packed tensor (all tokens, heads, images). */
float orc_amax_bf16(const uint16_t* x, int64_t n) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(orc_bf16_to_float(x[i]));
        if (a > m) m = a;
    }
    return m;
}

/* descale = max(v / 448, 1e-10), v in the amax domain, fp32 division. */
float orc_descale_from_amax(float v) {
    float d = v / 448.0f;
    return d > ORC_SCALE_FLOOR ? d : ORC_SCALE_FLOOR;
}

/* One dynamic-scaling forward for the three tensors q, k, v:
 * hist[t][pos] = amax[t]; pos = (pos + 1) mod 16;
 * descale[t] = max(max_j hist[t][j] / 448, 1e-10).
 * hist is float[3][16] (row t = tensor), pos is the shared write position. */
void orc_ring_update(float* hist, int32_t* pos, const float* amax3, float* descale3) {
    int32_t p = *pos;
    for (int t = 0; t < 3; ++t) hist[t * ORC_RING_SLOTS + p] = amax3[t];
    *pos = (p + 1) % ORC_RING_SLOTS;
    for (int t = 0; t < 3; ++t) {
        float m = 0.0f;
        for (int j = 0; j < ORC_RING_SLOTS; ++j) {
            float h = hist[t * ORC_RING_SLOTS + j];
            if (h > m) m = h;
        }
        descale3[t] = orc_descale_from_amax(m);
    }
}

/* x8 = e4m3(fp32(x) / descale) for one whole tensor (per-tensor scaling). */
void orc_quantize_per_tensor(const uint16_t* x, int64_t n, float descale, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(orc_bf16_to_float(x[i]) / descale);
}

/* ------------------------------------------------------------------------ */
/* per-token-group quantizer   [atrex-025] Reference Implementation          */
/* ------------------------------------------------------------------------ */

/* For each row r and each group g of `group` consecutive columns:
 *   amax = max |x| over the group (fp32)
 *   scale = max(amax / 448, 1e-10)               (fp32 division, then clamp)
 *   q = e4m3(clamp(x / scale, -448, 448))        (fp32 division)
 * scales is [m, n/group] row-major.  Returns 0, or -1 if n % group != 0. */
int orc_group_quant(const uint16_t* x, int64_t m, int64_t n, int32_t group, uint8_t* xq,
                    float* scales) {
    if (group <= 0 || n % group != 0) return -1;
    int64_t ng = n / group;
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t g = 0; g < ng; ++g) {
            const uint16_t* xs = x + r * n + g * group;
            float amax = 0.0f;
            for (int32_t i = 0; i < group; ++i) {
                float a = fabsf(orc_bf16_to_float(xs[i]));
                if (a > amax) amax = a;
            }
            float s = amax / 448.0f;
            if (s < ORC_SCALE_FLOOR) s = ORC_SCALE_FLOOR;
            scales[r * ng + g] = s;
            for (int32_t i = 0; i < group; ++i) {
                float y = orc_bf16_to_float(xs[i]) / s;
                if (y > 448.0f) y = 448.0f;
                if (y < -448.0f) y = -448.0f;
                xq[r * n + g * group + i] = orc_e4m3_encode(y);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* fp64 varlen attention over the dequantised FP8 tensors  [vLLM-FP8ViT] R7 */
/* ------------------------------------------------------------------------ */

/* Locate the segment holding token t: the i with cu[i] <= t < cu[i+1].
 * Returns -1 if t lies outside [cu[0], cu[num_seqs]). */
static int32_t orc_segment_of(const int32_t* cu, int32_t num_seqs, int64_t t) {
    for (int32_t i = 0; i < num_seqs; ++i)
        if (t >= cu[i] && t < cu[i + 1]) return i;
    return -1;
}

/* Exact attention for a list of (token, head) pairs.
 * q8, k8, v8: e4m3 codes, packed [T, H, D].  dq, dk, dv: per-tensor descales.
 * For token t in segment [a, b) and head h:
 *   s_j = sm_scale * sum_d (dq*q8[t,h,d]) * (dk*k8[j,h,d])   for a <= j < b
 *   p_j = exp(s_j - max_j s_j) / sum_j exp(s_j - max_j s_j)
 *   o[d] = sum_j p_j * (dv*v8[j,h,d])
 * all in fp64.  out is [n_pairs, D].  psum (optional, [n_pairs]) receives
 * sum_j p_j for invariant checks.  Returns 0, or -1 on a bad token/head. */
int orc_attn_pairs(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, float dq, float dk,
                   float dv, const int32_t* cu_seqlens, int32_t num_seqs, int32_t H, int32_t D,
                   float sm_scale, const int64_t* tokens, const int32_t* heads, int64_t n_pairs,
                   double* out, double* psum) {
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = orc_e4m3_decode((uint8_t)c);
    int32_t max_len = 0;
    for (int32_t i = 0; i < num_seqs; ++i) {
        int32_t len = cu_seqlens[i + 1] - cu_seqlens[i];
        if (len > max_len) max_len = len;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    if (!s || !qv) {
        free(s);
        free(qv);
        return -2;
    }
    const int64_t row = (int64_t)H * D;
    int rc = 0;
    for (int64_t n = 0; n < n_pairs; ++n) {
        int64_t t = tokens[n];
        int32_t h = heads[n];
        int32_t seg = orc_segment_of(cu_seqlens, num_seqs, t);
        if (seg < 0 || h < 0 || h >= H) {
            rc = -1;
            break;
        }
        int64_t a = cu_seqlens[seg], b = cu_seqlens[seg + 1];
        for (int32_t d = 0; d < D; ++d) qv[d] = table[q8[t * row + (int64_t)h * D + d]] * (double)dq;
        double smax = -INFINITY;
        for (int64_t j = a; j < b; ++j) {
            const uint8_t* kj = k8 + j * row + (int64_t)h * D;
            double acc = 0.0;
            for (int32_t d = 0; d < D; ++d) acc += qv[d] * (table[kj[d]] * (double)dk);
            s[j - a] = (double)sm_scale * acc;
            if (s[j - a] > smax) smax = s[j - a];
        }
        double l = 0.0;
        for (int64_t j = a; j < b; ++j) {
            s[j - a] = exp(s[j - a] - smax);
            l += s[j - a];
        }
        double* o = out + n * D;
        for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
        for (int64_t j = a; j < b; ++j) {
            const uint8_t* vj = v8 + j * row + (int64_t)h * D;
            double p = s[j - a] / l;
            for (int32_t d = 0; d < D; ++d) o[d] += p * (table[vj[d]] * (double)dv);
        }
        if (psum) {
            double ps = 0.0;
            for (int64_t j = a; j < b; ++j) ps += s[j - a] / l;
            psum[n] = ps;
        }
    }
    free(s);
    free(qv);
    return rc;
}

/* Whole-tensor attention: every token of every segment, every head.
 * out is [T, H, D] with T = cu_seqlens[num_seqs]. */
int orc_attn_full(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, float dq, float dk,
                  float dv, const int32_t* cu_seqlens, int32_t num_seqs, int32_t H, int32_t D,
                  float sm_scale, double* out) {
    int64_t T = cu_seqlens[num_seqs];
    int64_t np = (int64_t)(T - cu_seqlens[0]) * H;
    int64_t* toks = (int64_t*)malloc(sizeof(int64_t) * (size_t)(np > 0 ? np : 1));
    int32_t* hs = (int32_t*)malloc(sizeof(int32_t) * (size_t)(np > 0 ? np : 1));
    if (!toks || !hs) {
        free(toks);
        free(hs);
        return -2;
    }
    int64_t n = 0;
    for (int64_t t = cu_seqlens[0]; t < T; ++t)
        for (int32_t h = 0; h < H; ++h) {
            toks[n] = t;
            hs[n] = h;
            ++n;
        }
    int rc = orc_attn_pairs(q8, k8, v8, dq, dk, dv, cu_seqlens, num_seqs, H, D, sm_scale, toks,
                            hs, np, out + (int64_t)cu_seqlens[0] * H * D, NULL);
    free(toks);
    free(hs);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* fp64 varlen attention over BF16 tensors: the BF16 side of the pages'     */
/* BF16-vs-FP8 attention comparison [vLLM-FP8ViT, Performance]             */
/* ------------------------------------------------------------------------ */

/* As orc_attn_pairs, with q, k, v given as BF16 bit patterns [T, H, D] and no
 * descales: s_j = sm_scale * sum_d q[t,h,d] * k[j,h,d]; p = softmax(s);
 * o[d] = sum_j p_j * v[j,h,d]; all in fp64. */
int orc_attn_pairs_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const int32_t* cu_seqlens, int32_t num_seqs, int32_t H, int32_t D,
                        float sm_scale, const int64_t* tokens, const int32_t* heads,
                        int64_t n_pairs, double* out, double* psum) {
    int32_t max_len = 0;
    for (int32_t i = 0; i < num_seqs; ++i) {
        int32_t len = cu_seqlens[i + 1] - cu_seqlens[i];
        if (len > max_len) max_len = len;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    if (!s || !qv) {
        free(s);
        free(qv);
        return -2;
    }
    const int64_t row = (int64_t)H * D;
    int rc = 0;
    for (int64_t n = 0; n < n_pairs; ++n) {
        int64_t t = tokens[n];
        int32_t h = heads[n];
        int32_t seg = orc_segment_of(cu_seqlens, num_seqs, t);
        if (seg < 0 || h < 0 || h >= H) {
            rc = -1;
            break;
        }
        int64_t a = cu_seqlens[seg], b = cu_seqlens[seg + 1];
        for (int32_t d = 0; d < D; ++d)
            qv[d] = (double)orc_bf16_to_float(q[t * row + (int64_t)h * D + d]);
        double smax = -INFINITY;
        for (int64_t j = a; j < b; ++j) {
            const uint16_t* kj = k + j * row + (int64_t)h * D;
            double acc = 0.0;
            for (int32_t d = 0; d < D; ++d) acc += qv[d] * (double)orc_bf16_to_float(kj[d]);
            s[j - a] = (double)sm_scale * acc;
            if (s[j - a] > smax) smax = s[j - a];
        }
        double l = 0.0;
        for (int64_t j = a; j < b; ++j) {
            s[j - a] = exp(s[j - a] - smax);
            l += s[j - a];
        }
        double* o = out + n * D;
        for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
        for (int64_t j = a; j < b; ++j) {
            const uint16_t* vj = v + j * row + (int64_t)h * D;
            double p = s[j - a] / l;
            for (int32_t d = 0; d < D; ++d) o[d] += p * (double)orc_bf16_to_float(vj[d]);
        }
        if (psum) {
            double ps = 0.0;
            for (int64_t j = a; j < b; ++j) ps += s[j - a] / l;
            psum[n] = ps;
        }
    }
    free(s);
    free(qv);
    return rc;
}

/* FP8 output reference [vLLM-29920]: out8 = e4m3(float(o) / output_scale). */
void orc_fp8_output(const double* o, int64_t n, float output_scale, uint8_t* out8) {
    for (int64_t i = 0; i < n; ++i) out8[i] = orc_e4m3_encode((float)o[i] / output_scale);
}
