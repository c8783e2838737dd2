// Non-causal varlen FP8 flash attention for sm_100a (vLLM docs "FP8 ViT
// Encoder Attention": per-tensor FP8 Q/K/V, packed images attend only within
// themselves; vLLM issue "fused fp8 output for FlashAttention 3": an
// output_scale epilogue that writes e4m3).
//
// One CTA = one (image, head, 128-row query tile).  Warp roles:
//   warp 0      TMA producer: Q once, then K/V tiles of BN keys (64 at
//               head_dim 128, 96 at head_dim 72) into an NS-stage
//               shared-memory ring (SWIZZLE_32B, 32-byte boxes).
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer:
//               S = Q K^T (kind::f8f6f4, K-major A and B) into the TMEM S
//               buffer, O += P V (A = P from TMEM, B = V MN-major from
//               smem).  S(j+1) is issued as soon as the softmax warps have
//               copied S(j) into registers, so it is computed while they
//               work on tile j; P has TMEM columns of its own, so the next
//               QK never waits for the previous PV.  TMEM (256 columns, two
//               CTAs per SM): head_dim 128 has S 64 + two P slots of 32 + O
//               128; head_dim 72 has S 96 + one P slot of 48 + O 80, and its
//               softmax computes P(j) in registers and stores it once PV(j-1)
//               has read the slot.
//   warps 2..5  softmax + epilogue, one query row per thread (TMEM lane):
//               row max, exp2, row sum in registers; P written to its TMEM
//               slot as two e4m3 terms (hi + lo) so that the PV product
//               keeps ~8 mantissa bits while running on FP8 tensor cores; O
//               is rescaled in TMEM when the row max rises (after P is
//               written, when the previous PV has long completed).
// head_dim 72 is padded inside the kernel: the QK contraction runs over 96
// bytes starting at the head's offset rounded down to 16 bytes (TMA needs a
// 16-byte aligned x coordinate); bytes of the window outside the head are
// zeroed in Q, so the neighbouring head's K bytes contribute exactly 0.  PV
// runs with N = 80 and the epilogue picks the head's 72 columns.
// Epilogues (one per instance): BF16 o; e4m3 o / output_scale; at head_dim
// 128 the per-token-group quantizer on each head's row (a group is a head);
// and, with tile counters, the BF16 instance's group tail, where the CTA that
// completes a 128-column group across heads quantizes it (group_tail below).
#include <math.h>

#include <atomic>
#include <type_traits>

#include "attn_common.cuh"

namespace {

using namespace fp8vit_attn;

constexpr int kBM = 128;          // query rows per CTA (MMA M)
constexpr int kThreads = 192;     // 6 warps
constexpr int kTmemCols = 256;
constexpr int kQTileBytes = kBox * kBM;   // one [128 rows x 32 B] Q box
constexpr uint64_t kTimeoutNs = 2000000000ull;
// P is stored as 2^(x - m_ref + kPLog2); a tile max up to kSlackLog2 above the
// reference max keeps P <= 2^(6 + 2.75) = 430 < 448 (e4m3 max).
constexpr float kPLog2 = 6.0f;
constexpr float kSlackLog2 = 2.75f;
// head_dim 128 trades one binade of P's low end (values below 2^-11 of the
// reference max turn e4m3-subnormal one binade earlier) for a wider slack,
// 2^(5 + 3.75) = 430 as well: fewer O rescales (measured faster at 128,
// slower at 72).
constexpr float kPLog2D128 = 5.0f;
constexpr float kSlackLog2D128 = 3.75f;

template <int D>
struct Cfg;
template <>
struct Cfg<72> {
    static constexpr int KB = 3;    // 32-byte k-blocks of the QK contraction (96 bytes)
    static constexpr int VA = 3;    // 32-byte V column blocks loaded (96 bytes)
    static constexpr int NPV = 80;  // PV MMA N (covers head bytes [0,72) or [8,80))
    static constexpr int NS = 5;    // K/V pipeline stages
    static constexpr int BN = 96;   // keys per KV tile (QK MMA N, PV MMA K)
    static constexpr int PSLOTS = 1;
    // TMEM columns: S [0, 96), one P slot [96, 144), O [144, 224)
    static constexpr uint32_t TS = 0, TP = 96, TO = 144;
};
template <>
struct Cfg<128> {
    static constexpr int KB = 4;
    static constexpr int VA = 4;
    static constexpr int NPV = 128;
    static constexpr int NS = 4;
    static constexpr int BN = 64;
    static constexpr int PSLOTS = 2;
    // TMEM columns: S [0, 64), P slots [64 + 32b, 96 + 32b), O [128, 256)
    static constexpr uint32_t TS = 0, TP = 64, TO = 128;
};

// BF16 inputs (the same skeleton with kind::f16 MMAs): a 32-byte box column
// holds 16 elements, so the QK contraction takes KB = 8 k-blocks at
// head_dim 128 and 5 at head_dim 72 (a 160-byte window over the head's 144
// bytes; its last 16 bytes are zeroed in Q), V takes VA atoms of 16
// columns, and one PV MMA covers 16 keys.  P (BF16) occupies the same TMEM
// columns as the two e4m3 terms.  Stages: what two CTAs per SM leave room for.
template <int D>
struct CfgB;
template <>
struct CfgB<72> {
    static constexpr int KB = 5, VA = 5, NPV = 80, NS = 3, BN = 96, PSLOTS = 1;
    static constexpr uint32_t TS = 0, TP = 96, TO = 144;
};
template <>
struct CfgB<128> {
    static constexpr int KB = 8, VA = 8, NPV = 128, NS = 2, BN = 64, PSLOTS = 2;
    static constexpr uint32_t TS = 0, TP = 64, TO = 128;
};

template <class C>
struct SmemOf {
    static constexpr int Q = 0;
    static constexpr int K = Q + C::KB * kQTileBytes;
    static constexpr int KVT = kBox * C::BN;  // one [BN rows x 32 B] K or V box
    static constexpr int V = K + C::NS * C::KB * KVT;
    static constexpr int BAR = V + C::NS * C::VA * KVT;
    static constexpr int TOTAL = BAR + 256;
    static constexpr int ALLOC = TOTAL + 1024;  // slack for 1024-byte alignment
};
template <int D>
using Smem = SmemOf<Cfg<D>>;
template <int D, bool BF>
using CfgOf = std::conditional_t<BF, CfgB<D>, Cfg<D>>;


// D[tmem] (+)= A * B, kind::f16 (both operands bf16), issued by one thread;
// A from shared memory (descriptor) or from TMEM.
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}



// Four fp32 values that are exact in e4m3 -> their four codes in one word
// (first value in byte 0), by the 4-wide conversion; its rounding (rbits = 0:
// toward zero) never applies to exact values.
__device__ __forceinline__ uint32_t e4m3x4_exact(float a, float b, float c, float d) {
    uint32_t r;
    asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%4, %3, %2, %1}, %5;"
        : "=r"(r)
        : "f"(a), "f"(b), "f"(c), "f"(d), "r"(0u));
    return r;
}

// Four fp32 -> four e4m3 codes (RNE, satfinite), first value in byte 0.
__device__ __forceinline__ uint32_t e4m3x4_rn(float a, float b, float c, float d) {
    return (uint32_t)f32x2_to_e4m3x2(a, b) | ((uint32_t)f32x2_to_e4m3x2(c, d) << 16);
}

// Probabilities of one 32-key chunk: p = 2^(s * c - bias) (a score of -inf
// gives 0), summed into the two packed accumulators, then written as e4m3
// words pk[0..7] (hi) and pk[8..15] (lo), key 4i+k in byte k of word i, with
// hi + lo ~= p to ~8 significant bits, so that the PV product on FP8 tensor
// cores keeps about a BF16-width P.  hi = p with its fp32 mantissa cut to 3
// bits (a mask; exact in e4m3 wherever p is e4m3-normal, and the P scaling
// keeps the significant probabilities there), lo = RN_e4m3(p - hi) with
// p - hi exact in fp32: the only rounding, of lo, is to nearest, so the pair
// carries no bias and its error is below 2^-7 p.  Per four probabilities:
// four masks, two packed subtracts, one 4-wide conversion for hi and two
// 2-wide conversions for lo (no f16 round trip).
template <bool PLO>
__device__ __forceinline__ void p_chunk(const uint32_t (&r)[32], uint64_t c2, uint64_t nb2,
                                        uint64_t& l0, uint64_t& l1, uint32_t (&pk)[16]) {
    float p[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float x0, x1;
        f2unpack(ffma2(f2pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), c2, nb2),
                 x0, x1);
        p[2 * i] = ex2_approx(x0);
        p[2 * i + 1] = ex2_approx(x1);
    }
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        l0 = fadd2(l0, f2pack(p[2 * i], p[2 * i + 1]));
        l1 = fadd2(l1, f2pack(p[2 * i + 2], p[2 * i + 3]));
    }
    if constexpr (!PLO) {
        // single e4m3 term: P rounded once, straight from fp32
#pragma unroll
        for (int w = 0; w < 8; ++w)
            pk[w] = e4m3x4_rn(p[4 * w], p[4 * w + 1], p[4 * w + 2], p[4 * w + 3]);
    } else {
        const uint64_t m1 = f2pack(-1.0f, -1.0f);
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            float hf[4], lf[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                hf[i] = __uint_as_float(__float_as_uint(p[4 * w + i]) & 0xFFF00000u);
            f2unpack(ffma2(f2pack(hf[0], hf[1]), m1, f2pack(p[4 * w], p[4 * w + 1])), lf[0], lf[1]);
            f2unpack(ffma2(f2pack(hf[2], hf[3]), m1, f2pack(p[4 * w + 2], p[4 * w + 3])), lf[2],
                     lf[3]);
            pk[w] = e4m3x4_exact(hf[0], hf[1], hf[2], hf[3]);
            pk[8 + w] = e4m3x4_rn(lf[0], lf[1], lf[2], lf[3]);
        }
    }
}

// One chunk's P words into TMEM: hi in the first 8 columns, lo (when kept)
// in the next 8.
template <bool PLO>
__device__ __forceinline__ void tmem_st_p(uint32_t taddr, const uint32_t (&pk)[16]) {
    if constexpr (PLO) {
        tmem_st16(taddr, pk);
    } else {
        uint32_t hi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) hi[i] = pk[i];
        tmem_st8(taddr, hi);
    }
}

// P of one 64-key tile written to a 32-column P slot: chunk c (keys
// 32c..32c+31) goes to columns [16c, 16c+8) (hi) and [16c+8, 16c+16) (lo).
// Returns the tile's probability sum.
template <bool PLO>
__device__ __forceinline__ float tile_p(const uint32_t (&a)[32], const uint32_t (&b)[32],
                                        uint32_t tPb, uint64_t c2, uint64_t nb2) {
    uint32_t pk[16];
    uint64_t l0 = f2pack(0.0f, 0.0f), l1 = l0;
    p_chunk<PLO>(a, c2, nb2, l0, l1, pk);
    tmem_st_p<PLO>(tPb, pk);
    p_chunk<PLO>(b, c2, nb2, l0, l1, pk);
    tmem_st_p<PLO>(tPb + 16, pk);
    float s0, s1;
    f2unpack(fadd2(l0, l1), s0, s1);
    return s0 + s1;
}

// BF16 probabilities of one 32-key chunk: p = 2^(s * c - bias), summed into
// the packed accumulators, rounded to bf16 (RNE) two per word (key 2w in the
// low half), 16 words = TMEM columns [0, 16) of the chunk.
__device__ __forceinline__ void p_chunk_bf16(const uint32_t (&r)[32], uint64_t c2, uint64_t nb2,
                                             uint64_t& l0, uint64_t& l1, uint32_t (&pk)[16]) {
    float p[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float x0, x1;
        f2unpack(ffma2(f2pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), c2, nb2),
                 x0, x1);
        p[2 * i] = ex2_approx(x0);
        p[2 * i + 1] = ex2_approx(x1);
    }
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        l0 = fadd2(l0, f2pack(p[2 * i], p[2 * i + 1]));
        l1 = fadd2(l1, f2pack(p[2 * i + 2], p[2 * i + 3]));
    }
#pragma unroll
    for (int w = 0; w < 16; ++w) {
        __nv_bfloat162 b = __floats2bfloat162_rn(p[2 * w], p[2 * w + 1]);
        pk[w] = *reinterpret_cast<uint32_t*>(&b);
    }
}

// P chunk into TMEM for either input type; returns nothing, sums accumulate.
template <bool BF, bool PLO>
__device__ __forceinline__ void p_chunk_any(const uint32_t (&r)[32], uint64_t c2, uint64_t nb2,
                                            uint64_t& l0, uint64_t& l1, uint32_t (&pk)[16]) {
    if constexpr (BF) p_chunk_bf16(r, c2, nb2, l0, l1, pk);
    else p_chunk<PLO>(r, c2, nb2, l0, l1, pk);
}
template <bool BF, bool PLO>
__device__ __forceinline__ void tmem_st_p_any(uint32_t taddr, const uint32_t (&pk)[16]) {
    if constexpr (BF) tmem_st16(taddr, pk);
    else tmem_st_p<PLO>(taddr, pk);
}


// Group tail of the bf16-output kernel, run when it is given tile counters (atrex-bench "#025 per_token_group_quant_fp8":
// 128-wide groups of a token row, fp32 scale = amax / 448, codes of x / scale;
// vLLM issue "fused fp8 output for FlashAttention 3": the o-proj input is
// produced by the attention call).  When a 128-column group spans several
// heads (head_dim 72: 16 heads are 9 groups, each spanning 2 or 3 heads) no
// single head CTA holds a whole group, so each CTA stores its bf16 head slice
// as usual and then counts itself in on every group its columns touch; the
// CTA whose arrival completes a group (its last head to finish) quantizes
// that group's column block for the tile's token rows.  Nobody waits on
// another CTA: the counters only elect who runs each group, then reset for
// the next launch.  A block is 128 rows x 256 bytes, read back (L2-hot) with
// all of its loads issued at once: each half warp takes a token row, 8 values
// a lane, with the arithmetic of group_quant_kernel (same helpers), so codes
// and scales equal those of per_token_group_quant_fp8 over the stored output.
constexpr int kTailRowsPerPass = kThreads / 16;                          // half warps
constexpr int kTailRowSlots = (kBM + kTailRowsPerPass - 1) / kTailRowsPerPass;

template <int D>
__device__ __noinline__ void group_tail(volatile uint32_t* elect, volatile int32_t* abort_flag,
                                        uint32_t* tile_cnt, int seg, int32_t seg_start,
                                        int32_t seg_len, int qt, int h, int num_heads,
                                        const uint16_t* out, uint8_t* xq, float* gscales) {
    const int tid = threadIdx.x;
    const int ncol = num_heads * D, ngr = ncol >> 7;
    // groups this head's columns [h*D, h*D + D) touch
    const int g0 = (h * D) >> 7, g1 = (h * D + D - 1) >> 7;
    if (tid == 0) {
        // Every CTA of the tile arrives exactly once per launch (the error
        // paths too), so each count returns to zero with its last arrival.
        // Tiles are numbered seg_start / 128 + qt + seg: distinct across
        // segments because cu_seqlens is a cumulative sum.
        uint32_t* cnt = tile_cnt + (int64_t)((seg_start >> 7) + qt + seg) * ngr;
        __threadfence();  // this CTA's bf16 stores (ordered by the barrier above)
        uint32_t mine = 0;
        for (int g = g0; g <= g1; ++g) {
            // heads whose columns meet [128 g, 128 g + 128)
            const uint32_t heads = (uint32_t)(min(128 * g + 127, ncol - 1) / D - (128 * g) / D + 1);
            if (atomicAdd(cnt + g, 1u) == heads - 1) {
                atomicExch(cnt + g, 0u);
                mine |= 1u << (g - g0);
            }
        }
        if (mine) __threadfence();  // the other heads' stores, before the reads below
        *elect = *abort_flag == 0 ? mine : 0u;
    }
    __syncthreads();
    const uint32_t mine = *elect;
    if (!mine) return;

    const int q0 = qt * kBM;
    const int rows = min(kBM, seg_len - q0);
    const int64_t tok0 = (int64_t)seg_start + q0;
    const int hw = tid >> 4, l16 = tid & 15;
    for (int g = g0; g <= g1; ++g) {
        if (!((mine >> (g - g0)) & 1u)) continue;
        uint4 x[kTailRowSlots];
#pragma unroll
        for (int u = 0; u < kTailRowSlots; ++u) {
            const int r = u * kTailRowsPerPass + hw;
            x[u] = r < rows ? __ldcg(reinterpret_cast<const uint4*>(out + (tok0 + r) * ncol +
                                                                    g * 128) + l16)
                            : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kTailRowSlots; ++u) {
            const int r = u * kTailRowsPerPass + hw;
            uint32_t a = __vmaxu2(__vmaxu2(x[u].x & 0x7FFF7FFFu, x[u].y & 0x7FFF7FFFu),
                                  __vmaxu2(x[u].z & 0x7FFF7FFFu, x[u].w & 0x7FFF7FFFu));
            a = max(a & 0xFFFFu, a >> 16);
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
            const float sc = group_scale_of_amax(bf16_bits_to_f32(a));
            const float nr = -__frcp_rn(sc);
            const uint2 q = quant8_small(x[u], f2_pack(sc, sc), f2_pack(nr, nr));
            if (r < rows) {
                const int64_t tok = tok0 + r;
                *reinterpret_cast<uint2*>(xq + tok * ncol + g * 128 + l16 * 8) = q;
                if (l16 == 0) gscales[tok * ngr + g] = sc;
            }
        }
    }
}


// OUT selects the epilogue at compile time; PLO keeps P as two e4m3 terms
// (hi + lo, two PV MMAs) or, when false, as one.  BF: the inputs are BF16
// (no descales) and both products run as kind::f16 MMAs with P in BF16.
// QB: Q arrives as BF16 (qbf) and the prologue quantizes it with the Q
// descale into the e4m3 Q tile (each softmax thread its own row), so the
// per-tensor quantizer need not write or read Q's codes.
template <int D, int OUT, bool PLO, bool BF = false, bool QB = false>
__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ dq_p,
                    const float* __restrict__ dk_p, const float* __restrict__ dv_p,
                    const int32_t* __restrict__ cu, int32_t max_seqlen, int64_t total_tokens,
                    int32_t num_heads, float sm_scale, void* __restrict__ out,
                    const float* __restrict__ out_scale_p, float* __restrict__ gscales,
                    fp8vit_scratch* __restrict__ scr, const uint16_t* __restrict__ qbf,
                    uint8_t* __restrict__ xq, uint32_t* __restrict__ tile_cnt) {
    static_assert(OUT != kOutGroupQ || D == 128, "a 128-wide group is one head at head_dim 128");
    static_assert(!BF || OUT == kOutBf16, "bf16 inputs: bf16 output");
    static_assert(!(BF && QB), "BF16 Q is quantized only on the FP8 path");
    using C = CfgOf<D, BF>;
    using L = SmemOf<C>;
    constexpr int E = BF ? 2 : 1;  // bytes per element
    constexpr int NS = C::NS;

    const int qt = blockIdx.x, h = blockIdx.y, seg = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int32_t seg_start = cu[seg];
    const int32_t seg_end = cu[seg + 1];
    const int32_t seg_len = seg_end - seg_start;
    if (seg_start < 0 || seg_len < 0 || seg_len > max_seqlen || (int64_t)seg_end > total_tokens) {
        if (threadIdx.x == 0 && qt == 0 && h == 0)
            fp8vit_report(scr, FP8VIT_EINVAL, SITE_ATTN_SEQLENS);
        return;
    }
    const int q0 = qt * kBM;
    if (q0 >= seg_len) return;
    const int n_kv = (seg_len + C::BN - 1) / C::BN;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sQ = smem_u32(sm + L::Q);
    const uint32_t sK = smem_u32(sm + L::K);
    const uint32_t sV = smem_u32(sm + L::V);
    const uint32_t bar0 = smem_u32(sm + L::BAR);
    // barrier indices
    // s_full / s_free complete once per tile (phase j & 1): S(j+1) is only
    // issued after s_free(j), which the softmax warps arrive on after
    // waiting for s_full(j), so neither can run two phases ahead of its
    // waiter.  P and PV events come in pairs indexed by the tile's parity
    // (b = j & 1), tile j's event being completion (j >> 1) of barrier b:
    // a waiter for tile j - 1 or j - 2 can never see that barrier two
    // phases ahead, because PV(j) needs P(j), which the waiter writes later.
    const uint32_t b_q_full = bar0 + 8 * 0;
    const uint32_t b_q_ready = bar0 + 8 * 1;
    const uint32_t b_drain = bar0 + 8 * 2;
    const uint32_t b_s_full = bar0 + 8 * 3;                      // S(j) computed
    const uint32_t b_s_free = bar0 + 8 * 4;                      // S(j) copied to registers
    auto b_p_full = [&](int b) { return bar0 + 8 * (5 + b); };   // P(j) written
    auto b_o_ready = [&](int b) { return bar0 + 8 * (7 + b); };  // PV(j) complete
    auto b_kv_full = [&](int s) { return bar0 + 8 * (9 + s); };  // K and V of a stage landed
    auto b_kv_empty = [&](int s) { return bar0 + 8 * (9 + NS + s); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::BAR + 8 * (9 + 2 * NS));
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
    // Group tail (bf16 output with tile counters): the CTA's elected groups, after the TMEM
    // slot and the abort flag.
    volatile uint32_t* elect = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);
    static_assert(8 * (9 + 2 * NS) + 12 <= L::TOTAL - L::BAR, "barrier area");

    if (threadIdx.x == 0) {
        mbar_init(b_q_full, 1);
        mbar_init(b_q_ready, 4);  // one elected arrival per softmax warp
        mbar_init(b_drain, 1);
        mbar_init(b_s_full, 1);
        mbar_init(b_s_free, 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(b_p_full(b), 4);
            mbar_init(b_o_ready(b), 1);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(b_kv_full(s), 1);
            mbar_init(b_kv_empty(s), 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // x coordinate (bytes) of the head's window: head offset rounded down to 16.
    const int32_t x0 = (h * D * E) & ~15;
    const int col_off = (h * D * E - x0) / E;  // 0, or 8 for odd heads at D = 72 (e4m3)

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            if constexpr (!QB) {
                mbar_arrive_expect_tx(b_q_full, C::KB * kQTileBytes);
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_2d(sQ + kb * kQTileBytes, &tm_q, x0 + kBox * kb, seg_start + q0,
                                b_q_full);
            }
            int issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % NS;
                if (j >= NS &&
                    !mbar_wait_bounded(b_kv_empty(s), ((j / NS) - 1) & 1, abort_flag, scr,
                                       SITE_ATTN_WAIT_EMPTY, kTimeoutNs))
                    break;
                const int32_t row = seg_start + j * C::BN;
                mbar_arrive_expect_tx(b_kv_full(s), (C::KB + C::VA) * L::KVT);
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_2d(sK + (s * C::KB + kb) * L::KVT, &tm_k, x0 + kBox * kb, row,
                                b_kv_full(s));
                for (int a = 0; a < C::VA; ++a)
                    tma_load_2d(sV + (s * C::VA + a) * L::KVT, &tm_v, x0 + kBox * a, row,
                                b_kv_full(s));
                ++issued;
            }
            // Drain: every issued copy must land before the CTA may exit.
            if constexpr (!QB) mbar_wait_drain(b_q_full, 0, scr);
            for (int j = issued - 1; j >= 0 && j >= issued - NS; --j)
                mbar_wait_drain(b_kv_full(j % NS), (j / NS) & 1, scr);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // S(j) = Q K_j^T goes to the S buffer.  S(j+1) is issued as soon as
        // the softmax warps have copied S(j) into registers (s_free), before
        // P(j) is waited for, so the tensor cores compute the next scores
        // while the softmax warps work on the current ones.
        if (lane == 0) {
            constexpr uint32_t idesc_qk = BF ? idesc_bf16(C::BN, false) : idesc_e4m3(C::BN, false);
            constexpr uint32_t idesc_pv = BF ? idesc_bf16(C::NPV, true) : idesc_e4m3(C::NPV, true);
            // The issue loop is on the tensor core's critical path: a single
            // thread's scalar work between MMAs is comparable to an MMA, so
            // descriptors are formed once and advanced by constants (one box
            // is KVT >> 4 descriptor address units), and stages and phases
            // are counters instead of divisions.
            constexpr uint64_t kQBox = kQTileBytes >> 4, kKVBox = L::KVT >> 4;
            const uint32_t tO = tmem + C::TO, tS = tmem + C::TS;
            const uint64_t qd = desc_k_sw32(sQ), kd0 = desc_k_sw32(sK);
            const uint64_t vd0 = desc_mn_sw32<L::KVT>(sV);
            const bool skip_first_s = *reinterpret_cast<volatile uint32_t*>(&scr->inject_attn) != 0;
            auto issue_qk = [&](int s) {
                const uint64_t kd = kd0 + (uint64_t)(s * C::KB) * kKVBox;
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb) {
                    if constexpr (BF) umma_bf16_ss(tS, qd + kb * kQBox, kd + kb * kKVBox, idesc_qk, kb > 0 ? 1u : 0u);
                    else umma_f8_ss(tS, qd + kb * kQBox, kd + kb * kKVBox, idesc_qk, kb > 0 ? 1u : 0u);
                }
            };
            bool ok = mbar_wait_bounded(b_q_ready, 0, abort_flag, scr, SITE_ATTN_WAIT_QREADY,
                                        kTimeoutNs);
            bool issued_any = false;
            if (ok) {
                ok = mbar_wait_bounded(b_kv_full(0), 0, abort_flag, scr, SITE_ATTN_WAIT_K,
                                       kTimeoutNs);
                if (ok) {
                    tc_fence_after();
                    issue_qk(0);
                    // test hook (fp8vit_inject_attn_timeout): S(0) is never
                    // announced, so the softmax warps' bounded wait runs out
                    if (!skip_first_s) umma_commit(b_s_full);
                    issued_any = true;
                }
            }
            int sk = NS > 1 ? 1 : 0, sv = 0;  // stages of the next QK and of the next PV
            uint32_t phk = NS > 1 ? 0u : 1u;   // fill phase of stage sk
            for (int j = 0; ok && j < n_kv; ++j) {
                if (j + 1 < n_kv) {
                    if (!mbar_wait_bounded(b_kv_full(sk), phk, abort_flag, scr, SITE_ATTN_WAIT_K,
                                           kTimeoutNs))
                        break;
                    if (!mbar_wait_bounded(b_s_free, j & 1, abort_flag, scr, SITE_ATTN_WAIT_SFREE,
                                           kTimeoutNs))
                        break;
                    tc_fence_after();
                    issue_qk(sk);
                    umma_commit(b_s_full);
                    if (++sk == NS) {
                        sk = 0;
                        phk ^= 1u;
                    }
                }
                // V(j) landed with K(j), which QK(j) waited for.
                if (!mbar_wait_bounded(b_p_full(j & 1), (j >> 1) & 1, abort_flag, scr,
                                       SITE_ATTN_WAIT_P, kTimeoutNs))
                    break;
                tc_fence_after();
                const uint32_t tPb = tmem + C::TP + (C::PSLOTS == 2 ? 32 * (j & 1) : 0);
                const uint64_t vd = vd0 + (uint64_t)(sv * C::VA) * kKVBox;
#pragma unroll
                for (int kk = 0; kk < C::BN / 32; ++kk) {
                    const uint64_t bdesc = vd + (uint64_t)((kk * 32 * kBox) >> 4);
                    if constexpr (BF) {
                        // keys 32kk..32kk+15 at P columns +0, the next 16 keys at +8
                        const uint64_t bdesc2 = vd + (uint64_t)(((kk * 32 + 16) * kBox) >> 4);
                        umma_bf16_ts(tO, tPb + 16 * kk, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                        umma_bf16_ts(tO, tPb + 16 * kk + 8, bdesc2, idesc_pv, 1u);
                    } else {
                        umma_f8_ts(tO, tPb + 16 * kk, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                        if constexpr (PLO) umma_f8_ts(tO, tPb + 16 * kk + 8, bdesc, idesc_pv, 1u);
                    }
                }
                umma_commit(b_o_ready(j & 1));
                umma_commit(b_kv_empty(sv));
                if (++sv == NS) sv = 0;
            }
            // Never leave MMAs in flight: one more commit tracks all of them.
            if (issued_any) {
                umma_commit(b_drain);
                mbar_wait_drain(b_drain, 0, scr);
            }
        }
    } else {
        // ---------------- softmax + epilogue (warps 2..5) ----------------
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // query row in the tile == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tS = lane_base + C::TS, tP = lane_base + C::TP, tO = lane_base + C::TO;
        const float dq = BF ? 1.0f : *dq_p, dk = BF ? 1.0f : *dk_p, dv = BF ? 1.0f : *dv_p;
        const float scale_log2 = sm_scale * dq * dk * 1.4426950408889634f;

        bool ok = true;
        if constexpr (QB) {
            // This row's BF16 Q of the head, divided by the Q descale (IEEE
            // fp32, as the per-tensor quantizer) and rounded to e4m3, into the
            // QK window of KB x 32 bytes: the head at col_off, zeros around
            // it (so the neighbouring head's K bytes contribute exactly 0), and
            // zeros for rows past the image.  SW32 layout as the TMA writes it:
            // row r of k-block kb at kb*4096 + r*32, 16-byte chunk c at c ^ ((r>>2)&1).
            uint32_t wq[C::KB * 8];
#pragma unroll
            for (int i = 0; i < C::KB * 8; ++i) wq[i] = 0;
            if (q0 + row < seg_len) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    qbf + ((int64_t)(seg_start + q0 + row) * num_heads + h) * D);
                const float rq = __frcp_rn(dq);
#pragma unroll
                for (int v = 0; v < D / 8; ++v) {
                    const uint2 c = quant8(__ldg(src + v), dq, rq);
                    if (col_off == 0) {
                        wq[2 * v] = c.x;
                        wq[2 * v + 1] = c.y;
                    } else {
                        wq[2 * v + 2] = c.x;
                        wq[2 * v + 3] = c.y;
                    }
                }
            }
            const int sw = (row >> 2) & 1;
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    *reinterpret_cast<uint4*>(sm + L::Q + kb * kQTileBytes + row * kBox +
                                              ((c ^ sw) << 4)) =
                        make_uint4(wq[8 * kb + 4 * c], wq[8 * kb + 4 * c + 1],
                                   wq[8 * kb + 4 * c + 2], wq[8 * kb + 4 * c + 3]);
        } else {
            ok = mbar_wait_bounded(b_q_full, 0, abort_flag, scr, SITE_ATTN_WAIT_Q, kTimeoutNs);
            ok = __all_sync(0xFFFFFFFFu, ok);
        }
        if (QB) {
            // the Q tile is complete as written above
        } else if (ok && D == 72 && BF) {
            // BF16: the 160-byte window's last 16 bytes (chunk 1 of k-block 4)
            // belong to the next head.
            const int sw = (row >> 2) & 1;
            *reinterpret_cast<uint4*>(sm + L::Q + 4 * kQTileBytes + row * kBox + ((1 ^ sw) << 4)) =
                make_uint4(0, 0, 0, 0);
        } else if (ok && D == 72) {
            // Zero the window bytes outside this head: [72,96) for even heads,
            // [0,8) and [80,96) for odd heads.  SW32 layout: row r of k-block
            // kb at kb*4096 + r*32, 16-byte chunk c stored at chunk c ^ ((r>>2)&1).
            uint8_t* q = sm + L::Q;
            const int sw = (row >> 2) & 1;
            uint8_t* kb2 = q + 2 * kQTileBytes + row * kBox;
            *reinterpret_cast<uint4*>(kb2 + ((1 ^ sw) << 4)) = make_uint4(0, 0, 0, 0);
            if (col_off == 0)
                *reinterpret_cast<uint2*>(kb2 + ((0 ^ sw) << 4) + 8) = make_uint2(0, 0);
            else
                *reinterpret_cast<uint2*>(q + row * kBox + ((0 ^ sw) << 4)) = make_uint2(0, 0);
        }
        fence_proxy_async_smem();
        warp_arrive(b_q_ready, lane);

        // Running state per row, in log2 units of the scaled score
        // (x = s * scale_log2): m_ref is the reference max the exponentials
        // are taken against, l_run the sum of the probabilities written to P.
        // P = 2^(x - m_ref + kPLog2): values up to 2^(kPLog2 + kSlackLog2)
        // stay inside e4m3 (max 448), so O and l are rescaled only when a
        // tile's max exceeds m_ref by more than kSlackLog2 (both are scaled
        // by the same factor, so the final o = O / l is unchanged).
        float m_ref = -INFINITY, l_run = 0.0f;
        constexpr int NCH = C::BN / 32;
        for (int j = 0; ok && j < n_kv; ++j) {
            const int b = j & 1;
            ok = mbar_wait_bounded(b_s_full, j & 1, abort_flag, scr, SITE_ATTN_WAIT_S, kTimeoutNs);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) break;
            tc_fence_after();
            const int nvalid = min(C::BN, seg_len - j * C::BN);
            uint32_t r[NCH][32];
            if constexpr (NCH == 2) {
                tmem_ld64_sync(tS, r[0], r[1]);
            } else {
#pragma unroll
                for (int c = 0; c < NCH; ++c) tmem_ld32(tS + 32 * c, r[c]);
                tmem_wait_ld();
            }
            tc_fence_before();
            warp_arrive(b_s_free, lane);  // the S buffer may take S(j+1) now
            if (nvalid < C::BN) {
                // keys past the segment end score -inf: one code path below
#pragma unroll
                for (int c = 0; c < NCH; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[c][i] = 32 * c + i < nvalid ? r[c][i] : 0xFF800000u;
            }
            const float mx = tile_row_max<NCH>(r);
            const float mxc = mx * scale_log2;
            // j == 0 sets the reference; the first PV initialises O.
            constexpr float slack = (D == 128 && !BF) ? kSlackLog2D128 : kSlackLog2;
            constexpr float plog2 = (D == 128 && !BF) ? kPLog2D128 : kPLog2;
            const bool need = j == 0 || mxc > m_ref + slack;
            const bool rescale = j > 0 && __any_sync(0xFFFFFFFFu, need);
            const float alpha = (j > 0 && need) ? ex2_approx(m_ref - mxc) : 1.0f;
            if (need) m_ref = mxc;
            // P = 2^(x - bias), bias = m_ref - kPLog2
            const float bias = m_ref - plog2;
            const uint64_t c2 = f2pack(scale_log2, scale_log2);
            const uint64_t nb2 = f2pack(-bias, -bias);
            if constexpr (C::PSLOTS == 2) {
                // P slot b held P(j - 2).  PV(j - 2) was issued before QK(j),
                // and the commit that completed s_full(j) tracks every earlier
                // MMA of the issuer, so PV(j - 2) has completed: the slot is free.
                if constexpr (BF) {
                    uint32_t pk[16];
                    uint64_t l0 = f2pack(0.0f, 0.0f), l1 = l0;
                    p_chunk_bf16(r[0], c2, nb2, l0, l1, pk);
                    tmem_st16(tP + 32 * b, pk);
                    p_chunk_bf16(r[1], c2, nb2, l0, l1, pk);
                    tmem_st16(tP + 32 * b + 16, pk);
                    float s0, s1;
                    f2unpack(fadd2(l0, l1), s0, s1);
                    l_run = l_run * alpha + (s0 + s1);
                } else {
                    l_run = l_run * alpha + tile_p<PLO>(r[0], r[1], tP + 32 * b, c2, nb2);
                }
                if (rescale) {
                    // O holds PV(0..j-1): wait for PV(j - 1), then scale it.
                    ok = mbar_wait_bounded(b_o_ready((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag,
                                           scr, SITE_ATTN_WAIT_O, kTimeoutNs);
                    ok = __all_sync(0xFFFFFFFFu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    rescale_o<C::NPV>(tO, alpha);
                }
            } else {
                // One P slot: P(j) is computed in registers, then stored once
                // PV(j - 1) has read P(j - 1) (and completed O for a rescale).
                uint64_t l0 = f2pack(0.0f, 0.0f), l1 = l0;
                uint32_t pk[NCH][16];
#pragma unroll
                for (int c = 0; c < NCH; ++c) p_chunk_any<BF, PLO>(r[c], c2, nb2, l0, l1, pk[c]);
                float s0, s1;
                f2unpack(fadd2(l0, l1), s0, s1);
                l_run = l_run * alpha + (s0 + s1);
                if (j > 0) {
                    ok = mbar_wait_bounded(b_o_ready((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag,
                                           scr, SITE_ATTN_WAIT_O, kTimeoutNs);
                    ok = __all_sync(0xFFFFFFFFu, ok);
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int c = 0; c < NCH; ++c) tmem_st_p_any<BF, PLO>(tP + 16 * c, pk[c]);
                if (rescale) rescale_o<C::NPV>(tO, alpha);
            }
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(b_p_full(b), lane);
        }
        // epilogue
        if (ok) {
            // PV(n_kv - 1)'s commit tracks every earlier MMA of the issuer too.
            ok = mbar_wait_bounded(b_o_ready((n_kv - 1) & 1), ((n_kv - 1) >> 1) & 1, abort_flag,
                                   scr, SITE_ATTN_WAIT_O, kTimeoutNs);
            ok = __all_sync(0xFFFFFFFFu, ok);
        }
        if (ok) {
            tc_fence_after();
            const bool valid = (q0 + row) < seg_len;
            const float inv = __fdiv_rn(dv, l_run);
            const int64_t tok = (int64_t)seg_start + q0 + row;
            const int64_t off = (tok * num_heads + h) * D;
            if constexpr (OUT == kOutGroupQ) {
                // The row's bf16 output values, exactly as the bf16 epilogue
                // would store them, quantized as one group of 128: pass 1 takes
                // their amax, pass 2 reloads O and writes the codes.
                uint32_t am = 0;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const uint4 w = bf16x8_of_o(tO + 8 * c, inv);
                    am = __vmaxu2(am, w.x & 0x7FFF7FFFu);
                    am = __vmaxu2(am, w.y & 0x7FFF7FFFu);
                    am = __vmaxu2(am, w.z & 0x7FFF7FFFu);
                    am = __vmaxu2(am, w.w & 0x7FFF7FFFu);
                }
                am = max(am & 0xFFFFu, am >> 16);
                const float sc = group_scale_of_amax(bf16_bits_to_f32(am));
                const float nr = -__frcp_rn(sc);
                const uint64_t s2 = f2_pack(sc, sc), nr2 = f2_pack(nr, nr);
                uint8_t* xq = reinterpret_cast<uint8_t*>(out) + off;
#pragma unroll
                for (int c = 0; c < D / 8; c += 2) {
                    const uint2 a = quant8_small(bf16x8_of_o(tO + 8 * c, inv), s2, nr2);
                    const uint2 b = quant8_small(bf16x8_of_o(tO + 8 * c + 8, inv), s2, nr2);
                    if (valid)
                        *reinterpret_cast<uint4*>(xq + 8 * c) = make_uint4(a.x, a.y, b.x, b.y);
                }
                if (valid) gscales[tok * num_heads + h] = sc;
            } else {
                const float oscale = OUT == kOutE4m3 ? *out_scale_p : 1.0f;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    uint32_t r[8];
                    tmem_ld8_sync(tO + col_off + 8 * c, r);
                    float o[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) o[i] = __uint_as_float(r[i]) * inv;
                    if (!valid) continue;
                    if constexpr (OUT == kOutE4m3) {
                        uint32_t w0 = (uint32_t)f32x2_to_e4m3x2(__fdiv_rn(o[0], oscale), __fdiv_rn(o[1], oscale)) |
                                      ((uint32_t)f32x2_to_e4m3x2(__fdiv_rn(o[2], oscale), __fdiv_rn(o[3], oscale)) << 16);
                        uint32_t w1 = (uint32_t)f32x2_to_e4m3x2(__fdiv_rn(o[4], oscale), __fdiv_rn(o[5], oscale)) |
                                      ((uint32_t)f32x2_to_e4m3x2(__fdiv_rn(o[6], oscale), __fdiv_rn(o[7], oscale)) << 16);
                        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(out) + off + 8 * c) =
                            make_uint2(w0, w1);
                    } else {
                        uint32_t w[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            __nv_bfloat162 b = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
                            w[i] = *reinterpret_cast<uint32_t*>(&b);
                        }
                        *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + off + 8 * c) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if constexpr (OUT == kOutBf16 && !BF)
        if (tile_cnt)
            group_tail<D>(elect, abort_flag, tile_cnt, seg, seg_start, seg_len, qt, h,
                          num_heads, reinterpret_cast<const uint16_t*>(out), xq, gscales);
}


// qbf non-null: Q is BF16 (the kernel quantizes it with dq in its prologue)
// and q8 is ignored.
template <int D, int OUT>
fp8vit_status launch(fp8vit_ctx* ctx, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                     const float* dq, const float* dk, const float* dv, const int32_t* cu,
                     int32_t num_seqs, int32_t max_seqlen, int64_t T, int32_t H, float sm_scale,
                     void* out, const float* out_scale, float* gscales, cudaStream_t st,
                     const uint16_t* qbf = nullptr, uint8_t* xq = nullptr,
                     uint32_t* tile_cnt = nullptr) {
    CUtensorMap mq, mk, mv;
    const int64_t row_bytes = (int64_t)H * D;
    if (!cached_map(ctx, &mk, k8, T, row_bytes, Cfg<D>::BN) ||
        !cached_map(ctx, &mv, v8, T, row_bytes, Cfg<D>::BN))
        return FP8VIT_ECUDA;
    if (qbf) mq = mk;  // not read by the kernel
    else if (!cached_map(ctx, &mq, q8, T, row_bytes, kBM)) return FP8VIT_ECUDA;
    // The dynamic shared-memory limit is a per-device setting of each kernel
    // instance: raise it once per (device, instance).
    static std::atomic<uint64_t> attr_set[4];
    const bool two_terms = ctx->attn_p_terms != 1;
    const int inst = (two_terms ? 1 : 0) + (qbf ? 2 : 0);
    auto kern = two_terms ? attn_fwd_kernel<D, OUT, true> : attn_fwd_kernel<D, OUT, false>;
    if (qbf)
        kern = two_terms ? attn_fwd_kernel<D, OUT, true, false, true>
                         : attn_fwd_kernel<D, OUT, false, false, true>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP8VIT_ECUDA;
    const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
    if (!bit || !(attr_set[inst].load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Smem<D>::ALLOC) != cudaSuccess)
            return FP8VIT_ECUDA;
        attr_set[inst].fetch_or(bit);
    }
    dim3 grid((unsigned)((max_seqlen + kBM - 1) / kBM), (unsigned)H, (unsigned)num_seqs);
    kern<<<grid, kThreads, Smem<D>::ALLOC, st>>>(mq, mk, mv, dq, dk, dv, cu, max_seqlen, T, H,
                                                 sm_scale, out, out_scale, gscales,
                                                 ctx->d_scratch, qbf, xq, tile_cnt);
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

template <int D>
fp8vit_status launch_bf16(fp8vit_ctx* ctx, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* cu, int32_t num_seqs,
                          int32_t max_seqlen, int64_t T, int32_t H, float sm_scale, void* out,
                          cudaStream_t st) {
    using C = CfgB<D>;
    using L = SmemOf<C>;
    CUtensorMap mq, mk, mv;
    const int64_t row_bytes = (int64_t)H * D * 2;
    if (!cached_map(ctx, &mq, q, T, row_bytes, kBM) || !cached_map(ctx, &mk, k, T, row_bytes, C::BN) ||
        !cached_map(ctx, &mv, v, T, row_bytes, C::BN))
        return FP8VIT_ECUDA;
    static std::atomic<uint64_t> attr_set;
    auto kern = attn_fwd_kernel<D, kOutBf16, true, true>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP8VIT_ECUDA;
    const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
    if (!bit || !(attr_set.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) !=
            cudaSuccess)
            return FP8VIT_ECUDA;
        attr_set.fetch_or(bit);
    }
    dim3 grid((unsigned)((max_seqlen + kBM - 1) / kBM), (unsigned)H, (unsigned)num_seqs);
    kern<<<grid, kThreads, L::ALLOC, st>>>(mq, mk, mv, nullptr, nullptr, nullptr, cu, max_seqlen, T,
                                           H, sm_scale, out, nullptr, nullptr, ctx->d_scratch,
                                           nullptr, nullptr, nullptr);
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}


}  // namespace

extern "C" fp8vit_status fp8_varlen_attn_fwd(
    fp8vit_ctx* ctx, const uint8_t* d_q8, const uint8_t* d_k8, const uint8_t* d_v8,
    const float* d_q_descale, const float* d_k_descale, const float* d_v_descale,
    const int32_t* d_cu_seqlens, int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
    int32_t num_heads, int32_t head_dim, float softmax_scale, void* d_out, int32_t out_dtype,
    const float* d_output_scale, void* stream) {
    if (!ctx || !d_q8 || !d_k8 || !d_v8 || !d_q_descale || !d_k_descale || !d_v_descale ||
        !d_cu_seqlens || !d_out)
        return FP8VIT_EINVAL;
    if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || total_tokens > INT32_MAX ||
        num_heads < 1)
        return FP8VIT_EINVAL;
    if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return FP8VIT_EINVAL;
    if (out_dtype != 0 && out_dtype != 1) return FP8VIT_EINVAL;
    if ((out_dtype == 1) != (d_output_scale != nullptr)) return FP8VIT_EINVAL;
    if (head_dim != 72 && head_dim != 128) return FP8VIT_EUNSUPPORTED;
    if (((int64_t)num_heads * head_dim) % 16 != 0) return FP8VIT_EUNSUPPORTED;
    if (misaligned(d_q8, 16) || misaligned(d_k8, 16) || misaligned(d_v8, 16) ||
        misaligned(d_out, out_dtype == 0 ? 16 : 8) || misaligned(d_cu_seqlens, 4))
        return FP8VIT_EINVAL;
    if (num_heads > 65535 || num_seqs > 65535) return FP8VIT_EUNSUPPORTED;
    if (num_seqs == 0 || max_seqlen == 0 || total_tokens == 0) return FP8VIT_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (head_dim == 72)
        return out_dtype == 0
                   ? launch<72, kOutBf16>(ctx, d_q8, d_k8, d_v8, d_q_descale, d_k_descale,
                                          d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                          total_tokens, num_heads, softmax_scale, d_out, nullptr,
                                          nullptr, st)
                   : launch<72, kOutE4m3>(ctx, d_q8, d_k8, d_v8, d_q_descale, d_k_descale,
                                          d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                          total_tokens, num_heads, softmax_scale, d_out,
                                          d_output_scale, nullptr, st);
    return out_dtype == 0
               ? launch<128, kOutBf16>(ctx, d_q8, d_k8, d_v8, d_q_descale, d_k_descale,
                                       d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                       total_tokens, num_heads, softmax_scale, d_out, nullptr,
                                       nullptr, st)
               : launch<128, kOutE4m3>(ctx, d_q8, d_k8, d_v8, d_q_descale, d_k_descale,
                                       d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                       total_tokens, num_heads, softmax_scale, d_out,
                                       d_output_scale, nullptr, st);
}

extern "C" fp8vit_status fp8_varlen_attn_fwd_qbf16(
    fp8vit_ctx* ctx, const uint16_t* d_q, const uint8_t* d_k8, const uint8_t* d_v8,
    const float* d_q_descale, const float* d_k_descale, const float* d_v_descale,
    const int32_t* d_cu_seqlens, int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
    int32_t num_heads, int32_t head_dim, float softmax_scale, void* d_out, int32_t out_dtype,
    const float* d_output_scale, void* stream) {
    if (!ctx || !d_q || !d_k8 || !d_v8 || !d_q_descale || !d_k_descale || !d_v_descale ||
        !d_cu_seqlens || !d_out)
        return FP8VIT_EINVAL;
    if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || total_tokens > INT32_MAX ||
        num_heads < 1)
        return FP8VIT_EINVAL;
    if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return FP8VIT_EINVAL;
    if (out_dtype != 0 && out_dtype != 1) return FP8VIT_EINVAL;
    if ((out_dtype == 1) != (d_output_scale != nullptr)) return FP8VIT_EINVAL;
    if (head_dim != 72 && head_dim != 128) return FP8VIT_EUNSUPPORTED;
    if (((int64_t)num_heads * head_dim) % 16 != 0) return FP8VIT_EUNSUPPORTED;
    if (misaligned(d_q, 16) || misaligned(d_k8, 16) || misaligned(d_v8, 16) ||
        misaligned(d_out, out_dtype == 0 ? 16 : 8) || misaligned(d_cu_seqlens, 4))
        return FP8VIT_EINVAL;
    if (num_heads > 65535 || num_seqs > 65535) return FP8VIT_EUNSUPPORTED;
    if (num_seqs == 0 || max_seqlen == 0 || total_tokens == 0) return FP8VIT_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (head_dim == 72)
        return out_dtype == 0
                   ? launch<72, kOutBf16>(ctx, nullptr, d_k8, d_v8, d_q_descale, d_k_descale,
                                          d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                          total_tokens, num_heads, softmax_scale, d_out, nullptr,
                                          nullptr, st, d_q)
                   : launch<72, kOutE4m3>(ctx, nullptr, d_k8, d_v8, d_q_descale, d_k_descale,
                                          d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                          total_tokens, num_heads, softmax_scale, d_out,
                                          d_output_scale, nullptr, st, d_q);
    return out_dtype == 0
               ? launch<128, kOutBf16>(ctx, nullptr, d_k8, d_v8, d_q_descale, d_k_descale,
                                       d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                       total_tokens, num_heads, softmax_scale, d_out, nullptr,
                                       nullptr, st, d_q)
               : launch<128, kOutE4m3>(ctx, nullptr, d_k8, d_v8, d_q_descale, d_k_descale,
                                       d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                       total_tokens, num_heads, softmax_scale, d_out,
                                       d_output_scale, nullptr, st, d_q);
}

extern "C" fp8vit_status fp8_varlen_attn_fwd_group_quant(
    fp8vit_ctx* ctx, const uint8_t* d_q8, const uint8_t* d_k8, const uint8_t* d_v8,
    const float* d_q_descale, const float* d_k_descale, const float* d_v_descale,
    const int32_t* d_cu_seqlens, int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
    int32_t num_heads, int32_t head_dim, float softmax_scale, uint8_t* d_xq, float* d_scales,
    void* stream) {
    if (!ctx || !d_q8 || !d_k8 || !d_v8 || !d_q_descale || !d_k_descale || !d_v_descale ||
        !d_cu_seqlens || !d_xq || !d_scales)
        return FP8VIT_EINVAL;
    if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || total_tokens > INT32_MAX ||
        num_heads < 1)
        return FP8VIT_EINVAL;
    if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return FP8VIT_EINVAL;
    if (head_dim != 128) return FP8VIT_EUNSUPPORTED;
    if (misaligned(d_q8, 16) || misaligned(d_k8, 16) || misaligned(d_v8, 16) ||
        misaligned(d_xq, 16) || misaligned(d_scales, 4) || misaligned(d_cu_seqlens, 4))
        return FP8VIT_EINVAL;
    if (num_heads > 65535 || num_seqs > 65535) return FP8VIT_EUNSUPPORTED;
    if (num_seqs == 0 || max_seqlen == 0 || total_tokens == 0) return FP8VIT_OK;
    return launch<128, kOutGroupQ>(ctx, d_q8, d_k8, d_v8, d_q_descale, d_k_descale, d_v_descale,
                                   d_cu_seqlens, num_seqs, max_seqlen, total_tokens, num_heads,
                                   softmax_scale, d_xq, nullptr, d_scales,
                                   reinterpret_cast<cudaStream_t>(stream));
}

extern "C" fp8vit_status fp8_varlen_attn_fwd_bf16_group_quant(
    fp8vit_ctx* ctx, const uint8_t* d_q8, const uint8_t* d_k8, const uint8_t* d_v8,
    const float* d_q_descale, const float* d_k_descale, const float* d_v_descale,
    const int32_t* d_cu_seqlens, int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
    int32_t num_heads, int32_t head_dim, float softmax_scale, uint16_t* d_out, uint8_t* d_xq,
    float* d_scales, uint32_t* d_tile_counters, void* stream) {
    if (!ctx || !d_q8 || !d_k8 || !d_v8 || !d_q_descale || !d_k_descale || !d_v_descale ||
        !d_cu_seqlens || !d_out || !d_xq || !d_scales || !d_tile_counters)
        return FP8VIT_EINVAL;
    if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || total_tokens > INT32_MAX ||
        num_heads < 1)
        return FP8VIT_EINVAL;
    if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return FP8VIT_EINVAL;
    if (head_dim != 72 && head_dim != 128) return FP8VIT_EUNSUPPORTED;
    if (((int64_t)num_heads * head_dim) % 128 != 0) return FP8VIT_EINVAL;
    if (misaligned(d_q8, 16) || misaligned(d_k8, 16) || misaligned(d_v8, 16) ||
        misaligned(d_out, 16) || misaligned(d_xq, 16) || misaligned(d_scales, 4) ||
        misaligned(d_tile_counters, 4) || misaligned(d_cu_seqlens, 4))
        return FP8VIT_EINVAL;
    if (num_heads > 65535 || num_seqs > 65535) return FP8VIT_EUNSUPPORTED;
    if (num_seqs == 0 || max_seqlen == 0 || total_tokens == 0) return FP8VIT_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (head_dim == 72)
        return launch<72, kOutBf16>(ctx, d_q8, d_k8, d_v8, d_q_descale, d_k_descale,
                                          d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                          total_tokens, num_heads, softmax_scale, d_out, nullptr,
                                          d_scales, st, nullptr, d_xq, d_tile_counters);
    return launch<128, kOutBf16>(ctx, d_q8, d_k8, d_v8, d_q_descale, d_k_descale,
                                       d_v_descale, d_cu_seqlens, num_seqs, max_seqlen,
                                       total_tokens, num_heads, softmax_scale, d_out, nullptr,
                                       d_scales, st, nullptr, d_xq, d_tile_counters);
}

extern "C" fp8vit_status bf16_varlen_attn_fwd(fp8vit_ctx* ctx, const uint16_t* d_q,
                                              const uint16_t* d_k, const uint16_t* d_v,
                                              const int32_t* d_cu_seqlens, int32_t num_seqs,
                                              int32_t max_seqlen, int64_t total_tokens,
                                              int32_t num_heads, int32_t head_dim,
                                              float softmax_scale, uint16_t* d_out,
                                              void* stream) {
    if (!ctx || !d_q || !d_k || !d_v || !d_cu_seqlens || !d_out) return FP8VIT_EINVAL;
    if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || total_tokens > INT32_MAX ||
        num_heads < 1)
        return FP8VIT_EINVAL;
    if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return FP8VIT_EINVAL;
    if (head_dim != 72 && head_dim != 128) return FP8VIT_EUNSUPPORTED;
    if (misaligned(d_q, 16) || misaligned(d_k, 16) || misaligned(d_v, 16) ||
        misaligned(d_out, 16) || misaligned(d_cu_seqlens, 4))
        return FP8VIT_EINVAL;
    if (num_heads > 65535 || num_seqs > 65535) return FP8VIT_EUNSUPPORTED;
    if (num_seqs == 0 || max_seqlen == 0 || total_tokens == 0) return FP8VIT_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (head_dim == 72)
        return launch_bf16<72>(ctx, d_q, d_k, d_v, d_cu_seqlens, num_seqs, max_seqlen,
                               total_tokens, num_heads, softmax_scale, d_out, st);
    return launch_bf16<128>(ctx, d_q, d_k, d_v, d_cu_seqlens, num_seqs, max_seqlen, total_tokens,
                            num_heads, softmax_scale, d_out, st);
}
