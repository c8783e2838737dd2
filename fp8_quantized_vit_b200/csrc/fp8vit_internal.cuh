// Internal declarations of libfp8vit: the context, status reporting and the
// sm_100a PTX wrappers (mbarrier, TMA, tcgen05) the kernels share.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "fp8vit.h"

// Device scratch owned by a context (one cudaMalloc in fp8vit_create).
struct fp8vit_scratch {
    int32_t status;        // first device-detected fault (fp8vit_status), 0 = none
    int32_t site;          // kernel-specific location code of that fault
    uint32_t amax_bits[3]; // running |x| maxima (bf16 bit patterns) of q, k, v
    uint32_t arrivals;     // CTAs of the current amax launch that have finished
    uint32_t inject_attn;  // test hook: attention CTAs skip their first S-ready commit
    uint32_t release;      // generation counter of the fused amax/quantize grid barrier
    float descale[3];      // descales published across that barrier
    uint32_t pad[21];      // to 128 bytes
};

// Tensor maps the attention launches encode, kept per context: a layer
// reuses its buffers from call to call, so the maps of (base, shape, box)
// repeat and need not be encoded again on every launch.
struct fp8vit_tmap_entry {
    const void* base;
    int64_t rows, row_bytes;
    int32_t box_rows;
    bool valid;
    CUtensorMap map;
};
constexpr int kTmapCacheSize = 12;

struct fp8vit_ctx {
    int32_t device;
    int32_t num_sms;
    fp8vit_scratch* d_scratch;
    int32_t attn_p_terms;  // 2 = P as e4m3 hi + lo (default), 1 = single e4m3 term
    int64_t l2_bytes;      // the device's L2 size
    std::mutex tmap_mu;    // guards the cache below (calls may come from several threads)
    fp8vit_tmap_entry tmaps[kTmapCacheSize] = {};
    int32_t tmap_next = 0;  // round-robin replacement
    uint64_t tmap_hits = 0, tmap_misses = 0;
};

// Ring state layout (FP8VIT_RING_BYTES == 256).
struct fp8vit_ring {
    float hist[3][16];
    int32_t pos;
    int32_t pad[15];
};
static_assert(sizeof(fp8vit_ring) == FP8VIT_RING_BYTES, "ring layout");

#define FP8VIT_CUDA_TRY(expr)                          \
    do {                                               \
        cudaError_t e_ = (expr);                       \
        if (e_ != cudaSuccess) return FP8VIT_ECUDA;    \
    } while (0)

static_assert(sizeof(fp8vit_scratch) == 128, "scratch layout");

// Site codes recorded with a device fault.
enum : int32_t {
    SITE_ATTN_SEQLENS = 100,
    SITE_ATTN_WAIT_Q = 110,
    SITE_ATTN_WAIT_K = 111,
    SITE_ATTN_WAIT_V = 112,
    SITE_ATTN_WAIT_S = 113,
    SITE_ATTN_WAIT_P = 114,
    SITE_ATTN_WAIT_O = 115,
    SITE_ATTN_WAIT_EMPTY = 116,
    SITE_ATTN_WAIT_QREADY = 117,
    SITE_ATTN_DRAIN = 118,
    SITE_ATTN_WAIT_SFREE = 119,
    SITE_QUANT_BARRIER = 200,
};

__device__ __forceinline__ void fp8vit_report(fp8vit_scratch* s, int32_t status, int32_t site) {
    if (atomicCAS(&s->status, 0, status) == 0) atomicExch(&s->site, site);
}

// ---------------------------------------------------------------------------
// e4m3 helpers (hardware conversions: RNE, satfinite)
// ---------------------------------------------------------------------------

// Two floats -> two e4m3 codes packed in 16 bits (lo -> bits 0..7).
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

// Two e4m3 codes (bits 0..7 -> .x) back to two floats (exact).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t v) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// ---------------------------------------------------------------------------
// Per-token-group quantization arithmetic (atrex-bench "#025
// per_token_group_quant_fp8": scale = max(amax / 448, 1e-10), code =
// e4m3(clamp(x / scale, +-448))), shared by the group quantizer and the
// attention epilogue that fuses it, so both produce the same bytes.
// ---------------------------------------------------------------------------

// packed fp32 pairs (sm_100a f32x2 arithmetic)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// The group scale max(amax / 448, 1e-10) with the IEEE fp32 quotient, formed
// without a divide: q0 = RN(amax * RN(1/448)) and one FMA correction
// (Markstein, IBM J. Res. Dev. 34(1), 1990); exact for every non-negative
// finite bf16 amax (checked with exact rational arithmetic over all 32640).
__device__ __forceinline__ float group_scale_of_amax(float af) {
    const float q0 = __fmul_rn(af, 1.0f / 448.0f);
    const float sc = __fmaf_rn(__fmaf_rn(-448.0f, q0, af), 1.0f / 448.0f, q0);
    return sc > 1e-10f ? sc : 1e-10f;
}

// 8 bf16 / scale -> 8 e4m3 codes for quotients known to stay below 1024 in
// magnitude (inside a group |x| <= amax = 448 * scale), given s2 = (s, s)
// and nr2 = -(RN(1/s)) twice; two lanes per instruction, computed on -x:
//   q0 = RN((-x) * (-r)),  e = RN(q0 * s - x) (exact),  q = RN(q0 - e * r),
// the correctly rounded quotient (Markstein).  Working on -x keeps the sign
// of a zero quotient (x = -0 gives q = -0 and code 0x80) without a copysign:
// the only cancellation is q0 + (-0) terms, which then carry the operand's sign.
__device__ __forceinline__ uint2 quant8_small(const uint4& x, uint64_t s2, uint64_t nr2) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float nlo = __uint_as_float((w[i] << 16) ^ 0x80000000u);
        const float nhi = __uint_as_float((w[i] & 0xFFFF0000u) ^ 0x80000000u);
        const uint64_t nx = f2_pack(nlo, nhi);
        const uint64_t q0 = f2_mul(nx, nr2);
        const uint64_t e = f2_fma(q0, s2, nx);
        float qlo, qhi;
        f2_unpack(f2_fma(e, nr2, q0), qlo, qhi);
        c[i] = f32x2_to_e4m3x2(qlo, qhi);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// Per-tensor quantization arithmetic (vLLM docs "FP8 ViT Encoder Attention":
// x8 = e4m3(fp32(x) / descale)), shared by the per-tensor quantizers and the
// attention prologue that quantizes Q itself, so both produce the same bytes.

// x / s rounded to nearest fp32, given r = RN(1/s) (s > 0, finite).
// Markstein's correction (IBM J. Res. Dev. 34(1), 1990): with an exactly
// rounded reciprocal, q0 = RN(x r) is within one ulp of x / s, the
// remainder x - s q0 is exact in one FMA, and RN(q0 + rem r) is the
// correctly rounded quotient -- the IEEE division the quantizers are defined
// with, without a divide per element.  Quotients of magnitude >= 1024
// saturate to +-448 in e4m3 whatever their last bits, so they skip the
// correction (which would turn an overflowed q0 into NaN); the sign of a
// zero quotient is the sign of x.  Checked bit for bit against IEEE division
// on every finite BF16 value at 96 scales.
__device__ __forceinline__ float div_by_scale(float x, float s, float r) {
    const float q0 = __fmul_rn(x, r);
    const float rem = __fmaf_rn(-q0, s, x);
    const float q1 = __fmaf_rn(rem, r, q0);
    return copysignf(fabsf(q0) < 1024.0f ? q1 : q0, x);
}

// 8 bf16 (one 16-byte vector) / scale -> 8 e4m3 codes (8 bytes); r = RN(1/s).
__device__ __forceinline__ uint2 quant8(const uint4& x, float s, float r) {
    uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float lo = div_by_scale(__uint_as_float(w[i] << 16), s, r);
        float hi = div_by_scale(__uint_as_float(w[i] & 0xFFFF0000u), s, r);
        c[i] = f32x2_to_e4m3x2(lo, hi);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// ---------------------------------------------------------------------------
// sm_100a PTX wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on phase `parity` of an mbarrier.  Gives up when *abort is set
// by another thread of the CTA (abort may be null: then only the time limit
// ends the wait) or after timeout_ns; on a timeout it sets *abort and records
// FP8VIT_ETIMEOUT with `site`.  Returns false on give-up.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int32_t* abort, fp8vit_scratch* scr,
                                                  int32_t site, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (abort && *abort) return false;
            if (globaltimer_ns() - t0 > timeout_ns) {
                if (abort) *abort = 1;
                fp8vit_report(scr, FP8VIT_ETIMEOUT, site);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMA: 2-D tiled load global -> shared, completion on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// tcgen05: TMEM allocation (warp-collective).
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f8f6f4, issued by one thread.
__device__ __forceinline__ void umma_f8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f8f6f4, issued by one thread.
__device__ __forceinline__ void umma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all prior tcgen05 async operations of this
// thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                     taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Host: the driver's cuTensorMapEncodeTiled, resolved once through the runtime.
typedef CUresult (*fp8vit_encode_tiled_fn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                           const cuuint64_t*, const cuuint64_t*,
                                           const cuuint32_t*, const cuuint32_t*,
                                           CUtensorMapInterleave, CUtensorMapSwizzle,
                                           CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
fp8vit_encode_tiled_fn fp8vit_get_encode_tiled();
