// HBM-bound kernels of the path:
//   amax_ring_kernel   -- amax of q, k, v + 16-slot ring update + descales
//                         (vLLM "FP8 ViT Encoder Attention", Usage: dynamic scaling)
//   quant3_kernel      -- per-tensor e4m3 quantization of q, k, v
//                         (same page, intro: Q/K/V quantized right before attention)
//   group_quant_kernel -- per-token-group e4m3 quantization with fp32 scales
//                         (atrex-bench "#025 per_token_group_quant_fp8")
// All three stream 16-byte vectors with grid-stride loops sized to the SM
// count, and round with the hardware RNE-satfinite e4m3 conversion after an
// IEEE fp32 division (x / scale, as the pages' definitions divide).
#include <mutex>

#include "fp8vit_internal.cuh"

namespace {

constexpr int kAmaxThreads = 256;
constexpr int kQuantThreads = 256;
constexpr int kGroupThreads = 256;

// Per-lane |x| max of two packed bf16 values: clear the sign bits, then an
// unsigned max on each 16-bit half.  For non-NaN bf16, the order of the
// magnitude bit patterns is the order of the magnitudes.
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t w) {
    return __vmaxu2(acc, w & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t absmax_vec(uint32_t acc, const uint4& x) {
    acc = absmax2(acc, x.x);
    acc = absmax2(acc, x.y);
    acc = absmax2(acc, x.z);
    return absmax2(acc, x.w);
}

// 16-byte load that asks L2 to keep the line (evict_last priority): the
// fused amax/quantize kernel reads each vector again right after.
__device__ __forceinline__ uint64_t keep_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint4 ld_keep(const uint4* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

template <bool KEEP>
__device__ __forceinline__ uint4 ld_amax(const uint4* p, uint64_t pol) {
    if constexpr (KEEP) return ld_keep(p, pol);
    else return __ldcs(p);
}

// |x| max of one tensor over this thread's grid-stride share, four 16-byte
// loads in flight per thread.
__device__ __forceinline__ uint32_t amax_share(const uint4* __restrict__ p, int64_t n_elems) {
    const int64_t nvec = n_elems >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t a0 = 0, a1 = 0;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        const uint4 x0 = __ldcs(p + i), x1 = __ldcs(p + i + stride);
        const uint4 x2 = __ldcs(p + i + 2 * stride), x3 = __ldcs(p + i + 3 * stride);
        a0 = absmax_vec(absmax_vec(a0, x0), x2);
        a1 = absmax_vec(absmax_vec(a1, x1), x3);
    }
    for (; i < nvec; i += stride) a0 = absmax_vec(a0, __ldcs(p + i));
    const int tail = (int)(n_elems & 7);
    if (blockIdx.x == 0 && (int)threadIdx.x < tail)
        a0 = absmax2(a0, reinterpret_cast<const uint16_t*>(p)[(nvec << 3) + threadIdx.x]);
    a0 = __vmaxu2(a0, a1);
    return max(a0 & 0xFFFFu, a0 >> 16);
}

// Four CTAs (1024 threads) per SM with four loads in flight per thread:
// 64 KB of loads in flight per SM.
__device__ __forceinline__ void ring_rule(fp8vit_ring* ring, const float (&amax)[3],
                                       float* descale3);

// ring == nullptr: write the three amaxes (fp32) to out3 instead of running
// the ring rule (the sharded path all-reduces them first).
__global__ void __launch_bounds__(kAmaxThreads, 4) amax_ring_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
    int64_t n_elems, fp8vit_ring* __restrict__ ring, float* __restrict__ out3,
    fp8vit_scratch* __restrict__ scr) {
    uint32_t m[3];
    m[0] = amax_share(q, n_elems);
    m[1] = amax_share(k, n_elems);
    m[2] = amax_share(v, n_elems);
    __shared__ uint32_t red[3][kAmaxThreads / 32];
    __shared__ int is_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int t = 0; t < 3; ++t) {
        uint32_t w = __reduce_max_sync(0xFFFFFFFFu, m[t]);
        if (lane == 0) red[t][warp] = w;
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            uint32_t x = lane < (int)(blockDim.x >> 5) ? red[t][lane] : 0u;
            x = __reduce_max_sync(0xFFFFFFFFu, x);
            if (lane == 0) atomicMax(&scr->amax_bits[t], x);
        }
        if (lane == 0) {
            __threadfence();
            unsigned ticket = atomicAdd(&scr->arrivals, 1u);
            is_last = (ticket == gridDim.x - 1);
        }
    }
    __syncthreads();
    if (!is_last || threadIdx.x != 0) return;
    // Last CTA: every other CTA's atomicMax is visible.  Read and clear the
    // scratch for the next launch, then run the ring rule.
    __threadfence();
    float amax[3];
#pragma unroll
    for (int t = 0; t < 3; ++t) amax[t] = bf16_bits_to_f32(atomicExch(&scr->amax_bits[t], 0u));
    atomicExch(&scr->arrivals, 0u);
    if (ring == nullptr) {
#pragma unroll
        for (int t = 0; t < 3; ++t) out3[t] = amax[t];
        return;
    }
    ring_rule(ring, amax, out3);
}

// The 16-slot ring rule for one forward: write the amaxes at pos, advance
// pos, descale = max(max over the slots / 448, 1e-10) (fp32 division).
__device__ __forceinline__ void ring_rule(fp8vit_ring* ring, const float (&amax)[3],
                                       float* descale3) {
    int32_t p = ring->pos;
    p = ((p % 16) + 16) % 16;
#pragma unroll 1
    for (int t = 0; t < 3; ++t) {
        ring->hist[t][p] = amax[t];
        float mx = 0.0f;
#pragma unroll 1
        for (int j = 0; j < 16; ++j) mx = ring->hist[t][j] > mx ? ring->hist[t][j] : mx;
        const float d = __fdiv_rn(mx, 448.0f);
        descale3[t] = d > 1e-10f ? d : 1e-10f;
    }
    ring->pos = (p + 1) & 15;
}

__global__ void ring_push_kernel(const float* __restrict__ amax3, fp8vit_ring* __restrict__ ring,
                                 float* __restrict__ descale3) {
    const float a[3] = {amax3[0], amax3[1], amax3[2]};
    ring_rule(ring, a, descale3);
}

// One tensor's grid-stride share: four 16-byte loads in flight per thread.
__device__ __forceinline__ void quant_share(const uint4* __restrict__ p, uint2* __restrict__ o,
                                            int64_t n_elems, float s) {
    const float r = __frcp_rn(s);
    const int64_t nvec = n_elems >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        const uint4 x0 = __ldcs(p + i), x1 = __ldcs(p + i + stride);
        const uint4 x2 = __ldcs(p + i + 2 * stride), x3 = __ldcs(p + i + 3 * stride);
        __stcs(o + i, quant8(x0, s, r));
        __stcs(o + i + stride, quant8(x1, s, r));
        __stcs(o + i + 2 * stride, quant8(x2, s, r));
        __stcs(o + i + 3 * stride, quant8(x3, s, r));
    }
    for (; i < nvec; i += stride) __stcs(o + i, quant8(__ldcs(p + i), s, r));
    const int tail = (int)(n_elems & 7);
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
        const int64_t e = (nvec << 3) + threadIdx.x;
        const float y = div_by_scale(bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(p)[e]), s, r);
        reinterpret_cast<uint8_t*>(o)[e] = (uint8_t)(f32x2_to_e4m3x2(y, 0.0f) & 0xFF);
    }
}

__global__ void __launch_bounds__(kQuantThreads, 4) quant3_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
    int64_t n_elems, const float* __restrict__ descale3, uint2* __restrict__ q8,
    uint2* __restrict__ k8, uint2* __restrict__ v8) {
    if (q8) quant_share(q, q8, n_elems, descale3[0]);  // null: Q is quantized by the attention
    quant_share(k, k8, n_elems, descale3[1]);
    quant_share(v, v8, n_elems, descale3[2]);
}

// amax + ring rule + quantize in one launch, for the dynamic-scale path.
// The launch is cooperative (every block resident at once), so the blocks can
// meet at a grid barrier: phase 1 reduces the three amaxes as
// amax_ring_kernel does; the last block to arrive runs the ring rule and
// publishes the descales in the scratch; the others wait for the barrier's
// generation counter to move (bounded: a timeout records FP8VIT_ETIMEOUT
// and the block returns); phase 2 quantizes as quant3_kernel does.  The BF16
// tensors are read twice; KEEP (chosen when the three tensors fit in L2)
// loads them with evict_last priority in phase 1, so that more of phase 2's
// reads come from L2.
constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;

// |x| maxima of q, k and v over this thread's grid-stride share in one loop:
// six 16-byte loads in flight per thread (two vectors of each tensor), so
// tensors of a few tens of MB, where each thread owns only a dozen vectors,
// do not pay three separate load ramps.
template <bool KEEP>
__device__ __forceinline__ void amax3_share(const uint4* __restrict__ q,
                                            const uint4* __restrict__ k,
                                            const uint4* __restrict__ v, int64_t n_elems,
                                            uint32_t (&m)[3]) {
    const int64_t nvec = n_elems >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint64_t pol = KEEP ? keep_policy() : 0;
    uint32_t a[3] = {0u, 0u, 0u}, b[3] = {0u, 0u, 0u};
    for (; i + stride < nvec; i += 2 * stride) {
        const uint4 q0 = ld_amax<KEEP>(q + i, pol), k0 = ld_amax<KEEP>(k + i, pol);
        const uint4 v0 = ld_amax<KEEP>(v + i, pol), q1 = ld_amax<KEEP>(q + i + stride, pol);
        const uint4 k1 = ld_amax<KEEP>(k + i + stride, pol);
        const uint4 v1 = ld_amax<KEEP>(v + i + stride, pol);
        a[0] = absmax_vec(a[0], q0);
        a[1] = absmax_vec(a[1], k0);
        a[2] = absmax_vec(a[2], v0);
        b[0] = absmax_vec(b[0], q1);
        b[1] = absmax_vec(b[1], k1);
        b[2] = absmax_vec(b[2], v1);
    }
    if (i < nvec) {
        a[0] = absmax_vec(a[0], ld_amax<KEEP>(q + i, pol));
        a[1] = absmax_vec(a[1], ld_amax<KEEP>(k + i, pol));
        a[2] = absmax_vec(a[2], ld_amax<KEEP>(v + i, pol));
    }
    const int tail = (int)(n_elems & 7);
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
        const int64_t e = (nvec << 3) + threadIdx.x;
        a[0] = absmax2(a[0], reinterpret_cast<const uint16_t*>(q)[e]);
        a[1] = absmax2(a[1], reinterpret_cast<const uint16_t*>(k)[e]);
        a[2] = absmax2(a[2], reinterpret_cast<const uint16_t*>(v)[e]);
    }
#pragma unroll
    for (int t = 0; t < 3; ++t) {
        const uint32_t c = __vmaxu2(a[t], b[t]);
        m[t] = max(c & 0xFFFFu, c >> 16);
    }
}

// quant_share for q, k and v in one loop (v, k, q order: in the fused kernel
// the tensor read last in phase 1 is the likeliest to still be in L2).
__device__ __forceinline__ void quant3_share(const uint4* __restrict__ q,
                                             const uint4* __restrict__ k,
                                             const uint4* __restrict__ v, uint2* __restrict__ q8,
                                             uint2* __restrict__ k8, uint2* __restrict__ v8,
                                             int64_t n_elems, const float (&s)[3]) {
    const float rq = __frcp_rn(s[0]), rk = __frcp_rn(s[1]), rv = __frcp_rn(s[2]);
    const int64_t nvec = n_elems >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const bool wq = q8 != nullptr;  // null: Q is quantized by the attention kernel
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (wq) {
        for (; i + stride < nvec; i += 2 * stride) {
            const uint4 v0 = __ldcs(v + i), k0 = __ldcs(k + i), q0 = __ldcs(q + i);
            const uint4 v1 = __ldcs(v + i + stride), k1 = __ldcs(k + i + stride);
            const uint4 q1 = __ldcs(q + i + stride);
            __stcs(v8 + i, quant8(v0, s[2], rv));
            __stcs(k8 + i, quant8(k0, s[1], rk));
            __stcs(q8 + i, quant8(q0, s[0], rq));
            __stcs(v8 + i + stride, quant8(v1, s[2], rv));
            __stcs(k8 + i + stride, quant8(k1, s[1], rk));
            __stcs(q8 + i + stride, quant8(q1, s[0], rq));
        }
    } else {
        for (; i + stride < nvec; i += 2 * stride) {
            const uint4 v0 = __ldcs(v + i), k0 = __ldcs(k + i);
            const uint4 v1 = __ldcs(v + i + stride), k1 = __ldcs(k + i + stride);
            __stcs(v8 + i, quant8(v0, s[2], rv));
            __stcs(k8 + i, quant8(k0, s[1], rk));
            __stcs(v8 + i + stride, quant8(v1, s[2], rv));
            __stcs(k8 + i + stride, quant8(k1, s[1], rk));
        }
    }
    if (i < nvec) {
        __stcs(v8 + i, quant8(__ldcs(v + i), s[2], rv));
        __stcs(k8 + i, quant8(__ldcs(k + i), s[1], rk));
        if (wq) __stcs(q8 + i, quant8(__ldcs(q + i), s[0], rq));
    }
    const int tail = (int)(n_elems & 7);
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
        const int64_t e = (nvec << 3) + threadIdx.x;
        const uint4* src[3] = {q, k, v};
        uint2* dst[3] = {q8, k8, v8};
        const float r[3] = {rq, rk, rv};
#pragma unroll
        for (int t = wq ? 0 : 1; t < 3; ++t) {
            const float y = div_by_scale(
                bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(src[t])[e]), s[t], r[t]);
            reinterpret_cast<uint8_t*>(dst[t])[e] = (uint8_t)(f32x2_to_e4m3x2(y, 0.0f) & 0xFF);
        }
    }
}

template <bool KEEP>
__global__ void __launch_bounds__(kQuantThreads, 4) amax_ring_quant_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
    int64_t n_elems, fp8vit_ring* __restrict__ ring, float* __restrict__ descale3,
    uint2* __restrict__ q8, uint2* __restrict__ k8, uint2* __restrict__ v8,
    fp8vit_scratch* __restrict__ scr) {
    __shared__ uint32_t red[3][kQuantThreads / 32];
    __shared__ float sdesc[3];
    __shared__ int proceed;
    volatile uint32_t* release = &scr->release;
    // The generation before this launch's barrier: read before this block
    // arrives, so the last block cannot have advanced it yet.
    const uint32_t gen0 = threadIdx.x == 0 ? *release : 0u;
    uint32_t m[3];
    amax3_share<KEEP>(q, k, v, n_elems, m);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int t = 0; t < 3; ++t) {
        uint32_t w = __reduce_max_sync(0xFFFFFFFFu, m[t]);
        if (lane == 0) red[t][warp] = w;
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            uint32_t x = lane < (int)(blockDim.x >> 5) ? red[t][lane] : 0u;
            x = __reduce_max_sync(0xFFFFFFFFu, x);
            if (lane == 0) atomicMax(&scr->amax_bits[t], x);
        }
    }
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned ticket = atomicAdd(&scr->arrivals, 1u);
        int go = 1;
        if (ticket == gridDim.x - 1) {
            // Every other block's atomicMax is visible: take and clear the
            // maxima, run the ring rule, publish the descales, release.
            __threadfence();
            float amax[3];
#pragma unroll
            for (int t = 0; t < 3; ++t)
                amax[t] = bf16_bits_to_f32(atomicExch(&scr->amax_bits[t], 0u));
            atomicExch(&scr->arrivals, 0u);
            ring_rule(ring, amax, descale3);
            volatile float* pub = scr->descale;
#pragma unroll
            for (int t = 0; t < 3; ++t) pub[t] = descale3[t];
            __threadfence();
            atomicAdd(&scr->release, 1u);
        } else {
            const uint64_t t0 = globaltimer_ns();
            while (*release == gen0) {
                if (globaltimer_ns() - t0 > kBarrierTimeoutNs) {
                    fp8vit_report(scr, FP8VIT_ETIMEOUT, SITE_QUANT_BARRIER);
                    go = 0;
                    break;
                }
                __nanosleep(64);
            }
            __threadfence();
        }
        const volatile float* pub = scr->descale;
#pragma unroll
        for (int t = 0; t < 3; ++t) sdesc[t] = pub[t];
        proceed = go;
    }
    __syncthreads();
    if (!proceed) return;
    const float s3[3] = {sdesc[0], sdesc[1], sdesc[2]};
    quant3_share(q, k, v, q8, k8, v8, n_elems, s3);
}

// LPG = lanes per group = group / 8; each lane owns one 16-byte vector of
// its group; a warp covers 32 / LPG groups per step and keeps kUnroll steps
// (kUnroll loads per lane) in flight.
template <int LPG>
__global__ void __launch_bounds__(kGroupThreads) group_quant_kernel(
    const uint4* __restrict__ x, int64_t total_groups, uint2* __restrict__ xq,
    float* __restrict__ scales) {
    constexpr int kGPW = 32 / LPG;
    constexpr int kUnroll = 4;
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPG, gl = lane % LPG;
    const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t g0 = warp_id * kGPW * kUnroll; g0 < total_groups;
         g0 += nwarps * kGPW * kUnroll) {
        uint4 xv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = g0 + u * kGPW + sub;
            xv[u] = g < total_groups ? __ldcs(x + g * LPG + gl) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = g0 + u * kGPW + sub;
            uint32_t a = absmax_vec(0u, xv[u]);
            a = max(a & 0xFFFFu, a >> 16);
#pragma unroll
            for (int off = LPG / 2; off > 0; off >>= 1)
                a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
            const float sc = group_scale_of_amax(bf16_bits_to_f32(a));
            if (g < total_groups) {
                const float nr = -__frcp_rn(sc);
                __stcs(xq + g * LPG + gl, quant8_small(xv[u], f2_pack(sc, sc), f2_pack(nr, nr)));
                if (gl == 0) scales[g] = sc;
            }
        }
    }
}

inline bool misaligned(const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0;
}

// Resident blocks per SM of a kernel, queried once per kernel (later calls,
// e.g. inside a CUDA-graph capture, make no CUDA API call).
inline int resident_blocks(const void* kfn, int threads) {
    static std::mutex mu;
    static const void* keys[16];
    static int vals[16];
    static int n = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (keys[i] == kfn) return vals[i];
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, threads, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    if (n < 16) {
        keys[n] = kfn;
        vals[n] = per_sm;
        ++n;
    }
    return per_sm;
}

inline int grid_for(int64_t work_items, int threads, int per_thread, int max_blocks) {
    int64_t b = (work_items + (int64_t)threads * per_thread - 1) / ((int64_t)threads * per_thread);
    if (b < 1) b = 1;
    if (b > max_blocks) b = max_blocks;
    return (int)b;
}

}  // namespace

extern "C" {

fp8vit_status fp8_amax_ring_update(fp8vit_ctx* ctx, const uint16_t* d_q, const uint16_t* d_k,
                                   const uint16_t* d_v, int64_t n_elems, void* d_ring,
                                   float* d_descale3, void* stream) {
    if (!ctx || !d_q || !d_k || !d_v || !d_ring || !d_descale3 || n_elems < 0)
        return FP8VIT_EINVAL;
    if (misaligned(d_q, 16) || misaligned(d_k, 16) || misaligned(d_v, 16) ||
        misaligned(d_ring, 16) || misaligned(d_descale3, 4))
        return FP8VIT_EINVAL;
    const int grid = grid_for(n_elems >> 3, kAmaxThreads, 8, 4 * ctx->num_sms);
    amax_ring_kernel<<<grid, kAmaxThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4*>(d_q), reinterpret_cast<const uint4*>(d_k),
        reinterpret_cast<const uint4*>(d_v), n_elems, reinterpret_cast<fp8vit_ring*>(d_ring),
        d_descale3, ctx->d_scratch);
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

fp8vit_status fp8_amax3(fp8vit_ctx* ctx, const uint16_t* d_q, const uint16_t* d_k,
                        const uint16_t* d_v, int64_t n_elems, float* d_amax3, void* stream) {
    if (!ctx || !d_q || !d_k || !d_v || !d_amax3 || n_elems < 0) return FP8VIT_EINVAL;
    if (misaligned(d_q, 16) || misaligned(d_k, 16) || misaligned(d_v, 16) ||
        misaligned(d_amax3, 4))
        return FP8VIT_EINVAL;
    const int grid = grid_for(n_elems >> 3, kAmaxThreads, 8, 4 * ctx->num_sms);
    amax_ring_kernel<<<grid, kAmaxThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4*>(d_q), reinterpret_cast<const uint4*>(d_k),
        reinterpret_cast<const uint4*>(d_v), n_elems, nullptr, d_amax3, ctx->d_scratch);
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

fp8vit_status fp8_ring_push(const float* d_amax3, void* d_ring, float* d_descale3,
                            void* stream) {
    if (!d_amax3 || !d_ring || !d_descale3) return FP8VIT_EINVAL;
    if (misaligned(d_ring, 16) || misaligned(d_amax3, 4) || misaligned(d_descale3, 4))
        return FP8VIT_EINVAL;
    ring_push_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        d_amax3, reinterpret_cast<fp8vit_ring*>(d_ring), d_descale3);
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

fp8vit_status fp8_quantize_qkv_per_tensor(fp8vit_ctx* ctx, const uint16_t* d_q,
                                          const uint16_t* d_k, const uint16_t* d_v,
                                          int64_t n_elems, const float* d_descale3, uint8_t* d_q8,
                                          uint8_t* d_k8, uint8_t* d_v8, void* stream) {
    if (!ctx || !d_q || !d_k || !d_v || !d_descale3 || !d_k8 || !d_v8 || n_elems < 0)
        return FP8VIT_EINVAL;
    if (misaligned(d_q, 16) || misaligned(d_k, 16) || misaligned(d_v, 16) ||
        misaligned(d_q8, 8) || misaligned(d_k8, 8) || misaligned(d_v8, 8) ||
        misaligned(d_descale3, 4))
        return FP8VIT_EINVAL;
    // one resident wave of grid-stride blocks (see per_token_group_quant_fp8)
    const int per_sm = resident_blocks((const void*)quant3_kernel, kQuantThreads);
    const int grid = grid_for(n_elems >> 3, kQuantThreads, 4, per_sm * ctx->num_sms);
    quant3_kernel<<<grid, kQuantThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4*>(d_q), reinterpret_cast<const uint4*>(d_k),
        reinterpret_cast<const uint4*>(d_v), n_elems, d_descale3, reinterpret_cast<uint2*>(d_q8),
        reinterpret_cast<uint2*>(d_k8), reinterpret_cast<uint2*>(d_v8));
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

fp8vit_status fp8_amax_ring_quantize_qkv(fp8vit_ctx* ctx, const uint16_t* d_q,
                                         const uint16_t* d_k, const uint16_t* d_v,
                                         int64_t n_elems, void* d_ring, float* d_descale3,
                                         uint8_t* d_q8, uint8_t* d_k8, uint8_t* d_v8,
                                         void* stream) {
    if (!ctx || !d_q || !d_k || !d_v || !d_ring || !d_descale3 || !d_k8 || !d_v8 ||
        n_elems < 0)
        return FP8VIT_EINVAL;
    if (misaligned(d_q, 16) || misaligned(d_k, 16) || misaligned(d_v, 16) ||
        misaligned(d_ring, 16) || misaligned(d_descale3, 4) || misaligned(d_q8, 8) ||
        misaligned(d_k8, 8) || misaligned(d_v8, 8))
        return FP8VIT_EINVAL;
    // The one-launch kernel: faster than the two kernels up to about twice L2
    // of BF16 inputs (one launch, interleaved streams, part of the second read
    // served by L2; with evict_last loads when the inputs fit in L2).  Larger
    // tensors take the two kernels, which stream HBM slightly faster than the
    // barrier-split launch.  The results are identical.
    const bool keep = n_elems <= ctx->l2_bytes / 6;
    if (n_elems > ctx->l2_bytes / 3) {  // more than twice L2 in BF16 inputs
        const fp8vit_status st = fp8_amax_ring_update(ctx, d_q, d_k, d_v, n_elems, d_ring,
                                                      d_descale3, stream);
        if (st != FP8VIT_OK) return st;
        return fp8_quantize_qkv_per_tensor(ctx, d_q, d_k, d_v, n_elems, d_descale3, d_q8, d_k8,
                                           d_v8, stream);
    }
    auto kern = keep ? amax_ring_quant_kernel<true> : amax_ring_quant_kernel<false>;
    // one resident wave, which the cooperative launch requires anyway
    const int per_sm = resident_blocks((const void*)kern, kQuantThreads);
    const int grid = grid_for(n_elems >> 3, kQuantThreads, 4, per_sm * ctx->num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kQuantThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, kern, reinterpret_cast<const uint4*>(d_q),
        reinterpret_cast<const uint4*>(d_k), reinterpret_cast<const uint4*>(d_v), n_elems,
        reinterpret_cast<fp8vit_ring*>(d_ring), d_descale3, reinterpret_cast<uint2*>(d_q8),
        reinterpret_cast<uint2*>(d_k8), reinterpret_cast<uint2*>(d_v8), ctx->d_scratch);
    return e == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

fp8vit_status per_token_group_quant_fp8(fp8vit_ctx* ctx, const uint16_t* d_x, int64_t m,
                                        int64_t n, int32_t group, uint8_t* d_xq,
                                        float* d_scales, void* stream) {
    if (!ctx || !d_x || !d_xq || !d_scales || m < 0 || n < 0 || group <= 0) return FP8VIT_EINVAL;
    if (n % group != 0) return FP8VIT_EINVAL;
    if (group != 16 && group != 32 && group != 64 && group != 128 && group != 256)
        return FP8VIT_EUNSUPPORTED;
    if (misaligned(d_x, 16) || misaligned(d_xq, 8) || misaligned(d_scales, 4))
        return FP8VIT_EINVAL;
    if (m != 0 && n > INT64_MAX / m) return FP8VIT_EINVAL;
    const int64_t total_groups = m * (n / group);
    if (total_groups == 0) return FP8VIT_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int lpg = group / 8;
    const int64_t gpw = 32 / (lpg > 0 ? lpg : 1);
    // One resident wave: every block streams an equal grid-stride share, so a
    // grid larger than what fits at once would leave a partial second wave.
    const void* kfn = group == 16    ? (const void*)group_quant_kernel<2>
                      : group == 32  ? (const void*)group_quant_kernel<4>
                      : group == 64  ? (const void*)group_quant_kernel<8>
                      : group == 128 ? (const void*)group_quant_kernel<16>
                                     : (const void*)group_quant_kernel<32>;
    const int per_sm = resident_blocks(kfn, kGroupThreads);
    const int grid = grid_for((total_groups + gpw - 1) / gpw * 32, kGroupThreads, 4,
                              per_sm * ctx->num_sms);
    const uint4* x = reinterpret_cast<const uint4*>(d_x);
    uint2* xq = reinterpret_cast<uint2*>(d_xq);
    switch (group) {
        case 16: group_quant_kernel<2><<<grid, kGroupThreads, 0, st>>>(x, total_groups, xq, d_scales); break;
        case 32: group_quant_kernel<4><<<grid, kGroupThreads, 0, st>>>(x, total_groups, xq, d_scales); break;
        case 64: group_quant_kernel<8><<<grid, kGroupThreads, 0, st>>>(x, total_groups, xq, d_scales); break;
        case 128: group_quant_kernel<16><<<grid, kGroupThreads, 0, st>>>(x, total_groups, xq, d_scales); break;
        case 256: group_quant_kernel<32><<<grid, kGroupThreads, 0, st>>>(x, total_groups, xq, d_scales); break;
        default: return FP8VIT_EUNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of fp8_amax_ring_update.
//
// Some callers cannot allocate device memory at the point where they run the
// path: a serving process that has already handed (nearly) all free HBM to
// its own pool, code that must not pay cudaMalloc's implicit device-wide
// synchronisation, or a plug-in that has no place to keep a library context
// (fp8vit_create allocates).  For them this entry point takes its scratch
// from a fixed array compiled into the library's device image instead.
//
// Scratch: sizeof(fp8vit_scratch) = 128 bytes (three running |x| maxima, an
// arrival counter, status words), taken from a 256-byte array.  The amount
// does not grow with n_elems, so any size the context entry point accepts is
// accepted here; that the need fits the array is checked when the library is
// compiled.  Every GPU that loads the library holds the array until the
// process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = 256;
constexpr int kNoAllocMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char g_amax_noalloc_scratch[kNoAllocScratchBytes];
static_assert(sizeof(fp8vit_scratch) <= kNoAllocScratchBytes,
              "the amax scratch must fit the library's fixed array");

namespace {

struct NoAllocSetup {
    std::mutex mu;
    void* addr[kNoAllocMaxDevices] = {};
    int num_sms[kNoAllocMaxDevices] = {};
};

NoAllocSetup& noalloc_setup() {
    static NoAllocSetup s;
    return s;
}

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
fp8vit_status noalloc_scratch(void** addr, int* num_sms) {
    int dev = -1;
    FP8VIT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kNoAllocMaxDevices) return FP8VIT_EUNSUPPORTED;
    NoAllocSetup& s = noalloc_setup();
    std::lock_guard<std::mutex> lock(s.mu);
    if (!s.addr[dev]) {
        void* p = nullptr;
        FP8VIT_CUDA_TRY(cudaGetSymbolAddress(&p, g_amax_noalloc_scratch));
        int sms = 0;
        FP8VIT_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
        s.num_sms[dev] = sms;
        s.addr[dev] = p;
    }
    *addr = s.addr[dev];
    *num_sms = s.num_sms[dev];
    return FP8VIT_OK;
}

}  // namespace

extern "C" fp8vit_status fp8_amax_ring_update_noalloc(const uint16_t* d_q, const uint16_t* d_k,
                                                      const uint16_t* d_v, int64_t n_elems,
                                                      void* d_ring, float* d_descale3,
                                                      void* stream) {
    if (!d_q || !d_k || !d_v || !d_ring || !d_descale3 || n_elems < 0) return FP8VIT_EINVAL;
    if (misaligned(d_q, 16) || misaligned(d_k, 16) || misaligned(d_v, 16) ||
        misaligned(d_ring, 16) || misaligned(d_descale3, 4))
        return FP8VIT_EINVAL;
    void* scratch = nullptr;
    int num_sms = 0;
    fp8vit_status st = noalloc_scratch(&scratch, &num_sms);
    if (st != FP8VIT_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps whatever the previous call left; the kernel needs the
    // maxima and the arrival counter at zero.
    FP8VIT_CUDA_TRY(cudaMemsetAsync(scratch, 0, sizeof(fp8vit_scratch), cs));
    const int grid = grid_for(n_elems >> 3, kAmaxThreads, 8, 4 * num_sms);
    amax_ring_kernel<<<grid, kAmaxThreads, 0, cs>>>(
        reinterpret_cast<const uint4*>(d_q), reinterpret_cast<const uint4*>(d_k),
        reinterpret_cast<const uint4*>(d_v), n_elems, reinterpret_cast<fp8vit_ring*>(d_ring),
        d_descale3, reinterpret_cast<fp8vit_scratch*>(scratch));
    return cudaGetLastError() == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}
