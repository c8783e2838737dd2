// Pieces shared by the attention kernels (sm_100a): shared-memory and
// instruction descriptors for tcgen05.mma, TMEM load/store wrappers, packed
// fp32 arithmetic, the output modes and the host-side tensor-map encoder.
#pragma once

#include "fp8vit_internal.cuh"

namespace fp8vit_attn {

constexpr int kBox = 32;  // bytes per TMA box row (one SW32 atom row)

// Bounded wait used on a kernel's exit path: it ignores the CTA's abort flag,
// so a CTA leaves only after its own copies and MMAs have landed (or its own
// time limit ran out, which records FP8VIT_ETIMEOUT at SITE_ATTN_DRAIN).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity,
                                                fp8vit_scratch* scr) {
    return mbar_wait_bounded(bar, parity, nullptr, scr, SITE_ATTN_DRAIN, 2000000000ull);
}

// Shared-memory matrix descriptors (tcgen05 "version 1" format), 32-byte
// swizzle.  K-major: rows of 32 bytes, 8-row groups 256 bytes apart (SBO).
// MN-major (V): 32-byte atoms along N, one [keys x 32 B] box (KVT bytes) apart (LBO);
// 8-key groups 256 bytes apart (SBO).
__device__ __forceinline__ uint64_t desc_k_sw32(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(256 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)6 << 61);
}
template <int KVT>
__device__ __forceinline__ uint64_t desc_mn_sw32(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(KVT >> 4) << 16) |
           ((uint64_t)(256 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)6 << 61);
}

// Instruction descriptor, kind::f8f6f4: e4m3 x e4m3 -> f32, M = 128.
__host__ __device__ constexpr uint32_t idesc_e4m3(int n, bool b_mn_major) {
    return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}
// Instruction descriptor, kind::f16: bf16 x bf16 -> f32 (A and B format
// fields = 1), M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
    return idesc_e4m3(n, b_mn_major) | (1u << 7) | (1u << 10);
}

__device__ __forceinline__ void tmem_ld8_sync(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr)
        : "memory");
}

// 64 consecutive columns of this thread's lane into a[0..31], b[0..31], then wait.
__device__ __forceinline__ void tmem_ld64_sync(uint32_t taddr, uint32_t (&a)[32], uint32_t (&b)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]), "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]), "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]), "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]), "=r"(b[24]), "=r"(b[25]), "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// O *= alpha over columns [0, NPV) of this thread's lane, in 32-column steps
// (one load wait per step); NPV = 80 ends with two 8-column pieces.
template <int NPV>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll
    for (int c = 0; c + 32 <= NPV; c += 32) {
        uint32_t r[32];
        tmem_ld32(tO + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
        tmem_st32(tO + c, r);
    }
    if constexpr (NPV % 32 != 0) {
        static_assert(NPV % 32 == 16, "O tail is one 16-column piece");
        constexpr int c = NPV - 16;
        uint32_t r[8], s[8];
        tmem_ld8(tO + c, r);
        tmem_ld8(tO + c + 8, s);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            s[i] = __float_as_uint(__uint_as_float(s[i]) * alpha);
        }
        tmem_st8(tO + c, r);
        tmem_st8(tO + c + 8, s);
    }
}

// One arrival per warp: every lane's prior memory and tcgen05 operations
// (each lane has executed its own fences) are ordered before lane 0's arrive
// by the warp barrier.
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// ---- packed arithmetic used by the softmax --------------------------------

__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// Row max of one S tile of NCH 32-key chunks held in registers; keys past the
// segment end already hold -inf.
template <int NCH>
__device__ __forceinline__ float tile_row_max(const uint32_t (&r)[NCH][32]) {
    float m[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        float a = -INFINITY, b = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            a = fmax3(a, __uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1]));
            b = fmax3(b, __uint_as_float(r[c][i + 2]), __uint_as_float(r[c][i + 3]));
        }
        m[c] = fmaxf(a, b);
    }
    float mx = m[0];
#pragma unroll
    for (int c = 1; c < NCH; ++c) mx = fmaxf(mx, m[c]);
    return mx;
}

// Eight O columns of this thread's lane times inv, rounded to bf16 (RNE) and
// packed two per word: the values the bf16 epilogue stores.
__device__ __forceinline__ uint4 bf16x8_of_o(uint32_t taddr, float inv) {
    uint32_t r[8];
    tmem_ld8_sync(taddr, r);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[2 * i]) * inv,
                                                 __uint_as_float(r[2 * i + 1]) * inv);
        w[i] = *reinterpret_cast<uint32_t*>(&b);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Output modes, one epilogue per kernel instance.
enum : int {
    kOutBf16 = 0,     // o as bf16; with a tile-counter buffer, also its 128-wide
                      // groups quantized by the launch's group tail (any head_dim
                      // with num_heads * head_dim % 128 == 0)
    kOutE4m3 = 1,     // e4m3(o / output_scale)
    kOutGroupQ = 2,   // the bf16 o of each head quantized as one 128-wide group:
                      // e4m3 codes + one fp32 scale per (token, head); head_dim 128
};

// Host: a 2-D uint8 tensor map over a [rows, row_bytes] matrix with
// 32-byte x boxes of box_rows rows, 32-byte swizzle.
inline bool encode_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes,
                int box_rows) {
    fp8vit_encode_tiled_fn enc = fp8vit_get_encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)kBox, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The 2-D uint8 tensor map of encode_map, from the context's cache when the
// same (base, rows, row_bytes, box_rows) was encoded before; encodes and
// stores it otherwise.
inline bool cached_map(fp8vit_ctx* ctx, CUtensorMap* map, const void* base, int64_t rows,
                       int64_t row_bytes, int box_rows) {
    std::lock_guard<std::mutex> lock(ctx->tmap_mu);
    for (fp8vit_tmap_entry& e : ctx->tmaps) {
        if (e.valid && e.base == base && e.rows == rows && e.row_bytes == row_bytes &&
            e.box_rows == box_rows) {
            *map = e.map;
            ++ctx->tmap_hits;
            return true;
        }
    }
    if (!encode_map(map, base, rows, row_bytes, box_rows)) return false;
    fp8vit_tmap_entry& e = ctx->tmaps[ctx->tmap_next];
    ctx->tmap_next = (ctx->tmap_next + 1) % kTmapCacheSize;
    e.base = base;
    e.rows = rows;
    e.row_bytes = row_bytes;
    e.box_rows = box_rows;
    e.map = *map;
    e.valid = true;
    ++ctx->tmap_misses;
    return true;
}

inline bool misaligned(const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0;
}

}  // namespace fp8vit_attn

