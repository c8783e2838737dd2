// Context lifecycle, status reporting and the small host helpers of the ABI.
#include <cstddef>
#include <mutex>

#include "fp8vit_internal.cuh"

extern "C" {

int32_t fp8vit_version(void) { return 100; }

const char* fp8vit_status_string(fp8vit_status s) {
    switch (s) {
        case FP8VIT_OK: return "ok";
        case FP8VIT_EINVAL: return "invalid argument";
        case FP8VIT_EUNSUPPORTED: return "unsupported shape or mode";
        case FP8VIT_ECUDA: return "CUDA call failed";
        case FP8VIT_EIO: return "scale file I/O error";
        case FP8VIT_EPARSE: return "scale file parse error";
        case FP8VIT_ENOTFOUND: return "layer not found in scale file";
        case FP8VIT_ETIMEOUT: return "bounded wait timed out in a kernel";
    }
    return "unknown status";
}

fp8vit_status fp8vit_create(int32_t device, fp8vit_ctx** out) {
    if (!out) return FP8VIT_EINVAL;
    *out = nullptr;
    FP8VIT_CUDA_TRY(cudaSetDevice(device));
    int sms = 0;
    FP8VIT_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device));
    int l2 = 0;
    FP8VIT_CUDA_TRY(cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, device));
    fp8vit_scratch* scr = nullptr;
    FP8VIT_CUDA_TRY(cudaMalloc(&scr, sizeof(fp8vit_scratch)));
    if (cudaMemset(scr, 0, sizeof(fp8vit_scratch)) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(scr);
        return FP8VIT_ECUDA;
    }
    fp8vit_ctx* c = new fp8vit_ctx;
    c->device = device;
    c->num_sms = sms;
    c->d_scratch = scr;
    c->attn_p_terms = 2;
    c->l2_bytes = l2;
    *out = c;
    return FP8VIT_OK;
}

fp8vit_status fp8vit_destroy(fp8vit_ctx* ctx) {
    if (!ctx) return FP8VIT_OK;
    cudaError_t e = cudaFree(ctx->d_scratch);
    delete ctx;
    return e == cudaSuccess ? FP8VIT_OK : FP8VIT_ECUDA;
}

fp8vit_status fp8vit_tmap_cache_stats(fp8vit_ctx* ctx, uint64_t* hits, uint64_t* misses) {
    if (!ctx || !hits || !misses) return FP8VIT_EINVAL;
    std::lock_guard<std::mutex> lock(ctx->tmap_mu);
    *hits = ctx->tmap_hits;
    *misses = ctx->tmap_misses;
    return FP8VIT_OK;
}

fp8vit_status fp8vit_set_attn_p_terms(fp8vit_ctx* ctx, int32_t terms) {
    if (!ctx || (terms != 1 && terms != 2)) return FP8VIT_EINVAL;
    ctx->attn_p_terms = terms;
    return FP8VIT_OK;
}

fp8vit_status fp8vit_check(fp8vit_ctx* ctx, void* stream, int32_t* site) {
    if (site) *site = 0;
    if (!ctx) return FP8VIT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    FP8VIT_CUDA_TRY(cudaStreamSynchronize(st));
    int32_t hv[2] = {0, 0};
    FP8VIT_CUDA_TRY(cudaMemcpyAsync(hv, ctx->d_scratch, sizeof(hv), cudaMemcpyDeviceToHost, st));
    FP8VIT_CUDA_TRY(cudaStreamSynchronize(st));
    if (hv[0] != 0) {
        // A kernel gave up: clear the status word and the amax reduction state
        // (maxima, arrival counter), which a launch that timed out can leave
        // half-updated.  The stream is idle, and a context serves one stream.
        FP8VIT_CUDA_TRY(cudaMemsetAsync(ctx->d_scratch, 0,
                                        offsetof(fp8vit_scratch, release), st));
        FP8VIT_CUDA_TRY(cudaStreamSynchronize(st));
    }
    if (site) *site = hv[1];
    return static_cast<fp8vit_status>(hv[0]);
}

fp8vit_status fp8vit_inject_lost_arrival(fp8vit_ctx* ctx, void* stream) {
    if (!ctx) return FP8VIT_EINVAL;
    // An arrival count no block can complete: the next fused amax/quantize
    // launch on this context finds no last block, so its barrier wait runs out.
    const uint32_t bogus = 0x40000000u;
    FP8VIT_CUDA_TRY(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(ctx->d_scratch) +
                                        offsetof(fp8vit_scratch, arrivals),
                                    &bogus, sizeof(bogus), cudaMemcpyHostToDevice,
                                    reinterpret_cast<cudaStream_t>(stream)));
    FP8VIT_CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    return FP8VIT_OK;
}

fp8vit_status fp8vit_inject_attn_timeout(fp8vit_ctx* ctx, void* stream) {
    if (!ctx) return FP8VIT_EINVAL;
    // Until the next fp8vit_check clears it, every attention CTA launched on
    // this context skips the commit that announces its first scores, so its
    // softmax warps' bounded wait runs out (the kernel then aborts, drains
    // and returns).
    const uint32_t one = 1u;
    FP8VIT_CUDA_TRY(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(ctx->d_scratch) +
                                        offsetof(fp8vit_scratch, inject_attn),
                                    &one, sizeof(one), cudaMemcpyHostToDevice,
                                    reinterpret_cast<cudaStream_t>(stream)));
    FP8VIT_CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    return FP8VIT_OK;
}

fp8vit_status fp8vit_ring_init(void* d_ring, void* stream) {
    if (!d_ring || (reinterpret_cast<uintptr_t>(d_ring) & 15)) return FP8VIT_EINVAL;
    FP8VIT_CUDA_TRY(cudaMemsetAsync(d_ring, 0, FP8VIT_RING_BYTES,
                                    reinterpret_cast<cudaStream_t>(stream)));
    return FP8VIT_OK;
}

fp8vit_status fp8_ring_read_amax(const void* d_ring, float out_amax3[3], void* stream) {
    if (!d_ring || !out_amax3) return FP8VIT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    fp8vit_ring h;
    FP8VIT_CUDA_TRY(cudaMemcpyAsync(&h, d_ring, sizeof(h), cudaMemcpyDeviceToHost, st));
    FP8VIT_CUDA_TRY(cudaStreamSynchronize(st));
    for (int t = 0; t < 3; ++t) {
        float m = 0.0f;
        for (int j = 0; j < 16; ++j) m = h.hist[t][j] > m ? h.hist[t][j] : m;
        out_amax3[t] = m;
    }
    return FP8VIT_OK;
}

float fp8_descale_from_amax(float v) {
    volatile float num = v;  // keep the fp32 division a real division
    float d = num / 448.0f;
    return d > 1e-10f ? d : 1e-10f;
}

float fp8_descale_from_amax_margin(float amax, float margin) {
    volatile float prod = margin * amax;  // the fp32 product fp8_static_scales_save writes
    return fp8_descale_from_amax(prod);
}

}  // extern "C"

fp8vit_encode_tiled_fn fp8vit_get_encode_tiled() {
    static fp8vit_encode_tiled_fn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<fp8vit_encode_tiled_fn>(p);
    });
    return fn;
}
