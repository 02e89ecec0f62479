// hymba_attn_decode_static: the split-KV decode attention with its scratch in a
// fixed device array, for callers that cannot allocate device memory (see
// include/hymba.h). It launches the same two kernels as the attention step of
// hymba_mixer_decode; only where the per-split partial results live differs.
#include <mutex>

#include "kernels.h"

namespace hymba {

// Partial results of the key splits: [B, n_q_heads, n_split, v_head_dim + 4] fp32.
// Every GPU that loads the library holds this array until the process exits.
static constexpr size_t kStaticScratchBytes = size_t(8) << 20;
static __device__ __align__(256) float g_decode_scratch[kStaticScratchBytes / sizeof(float)];

static std::mutex g_static_mu;
static float* g_static_ptr[64];  // device address of g_decode_scratch, per device

// Looks up the array's device address once per device, with that device current.
// In host code g_decode_scratch names a host-side stand-in, never the device array.
static int static_scratch(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HYMBA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return HYMBA_ERR_CUDA;
        g_static_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_static_ptr[dev];
    return HYMBA_OK;
}

}  // namespace hymba

using namespace hymba;

extern "C" int hymba_attn_decode_static(const hymba_layer_cfg* cfg, const void* q, int64_t ldq, const hymba_kv* kv,
                                        void* o, int B, void* stream) {
    if (!cfg || !q || !kv || !o || B <= 0) return HYMBA_ERR_INVALID_ARG;
    if (cfg->head_dim != 64 || cfg->v_head_dim != 128 || cfg->n_kv_heads <= 0 || cfg->n_q_heads <= 0 ||
        cfg->n_q_heads % cfg->n_kv_heads || cfg->n_q_heads / cfg->n_kv_heads > 8 ||
        (cfg->dtype != HYMBA_F32 && cfg->dtype != HYMBA_BF16))
        return HYMBA_ERR_UNSUPPORTED;
    if (!kv->k_cache || !kv->v_cache || !kv->len || kv->cache_cap <= cfg->n_meta || kv->batch != B ||
        kv->n_meta != cfg->n_meta || kv->n_kv_heads != cfg->n_kv_heads || kv->head_dim != 64 ||
        kv->v_head_dim != 128 || kv->dtype != (cfg->dtype == HYMBA_BF16 ? HYMBA_F16 : HYMBA_F32))
        return HYMBA_ERR_KV_INCOMPATIBLE;
    if (ldq < (int64_t)cfg->n_q_heads * 64) return HYMBA_ERR_INVALID_ARG;
    const int n_split = (kv->cache_cap + 255) / 256;
    const size_t need = (size_t)B * cfg->n_q_heads * n_split * (cfg->v_head_dim + 4) * sizeof(float);
    if (need > kStaticScratchBytes) return HYMBA_ERR_SCRATCH_LIMIT;
    float* scratch = nullptr;
    int rc = static_scratch(&scratch);
    if (rc) return rc;
    Ctx ctx;
    if ((rc = launch_context(static_cast<cudaStream_t>(stream), &ctx))) return rc;
    // the query sits at the newest position the cache holds: len[b] - 1
    if (cfg->dtype == HYMBA_BF16)
        return launch_attn_decode<f16>(ctx, static_cast<const f16*>(q), ldq, static_cast<const f16*>(kv->k_cache),
                                       static_cast<const f16*>(kv->v_cache), kv->cache_cap, kv->len, -1, scratch,
                                       n_split, static_cast<f16*>(o), B, cfg->n_q_heads, cfg->n_kv_heads,
                                       cfg->v_head_dim, cfg->n_meta, cfg->window);
    return launch_attn_decode<float>(ctx, static_cast<const float*>(q), ldq, static_cast<const float*>(kv->k_cache),
                                     static_cast<const float*>(kv->v_cache), kv->cache_cap, kv->len, -1, scratch,
                                     n_split, static_cast<float*>(o), B, cfg->n_q_heads, cfg->n_kv_heads,
                                     cfg->v_head_dim, cfg->n_meta, cfg->window);
}
