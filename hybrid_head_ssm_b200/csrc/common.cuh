// Shared device helpers and the host-side launch context of libhymba.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "../../include/hymba.h"

namespace hymba {

typedef __nv_bfloat16 bf16;
typedef __half f16;

// ---------------------------------------------------------------------------
// host: launch context and tracing (defined in hymba_abi.cu)
// ---------------------------------------------------------------------------
struct Ctx {
    cudaStream_t stream;
    int* status;   // device status word of the current device
    int sm_count;
    int device;    // current device (0..63)
};

// records the start event when tracing covers this kernel
void trace_before(const Ctx& ctx, const char* name);
// records the end event, counts the launch and checks the launch error; returns true on error
bool trace_after(const Ctx& ctx, const char* name);

// Every kernel of the library is launched with programmatic stream serialization
// (programmatic dependent launch): its CTAs may start while the previous kernel on the
// stream drains, run their setup (barrier init, TMEM allocation, tensor-map prefetch)
// and then block in griddep_wait() until that kernel has completed and its writes are
// visible. Each kernel calls griddep_wait() before its first global memory access and
// then griddep_launch_dependents(), so the next kernel can be scheduled as SMs free up.
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// As launch_pdl, with the grid divided into thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                             unsigned cluster_x, cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#define HYMBA_LAUNCH_CLUSTER(ctx, name, kernel, grid, block, smem, cluster_x, ...)              \
    do {                                                                                         \
        ::hymba::trace_before((ctx), (name));                                                    \
        const cudaError_t launch_err_ = ::hymba::launch_pdl_cluster(                             \
            kernel, dim3(grid), dim3(block), (size_t)(smem), (cluster_x), (ctx).stream, __VA_ARGS__); \
        if (::hymba::trace_after((ctx), (name)) || launch_err_ != cudaSuccess) return HYMBA_ERR_CUDA; \
    } while (0)

#define HYMBA_LAUNCH(ctx, name, kernel, grid, block, smem, ...)                                  \
    do {                                                                                         \
        ::hymba::trace_before((ctx), (name));                                                    \
        const cudaError_t launch_err_ =                                                          \
            ::hymba::launch_pdl(kernel, dim3(grid), dim3(block), (size_t)(smem), (ctx).stream, __VA_ARGS__); \
        if (::hymba::trace_after((ctx), (name)) || launch_err_ != cudaSuccess) return HYMBA_ERR_CUDA; \
    } while (0)

// Opt `kernel` in to `smem` bytes of dynamic shared memory on the context's device, once
// per device: the attribute belongs to the device's context, so a process driving several
// GPUs sets it on each. `done` is the caller's mask of devices already set; threads that
// race here both set the same value.
template <typename K>
static inline bool smem_opt_in_once(std::atomic<unsigned long long>& done, K kernel, size_t smem, const Ctx& ctx) {
    const unsigned long long bit = 1ull << ctx.device;
    if (done.load(std::memory_order_acquire) & bit) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return false;
    done.fetch_or(bit, std::memory_order_release);
    return true;
}

static inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }
static inline long long round_up(long long a, long long b) { return (a + b - 1) / b * b; }

// ---------------------------------------------------------------------------
// device: dtype conversions, status word, fast exp2
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f(f16 v) { return __half2float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ f16 from_f<f16>(float v) { return __float2half_rn(v); }

// Wait for the previous kernel on the stream (programmatic dependent launch), then let
// the next one be scheduled. A no-op pair when the kernel was launched without it.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void griddep_sync() {
    griddep_wait();
    griddep_launch_dependents();
}

// Thread-block cluster primitives: this CTA's rank in its cluster, the cluster-wide
// barrier (every thread of every CTA arrives; release / acquire order shared-memory
// accesses across the cluster), and a load from another CTA's shared memory (DSMEM).
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local)), r;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(r) : "memory");
    return v;
}

__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// 2^x on the MUFU unit (ex2.approx, flush-to-zero).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float silu_f(float u) { return u / (1.0f + expf(-u)); }

__device__ __forceinline__ float softplus_f(float u) {
    return u > 20.0f ? u : log1pf(expf(u));
}

// softplus(u) = max(u, 0) + log(1 + e), e = exp(-|u|) in (0, 1], on the MUFU unit.
// For e < 2^-10 the series e - e^2/2 (+ e^3/3) replaces log(1 + e), whose argument
// would lose e's low bits when rounded to fp32; above it the absolute error of the
// MUFU log (about 1e-7) is below 1e-4 of the result.
__device__ __forceinline__ float softplus_fast(float u) {
    const float e = __expf(-fabsf(u));
    const float l = e < 9.765625e-4f ? e * (1.0f - e * (0.5f - e * (1.0f / 3.0f))) : __logf(1.0f + e);
    return fmaxf(u, 0.0f) + l;
}

// Store n (<= 64) consecutive fp32 values as T at dst (16-byte vector stores when
// the run is full and aligned).
template <typename T>
__device__ __forceinline__ void store_run(T* dst, const float* v, int n);

template <>
__device__ __forceinline__ void store_run<float>(float* dst, const float* v, int n) {
    if (n == 64 && ((uintptr_t)dst & 15) == 0) {
#pragma unroll
        for (int i = 0; i < 64; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
#pragma unroll
        for (int i = 0; i < 64; ++i)
            if (i < n) dst[i] = v[i];
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 p = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<bf16>(float lo, float hi) { return pack_bf16x2(lo, hi); }
template <> __device__ __forceinline__ uint32_t pack2<f16>(float lo, float hi) { return pack_f16x2(lo, hi); }

template <typename T>
__device__ __forceinline__ void store_run16(T* dst, const float* v, int n) {
    if (n == 64 && ((uintptr_t)dst & 15) == 0) {
#pragma unroll
        for (int i = 0; i < 64; i += 8) {
            uint4 q;
            q.x = pack2<T>(v[i], v[i + 1]);
            q.y = pack2<T>(v[i + 2], v[i + 3]);
            q.z = pack2<T>(v[i + 4], v[i + 5]);
            q.w = pack2<T>(v[i + 6], v[i + 7]);
            *reinterpret_cast<uint4*>(dst + i) = q;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 64; ++i)
            if (i < n) dst[i] = from_f<T>(v[i]);
    }
}

template <>
__device__ __forceinline__ void store_run<bf16>(bf16* dst, const float* v, int n) { store_run16<bf16>(dst, v, n); }
template <>
__device__ __forceinline__ void store_run<f16>(f16* dst, const float* v, int n) { store_run16<f16>(dst, v, n); }

}  // namespace hymba
