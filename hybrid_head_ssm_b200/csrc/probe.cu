// hymba_probe_unit_rates: throughput of the execution units that bound the
// CUDA-core kernels of the library (the selective scan's state decays and SiLU run on
// the MUFU exp2 unit; its recurrence and the softmax's scaling on the fp32 FMA pipe),
// measured on the device in results per clock per SM. The benchmark divides the scan's
// MUFU work by this rate instead of a nominal figure.
//
// One block of 1024 threads per SM, each thread running 8 independent chains of one
// instruction kind; a block times its loop with clock64 between two barriers. The
// chains are data dependent, so the compiler keeps every instruction, and 8 chains x 32
// warps keep enough instructions in flight to saturate the unit.
#include <mutex>

#include "kernels.h"

namespace hymba {

namespace {

constexpr int kProbeBlocks = 1024;  // upper bound on the SM count
constexpr int kProbeThreads = 1024;
__device__ unsigned long long g_probe_cycles[kProbeBlocks];
__device__ float g_probe_sink[kProbeBlocks];

__device__ __forceinline__ float ex2f32(float x) {
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t ex2f16x2(uint32_t x) {
    uint32_t y;
    asm volatile("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// mode 0: ex2.approx.f32 (+ one FADD per result to keep the chain bounded); mode 1:
// ex2.approx.f16x2 (two results per instruction, + one HADD2); mode 2: packed fp32 FMA
// (FFMA2, two results per instruction).
__global__ void __launch_bounds__(kProbeThreads, 1) probe_kernel(int iters, int mode) {
    float a[8];
    uint32_t hx[8];
    float2 f[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        a[k] = -0.001f * (float)(threadIdx.x + k);
        const __half2 h = __floats2half2_rn(-0.25f, -0.5f);
        hx[k] = *reinterpret_cast<const uint32_t*>(&h);
        f[k] = make_float2(0.001f * k, 0.002f * k);
    }
    const __half2 hm = __floats2half2_rn(-1.0f, -1.0f);
    const uint32_t hmu = *reinterpret_cast<const uint32_t*>(&hm);
    const float2 fa = make_float2(0.999f, 0.998f), fb = make_float2(0.001f, 0.002f);
    __syncthreads();
    const unsigned long long t0 = clock64();
    if (mode == 0) {
        for (int i = 0; i < iters; ++i)
#pragma unroll
            for (int k = 0; k < 8; ++k) a[k] = ex2f32(a[k]) - 1.5f;
    } else if (mode == 1) {
        for (int i = 0; i < iters; ++i)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t y = ex2f16x2(hx[k]);
                uint32_t z;
                asm volatile("add.rn.f16x2 %0, %1, %2;" : "=r"(z) : "r"(y), "r"(hmu));
                hx[k] = z;
            }
    } else {
        for (int i = 0; i < iters; ++i)
#pragma unroll
            for (int k = 0; k < 8; ++k) f[k] = __ffma2_rn(f[k], fa, fb);
    }
    __syncthreads();
    const unsigned long long t1 = clock64();
    float sink = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const __half2 h = *reinterpret_cast<const __half2*>(&hx[k]);
        sink += a[k] + __low2float(h) + f[k].x + f[k].y;
    }
    if (threadIdx.x == 0) {
        g_probe_cycles[blockIdx.x] = t1 - t0;
        g_probe_sink[blockIdx.x] = sink;
    }
}

}  // namespace

}  // namespace hymba

using namespace hymba;

extern "C" int hymba_probe_unit_rates(double* out, int n, void* stream) {
    if (!out || n < 3) return HYMBA_ERR_INVALID_ARG;
    Ctx ctx;
    int rc = launch_context(static_cast<cudaStream_t>(stream), &ctx);
    if (rc) return rc;
    const int blocks = ctx.sm_count;  // one block per SM (1024 threads, launch bound 1)
    if (blocks <= 0 || blocks > kProbeBlocks) return HYMBA_ERR_UNSUPPORTED;
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    void* cyc_dev = nullptr;
    if (cudaGetSymbolAddress(&cyc_dev, g_probe_cycles) != cudaSuccess) return HYMBA_ERR_CUDA;
    const int iters = 4096;
    // results per thread per mode: 8 chains x iters, x2 for the paired forms
    const double per_thread[3] = {8.0 * iters, 16.0 * iters, 16.0 * iters};
    for (int mode = 0; mode < 3; ++mode) {
        probe_kernel<<<blocks, kProbeThreads, 0, ctx.stream>>>(iters, mode);
        if (cudaGetLastError() != cudaSuccess) return HYMBA_ERR_CUDA;
        unsigned long long cyc[kProbeBlocks];
        if (cudaMemcpyAsync(cyc, cyc_dev, sizeof(unsigned long long) * blocks, cudaMemcpyDeviceToHost, ctx.stream) !=
                cudaSuccess ||
            cudaStreamSynchronize(ctx.stream) != cudaSuccess)
            return HYMBA_ERR_CUDA;
        unsigned long long mx = 1;
        for (int b = 0; b < blocks; ++b) mx = cyc[b] > mx ? cyc[b] : mx;
        out[mode] = per_thread[mode] * kProbeThreads / (double)mx;  // results per clock per SM (slowest SM)
    }
    return HYMBA_OK;
}
