// Fusion epilogue of the two head families: SiLU(z) gate of the Mamba branch,
// RMSNorm of each branch over its full width, beta1 / beta2 scaling and average:
//     Y = y_pre * SiLU(z),  U = (beta1 * g_a * O / rms(O) + beta2 * g_s * Y / rms(Y)) / 2
// ("Hymba Guide", Parallel Hybrid-Head Layer Formulation: both families feed one
// output projection; the normalise-scale-average form is the reading used here for
// how they are combined). One block per row; the row is staged in shared memory so
// HBM is read once and U written once.
#include "kernels.h"

namespace hymba {

namespace {

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
    const int nw = blockDim.x >> 5;
    for (int w = 0; w < nw; ++w) s += red[w];
    __syncthreads();
    return s;
}

template <typename I, typename T>
__global__ void __launch_bounds__(256)
fuse_kernel(const I* __restrict__ O, const I* __restrict__ ypre, const I* __restrict__ P,
            long long ldP, int col_z, const float* __restrict__ g_attn,
            const float* __restrict__ g_ssm, const float* __restrict__ beta1,
            const float* __restrict__ beta2, T* __restrict__ U, int di, float eps, int* len_inc) {
    extern __shared__ float sm[];
    float* so = sm;
    float* sy = sm + di;
    __shared__ float red[32];
    const long long row = blockIdx.x;
    float ss_o = 0.f, ss_y = 0.f;
    for (int c = threadIdx.x; c < di; c += blockDim.x) {
        const float o = to_f(O[row * di + c]);
        const float z = to_f(P[row * ldP + col_z + c]);
        const float y = to_f(ypre[row * di + c]) * silu_f(z);
        so[c] = o;
        sy[c] = y;
        ss_o = fmaf(o, o, ss_o);
        ss_y = fmaf(y, y, ss_y);
    }
    ss_o = block_sum(ss_o, red);
    ss_y = block_sum(ss_y, red);
    const float ro = 1.0f / sqrtf(ss_o / di + eps);
    const float ry = 1.0f / sqrtf(ss_y / di + eps);
    for (int c = threadIdx.x; c < di; c += blockDim.x) {
        const float u = 0.5f * (beta1[c] * g_attn[c] * so[c] * ro + beta2[c] * g_ssm[c] * sy[c] * ry);
        U[row * di + c] = from_f<T>(u);
    }
    if (len_inc && threadIdx.x == 0) len_inc[row] += 1;
}

}  // namespace

template <typename I, typename T>
int launch_fuse(const Ctx& ctx, const I* O, const I* ypre, const I* P, long long ldP, int col_z,
                const float* g_attn, const float* g_ssm, const float* beta1, const float* beta2,
                T* U, int rows, int di, float eps, int* len_inc) {
    if (rows <= 0) return HYMBA_OK;
    const size_t smem = (size_t)2 * di * sizeof(float);
    auto kern = fuse_kernel<I, T>;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return HYMBA_ERR_CUDA;
    }
    HYMBA_LAUNCH(ctx, "fuse", kern, rows, 256, smem, O, ypre, P, ldP, col_z, g_attn, g_ssm, beta1,
                 beta2, U, di, eps, len_inc);
    return HYMBA_OK;
}

template int launch_fuse<float, float>(const Ctx&, const float*, const float*, const float*, long long,
                                       int, const float*, const float*, const float*, const float*,
                                       float*, int, int, float, int*);
template int launch_fuse<f16, bf16>(const Ctx&, const f16*, const f16*, const f16*, long long, int,
                                    const float*, const float*, const float*, const float*, bf16*, int,
                                    int, float, int*);

}  // namespace hymba
