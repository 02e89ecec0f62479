// CUDA-core GEMM C = A B^T with fp32 accumulation. It is the path of the fp32 layer
// (tensor-core TF32 would not meet the fp32 tolerance) and of shapes the tcgen05
// GEMM does not take. 64x64 output tile per block, 256 threads, 4x4 per thread.
#include "kernels.h"

namespace hymba {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename TA, typename TO>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(const TA* __restrict__ A, long long lda, const TA* __restrict__ Bw, long long ldb,
                 int M, int N, int K, EpiArgs<TO> e) {
    griddep_sync();
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    __shared__ float Cs[TM][TN + 1];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < K; k0 += TK) {
        for (int i = tid; i < TM * TK; i += 256) {
            int r = i / TK, kk = i % TK;
            int gr = m0 + r, gk = k0 + kk;
            As[kk][r] = (gr < M && gk < K) ? to_f(A[(long long)gr * lda + gk]) : 0.f;
            int gn = n0 + r;
            Bs[kk][r] = (gn < N && gk < K) ? to_f(Bw[(long long)gn * ldb + gk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Cs[ty * 4 + i][tx * 4 + j] = acc[i][j];
    __syncthreads();
    if (tid < TM) {
        float v[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = Cs[tid][j];
        epi_run64<TO>(e, m0 + tid, n0, v);
    }
}

}  // namespace

template <typename TA, typename TO>
int launch_gemm_simt(const Ctx& ctx, const char* name, const TA* A, long long lda, const TA* Bw, long long ldb,
                     int M, int N, int K, const EpiArgs<TO>& e) {
    if (M <= 0 || N <= 0) return HYMBA_OK;
    if (e.accumulate) return HYMBA_ERR_UNSUPPORTED;  // split-K partial sums run on the tensor-core GEMM
    dim3 grid(ceil_div(N, TN), ceil_div(M, TM));
    auto kern = gemm_simt_kernel<TA, TO>;
    HYMBA_LAUNCH(ctx, name, kern, grid, 256, 0, A, lda, Bw, ldb, M, N, K, e);
    return HYMBA_OK;
}

#define INST(TA, TO)                                                                              \
    template int launch_gemm_simt<TA, TO>(const Ctx&, const char*, const TA*, long long, const TA*, long long, \
                                          int, int, int, const EpiArgs<TO>&);
INST(float, float)
INST(bf16, f16)
INST(f16, f16)
INST(bf16, bf16)
INST(bf16, float)
INST(f16, float)
INST(f16, bf16)
#undef INST

}  // namespace hymba
