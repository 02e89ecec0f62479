// Causal GQA attention over the meta-token prefix + sliding window on CUDA cores
// (the fp32 layer's path). "Jamba: Hybrid SSM-Transformer", section 1:
// softmax(Q K^T / sqrt(d_k)) V with GQA; 51cto Hymba-1.5B article, section 2:
// sliding-window layers; "Hymba Guide", Learnable Meta-Tokens: every query sees the
// meta keys. Key j is visible to query i iff j <= i and (j < n_meta or i - j < window).
//
// One block per (64-query tile, head, sequence); 4 threads per query, each owning a
// quarter of the head dims and of the V dims; online softmax in base 2.
#include "kernels.h"

namespace hymba {

namespace {

constexpr int DH = 64, QT = 64, KT = 32;

template <typename T, int DV>
__global__ void __launch_bounds__(256)
attn_prefill_simt_kernel(const T* __restrict__ P, long long ldP, const T* __restrict__ kseq,
                         const T* __restrict__ vseq, int kcap, T* __restrict__ O, int Tp, int H,
                         int G, int n_meta, int window, float scale_log2) {
    griddep_sync();
    __shared__ float Ks[KT][DH + 1];
    __shared__ float Vs[KT][DV + 1];
    const int i0 = blockIdx.x * QT, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, qi = tid >> 2, part = tid & 3;
    const int i = i0 + qi;
    const bool qvalid = i < Tp;
    const long long kvbase = ((long long)b * G + g) * kcap;

    float q[16];
    {
        const T* qp = P + ((long long)b * Tp + min(i, Tp - 1)) * ldP + h * DH + part * 16;
#pragma unroll
        for (int e = 0; e < 16; ++e) q[e] = to_f(qp[e]) * scale_log2;
    }
    constexpr int OV = DV / 4;
    float o[OV];
#pragma unroll
    for (int e = 0; e < OV; ++e) o[e] = 0.f;
    float mrun = -INFINITY, l = 0.f;

    const int i_last = min(i0 + QT, Tp) - 1;
    const int meta_end = min(n_meta, i_last + 1);
    const int lo = window > 0 ? max(n_meta, i0 - window + 1) : n_meta;
    const int hi = i_last + 1;
    for (int range = 0; range < 2; ++range) {
        const int start = range == 0 ? 0 : lo;
        const int end = range == 0 ? meta_end : hi;
        for (int j0 = start; j0 < end; j0 += KT) {
            __syncthreads();
            for (int idx = tid; idx < KT * DH; idx += 256) {
                int jj = idx / DH, e = idx % DH, j = j0 + jj;
                Ks[jj][e] = j < end ? to_f(kseq[(kvbase + j) * DH + e]) : 0.f;
            }
            for (int idx = tid; idx < KT * DV; idx += 256) {
                int jj = idx / DV, e = idx % DV, j = j0 + jj;
                Vs[jj][e] = j < end ? to_f(vseq[(kvbase + j) * DV + e]) : 0.f;
            }
            __syncthreads();
            const int nk = min(KT, end - j0);
            for (int jj = 0; jj < nk; ++jj) {
                const int j = j0 + jj;
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) s = fmaf(q[e], Ks[jj][part * 16 + e], s);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                const bool vis = qvalid && j <= i && (j < n_meta || window <= 0 || i - j < window);
                if (vis) {
                    const float mnew = fmaxf(mrun, s);
                    const float corr = exp2f(mrun - mnew);
                    const float p = exp2f(s - mnew);
                    l = l * corr + p;
#pragma unroll
                    for (int e = 0; e < OV; ++e) o[e] = fmaf(p, Vs[jj][part * OV + e], o[e] * corr);
                    mrun = mnew;
                }
            }
        }
    }
    if (qvalid) {
        const float inv = 1.f / l;
        T* op = O + ((long long)b * Tp + i) * ((long long)H * DV) + h * DV + part * OV;
#pragma unroll
        for (int e = 0; e < OV; ++e) op[e] = from_f<T>(o[e] * inv);
    }
}

}  // namespace

template <typename T>
int launch_attn_prefill_simt(const Ctx& ctx, const T* P, long long ldP, const T* k_seq,
                             const T* v_seq, int kcap, T* O, int B, int Tp, int H, int G, int dv,
                             int n_meta, int window) {
    dim3 grid(ceil_div(Tp, QT), H, B);
    const float scale_log2 = 1.4426950408889634f / 8.0f;  // log2(e) / sqrt(64)
    if (dv == 128) {
        auto kern = attn_prefill_simt_kernel<T, 128>;
        HYMBA_LAUNCH(ctx, "attn_prefill_simt", kern, grid, 256, 0,
                     P, ldP, k_seq, v_seq, kcap, O, Tp, H, G, n_meta, window, scale_log2);
    } else if (dv == 64) {
        auto kern = attn_prefill_simt_kernel<T, 64>;
        HYMBA_LAUNCH(ctx, "attn_prefill_simt", kern, grid, 256, 0,
                     P, ldP, k_seq, v_seq, kcap, O, Tp, H, G, n_meta, window, scale_log2);
    } else {
        return HYMBA_ERR_UNSUPPORTED;
    }
    return HYMBA_OK;
}

template int launch_attn_prefill_simt<float>(const Ctx&, const float*, long long, const float*,
                                             const float*, int, float*, int, int, int, int, int,
                                             int, int);
template int launch_attn_prefill_simt<f16>(const Ctx&, const f16*, long long, const f16*,
                                           const f16*, int, f16*, int, int, int, int, int, int,
                                           int);

}  // namespace hymba
