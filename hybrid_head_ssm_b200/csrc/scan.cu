// Mamba heads of the mixer, prefill: depthwise causal conv + SiLU, then the
// selective scan ("Jamba: Hybrid SSM-Transformer", How It Actually Works section 1;
// "Lecture 04", section 2):
//     h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) xc_t,   y_t = C_t . h_t + D xc_t
// with A = -exp(A_log) per (channel, state), fp32 state in registers.
//
// Layout: one block per (16-channel group, sequence); thread (c, n) owns state n of
// channel c, so each recurrence step is one exp2 and two FMAs per thread and the
// output is a 16-lane shuffle reduction. Time is walked in chunks of 32 rows staged
// in shared memory (x with a 3-row halo for the conv, Delta, B, C); the conv and its
// SiLU are done once per (row, channel) in the staging step.
#include "kernels.h"

namespace hymba {

namespace {

constexpr int CH = 16, NS = 16, TC = 32, KC = 4;
constexpr float LOG2E = 1.4426950408889634f;

template <typename T>
__global__ void __launch_bounds__(CH * NS)
conv_scan_prefill_kernel(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C,
                         const float* __restrict__ delta, const float* __restrict__ conv_w,
                         const float* __restrict__ conv_b, const float* __restrict__ A_log,
                         const float* __restrict__ Dp, T* __restrict__ ypre, float* __restrict__ h_out,
                         float* __restrict__ conv_out, int Tp, int di) {
    __shared__ float xs[TC + KC - 1][CH];
    __shared__ float ds[TC][CH];
    __shared__ float xcs[TC][CH];
    __shared__ float bs[TC][NS];
    __shared__ float cs[TC][NS];
    __shared__ float ys[TC][CH];
    const int b = blockIdx.y, c0 = blockIdx.x * CH;
    const int tid = threadIdx.x, cl = tid / NS, n = tid % NS, c = c0 + cl;
    const float A2 = -expf(A_log[(long long)c * NS + n]) * LOG2E;
    const float Dc = Dp[c];
    float h = 0.f;
    if (tid < (KC - 1) * CH) xs[tid / CH][tid % CH] = 0.f;

    for (int t0 = 0; t0 < Tp; t0 += TC) {
        const int nt = min(TC, Tp - t0);
        for (int idx = tid; idx < TC * CH; idx += CH * NS) {
            const int tt = idx / CH, cc = idx % CH;
            float xv = 0.f, dv = 0.f;
            if (tt < nt) {
                const long long row = (long long)b * Tp + t0 + tt;
                xv = to_f(P[row * ldP + col_x + c0 + cc]);
                dv = delta[row * di + c0 + cc];
            }
            xs[KC - 1 + tt][cc] = xv;
            ds[tt][cc] = dv;
        }
        for (int idx = tid; idx < TC * NS; idx += CH * NS) {
            const int tt = idx / NS, nn = idx % NS;
            float bv = 0.f, cv = 0.f;
            if (tt < nt) {
                const long long row = (long long)b * Tp + t0 + tt;
                bv = to_f(P[row * ldP + col_B + nn]);
                cv = to_f(P[row * ldP + col_C + nn]);
            }
            bs[tt][nn] = bv;
            cs[tt][nn] = cv;
        }
        __syncthreads();
        for (int idx = tid; idx < TC * CH; idx += CH * NS) {
            const int tt = idx / CH, cc = idx % CH;
            const float* w = conv_w + (long long)(c0 + cc) * KC;
            float acc = conv_b[c0 + cc];
#pragma unroll
            for (int k = 0; k < KC; ++k) acc = fmaf(w[k], xs[tt + k][cc], acc);
            xcs[tt][cc] = silu_f(acc);
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const float d = ds[tt][cl];
            const float xc = xcs[tt][cl];
            const float a = fast_exp2(d * A2);
            h = fmaf(a, h, (d * xc) * bs[tt][n]);
            float part = cs[tt][n] * h;
            part += __shfl_xor_sync(0xffffffffu, part, 8);
            part += __shfl_xor_sync(0xffffffffu, part, 4);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            if (n == 0) ys[tt][cl] = fmaf(Dc, xc, part);
        }
        __syncthreads();
        for (int idx = tid; idx < TC * CH; idx += CH * NS) {
            const int tt = idx / CH, cc = idx % CH;
            if (tt < nt) ypre[((long long)b * Tp + t0 + tt) * di + c0 + cc] = from_f<T>(ys[tt][cc]);
        }
        if (t0 + TC >= Tp) {
            // last chunk: conv state = the last KC inputs, oldest first
            if (conv_out && tid < KC * CH) {
                const int k = tid / CH, cc = tid % CH;
                conv_out[((long long)b * di + c0 + cc) * KC + k] = xs[nt - 1 + k][cc];
            }
        } else {
            __syncthreads();
            if (tid < (KC - 1) * CH) {
                const int k = tid / CH, cc = tid % CH;
                xs[k][cc] = xs[nt + k][cc];
            }
            __syncthreads();
        }
    }
    if (h_out) h_out[((long long)b * di + c) * NS + n] = h;
}

}  // namespace

template <typename T>
int launch_conv_scan_prefill(const Ctx& ctx, const T* P, long long ldP, int col_x, int col_B,
                             int col_C, const float* delta, const float* conv_w,
                             const float* conv_b, const float* A_log, const float* D, T* ypre,
                             float* h_out, float* conv_out, int B, int Tp, int di) {
    if (di % CH) return HYMBA_ERR_UNSUPPORTED;
    dim3 grid(di / CH, B);
    HYMBA_LAUNCH(ctx, "conv_scan_prefill", conv_scan_prefill_kernel<T>, grid, CH * NS, 0, P, ldP,
                 col_x, col_B, col_C, delta, conv_w, conv_b, A_log, D, ypre, h_out, conv_out, Tp, di);
    return HYMBA_OK;
}

template int launch_conv_scan_prefill<float>(const Ctx&, const float*, long long, int, int, int,
                                             const float*, const float*, const float*,
                                             const float*, const float*, float*, float*, float*,
                                             int, int, int);
template int launch_conv_scan_prefill<f16>(const Ctx&, const f16*, long long, int, int, int,
                                           const float*, const float*, const float*,
                                           const float*, const float*, f16*, float*, float*,
                                           int, int, int);

}  // namespace hymba
