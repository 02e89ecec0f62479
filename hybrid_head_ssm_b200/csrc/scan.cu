// Mamba heads of the mixer, prefill: depthwise causal conv + SiLU, then the
// selective scan ("Jamba: Hybrid SSM-Transformer", How It Actually Works section 1;
// "Lecture 04", section 2):
//     h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) xc_t,   y_t = C_t . h_t + D xc_t
// with A = -exp(A_log) per (channel, state) and the state in fp32 registers.
//
// One block per (8-channel group, sequence), 64 threads; thread (c, p) owns states 2p
// and 2p+1 of channel c and updates both with packed f32x2 arithmetic, so one
// recurrence step is two MUFU exp2 plus a handful of FMA-pipe instructions per thread,
// and the only serial dependency is one FMA per state. Time is walked in chunks of 64
// rows: x, Delta, B and C of the next chunk are copied into shared memory with cp.async
// while the current chunk is scanned; the conv and its SiLU are done once per
// (row, channel) when a chunk is unpacked. The C_t . h_t sum over the 8 threads of a
// channel is deferred: every 8 steps a transpose-reduce (4 + 2 + 1 shuffles) leaves
// thread p with the output of step p, so the reduction is off the recurrence's
// critical path.
#include "kernels.h"

namespace hymba {

namespace {

constexpr int CPB = 8;   // channels per block
constexpr int TPC = 8;   // threads per channel (2 states each)
constexpr int NTH = CPB * TPC;
constexpr int TC = 64;   // rows per chunk
constexpr int KC = 4;    // conv taps
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
    return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(r)
        : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
          "l"(*reinterpret_cast<uint64_t*>(&c)));
    return *reinterpret_cast<float2*>(&r);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename T>
struct Raw {  // one chunk as copied from global memory
    alignas(16) T x[TC][CPB];
    alignas(16) float d[TC][CPB];
    alignas(16) T b[TC][16];
    alignas(16) T c[TC][16];
};

// Queue the cp.async copies of rows [t0, t0 + TC) of sequence b (rows past Tp repeat
// the last row; their results are never stored).
template <typename T>
__device__ __forceinline__ void stage(Raw<T>& r, const T* P, long long ldP, int col_x, int col_B, int col_C,
                                      const float* delta, int di, int c0, long long row0, int t0, int Tp) {
    constexpr int XV = CPB * (int)sizeof(T) / 16;  // 16-byte pieces per row of x
    constexpr int BV = 16 * (int)sizeof(T) / 16;   // ... of B (and of C)
    constexpr int DVp = CPB * 4 / 16;              // ... of Delta
    constexpr int PER_ROW = XV + DVp + 2 * BV;
    for (int i = threadIdx.x; i < TC * PER_ROW; i += NTH) {
        const int tt = i / PER_ROW, k = i % PER_ROW;
        const long long row = row0 + min(t0 + tt, Tp - 1);
        const T* prow = P + row * ldP;
        if (k < XV) {
            cp_async16(reinterpret_cast<char*>(&r.x[tt][0]) + 16 * k,
                       reinterpret_cast<const char*>(prow + col_x + c0) + 16 * k);
        } else if (k < XV + DVp) {
            const int q = k - XV;
            cp_async16(reinterpret_cast<char*>(&r.d[tt][0]) + 16 * q,
                       reinterpret_cast<const char*>(delta + row * di + c0) + 16 * q);
        } else if (k < XV + DVp + BV) {
            const int q = k - XV - DVp;
            cp_async16(reinterpret_cast<char*>(&r.b[tt][0]) + 16 * q, reinterpret_cast<const char*>(prow + col_B) + 16 * q);
        } else {
            const int q = k - XV - DVp - BV;
            cp_async16(reinterpret_cast<char*>(&r.c[tt][0]) + 16 * q, reinterpret_cast<const char*>(prow + col_C) + 16 * q);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(NTH)
conv_scan_prefill_kernel(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C,
                         const float* __restrict__ delta, const float* __restrict__ conv_w,
                         const float* __restrict__ conv_b, const float* __restrict__ A_log,
                         const float* __restrict__ Dp, T* __restrict__ ypre, float* __restrict__ h_out,
                         float* __restrict__ conv_out, int Tp, int di) {
    __shared__ Raw<T> raw[2];
    __shared__ float2 dd[TC][CPB];   // (Delta, Delta * xc)
    __shared__ float4 bc[TC][TPC];   // (B_2p, B_2p+1, C_2p, C_2p+1)
    __shared__ float xd[TC][CPB];    // D * xc
    __shared__ float ys[TC][CPB];
    __shared__ float halo[KC - 1][CPB];
    __shared__ float wconv[CPB][KC + 1];

    const int b = blockIdx.y, c0 = blockIdx.x * CPB;
    const int tid = threadIdx.x, cl = tid / TPC, p = tid % TPC, c = c0 + cl;
    const long long row0 = (long long)b * Tp;
    const float2 A2 = make_float2(-expf(A_log[(long long)c * 16 + 2 * p]) * LOG2E,
                                  -expf(A_log[(long long)c * 16 + 2 * p + 1]) * LOG2E);
    if (tid < (KC - 1) * CPB) halo[tid / CPB][tid % CPB] = 0.f;
    if (tid < CPB) {
        for (int k = 0; k < KC; ++k) wconv[tid][k] = conv_w[(long long)(c0 + tid) * KC + k];
        wconv[tid][KC] = conv_b[c0 + tid];
    }
    float2 h = make_float2(0.f, 0.f);
    const int nchunk = (Tp + TC - 1) / TC;

    stage<T>(raw[0], P, ldP, col_x, col_B, col_C, delta, di, c0, row0, 0, Tp);
    cp_async_commit();
    for (int k = 0; k < nchunk; ++k) {
        const int t0 = k * TC, nt = min(TC, Tp - t0);
        if (k + 1 < nchunk)
            stage<T>(raw[(k + 1) & 1], P, ldP, col_x, col_B, col_C, delta, di, c0, row0, t0 + TC, Tp);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();
        Raw<T>& r = raw[k & 1];
        // unpack: conv + SiLU per (row, channel), B/C to fp32 pairs
        for (int i = tid; i < TC * CPB; i += NTH) {
            const int tt = i / CPB, cc = i % CPB;
            float acc = wconv[cc][KC];
#pragma unroll
            for (int q = 0; q < KC; ++q) {
                const int src = tt - (KC - 1) + q;
                const float xv = src >= 0 ? to_f(r.x[src][cc]) : halo[src + KC - 1][cc];
                acc = fmaf(wconv[cc][q], xv, acc);
            }
            const float xc = silu_f(acc);
            // rows past the end of the sequence get Delta = 0: exp2(0) = 1 and a zero
            // input leave the state exactly as it is after the last row
            const float d = tt < nt ? r.d[tt][cc] : 0.f;
            dd[tt][cc] = make_float2(d, d * xc);
            xd[tt][cc] = Dp[c0 + cc] * xc;
        }
        for (int i = tid; i < TC * TPC; i += NTH) {
            const int tt = i / TPC, q = i % TPC;
            bc[tt][q] = make_float4(to_f(r.b[tt][2 * q]), to_f(r.b[tt][2 * q + 1]), to_f(r.c[tt][2 * q]),
                                    to_f(r.c[tt][2 * q + 1]));
        }
        __syncthreads();
        if (k + 1 < nchunk && tid < (KC - 1) * CPB) {
            const int q = tid / CPB, cc = tid % CPB;
            halo[q][cc] = to_f(r.x[TC - (KC - 1) + q][cc]);
        }
        if (k + 1 == nchunk && conv_out && tid < KC * CPB) {
            // conv state: the last KC inputs of the sequence, oldest first
            const int q = tid / CPB, cc = tid % CPB;
            const int src = nt - KC + q;
            conv_out[((long long)b * di + c0 + cc) * KC + q] =
                src >= 0 ? to_f(r.x[src][cc]) : (src + KC - 1 >= 0 ? halo[src + KC - 1][cc] : 0.f);
        }
        // scan: 8 steps at a time, then the deferred C.h reduction
#pragma unroll 1
        for (int t8 = 0; t8 < TC; t8 += 8) {
            float yp[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float2 dv = dd[t8 + u][cl];
                const float4 q = bc[t8 + u][p];
                const float2 arg = mul2(make_float2(dv.x, dv.x), A2);
                const float2 a = make_float2(fast_exp2(arg.x), fast_exp2(arg.y));
                h = fma2(a, h, mul2(make_float2(dv.y, dv.y), make_float2(q.x, q.y)));
                const float2 ch = mul2(make_float2(q.z, q.w), h);
                yp[u] = ch.x + ch.y;
            }
            // transpose-reduce over the 8 threads of the channel: thread p ends with step p
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool hi = p & 4;
                const float send = hi ? yp[i] : yp[i + 4];
                const float keep = hi ? yp[i + 4] : yp[i];
                yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const bool hi = p & 2;
                const float send = hi ? yp[i] : yp[i + 2];
                const float keep = hi ? yp[i + 2] : yp[i];
                yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            }
            {
                const bool hi = p & 1;
                const float send = hi ? yp[0] : yp[1];
                const float keep = hi ? yp[1] : yp[0];
                yp[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
            }
            ys[t8 + p][cl] = yp[0] + xd[t8 + p][cl];
        }
        __syncthreads();
        // store the chunk: one row of 8 channels per thread
        for (int tt = tid; tt < nt; tt += NTH) {
            T* dst = ypre + (row0 + t0 + tt) * di + c0;
            if constexpr (sizeof(T) == 2) {
                uint4 v;
                v.x = pack2<T>(ys[tt][0], ys[tt][1]);
                v.y = pack2<T>(ys[tt][2], ys[tt][3]);
                v.z = pack2<T>(ys[tt][4], ys[tt][5]);
                v.w = pack2<T>(ys[tt][6], ys[tt][7]);
                *reinterpret_cast<uint4*>(dst) = v;
            } else {
                *reinterpret_cast<float4*>(dst) = make_float4(ys[tt][0], ys[tt][1], ys[tt][2], ys[tt][3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(ys[tt][4], ys[tt][5], ys[tt][6], ys[tt][7]);
            }
        }
    }
    cp_async_wait0();
    if (h_out) {
        float* dst = h_out + ((long long)b * di + c) * 16 + 2 * p;
        dst[0] = h.x;
        dst[1] = h.y;
    }
}

}  // namespace

template <typename T>
int launch_conv_scan_prefill(const Ctx& ctx, const T* P, long long ldP, int col_x, int col_B, int col_C,
                             const float* delta, const float* conv_w, const float* conv_b, const float* A_log,
                             const float* D, T* ypre, float* h_out, float* conv_out, int B, int Tp, int di) {
    if (di % CPB || (col_x % 8) || (col_B % 8) || (col_C % 8) || (ldP % 8)) return HYMBA_ERR_UNSUPPORTED;
    dim3 grid(di / CPB, B);
    HYMBA_LAUNCH(ctx, "conv_scan_prefill", conv_scan_prefill_kernel<T>, grid, NTH, 0, P, ldP, col_x, col_B, col_C,
                 delta, conv_w, conv_b, A_log, D, ypre, h_out, conv_out, Tp, di);
    return HYMBA_OK;
}

template int launch_conv_scan_prefill<float>(const Ctx&, const float*, long long, int, int, int, const float*,
                                             const float*, const float*, const float*, const float*, float*, float*,
                                             float*, int, int, int);
template int launch_conv_scan_prefill<f16>(const Ctx&, const f16*, long long, int, int, int, const float*,
                                           const float*, const float*, const float*, const float*, f16*, float*,
                                           float*, int, int, int);

}  // namespace hymba
