// Mamba heads of the mixer, prefill: depthwise causal conv + SiLU, then the
// selective scan ("Jamba: Hybrid SSM-Transformer", How It Actually Works section 1;
// "Lecture 04", section 2):
//     h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) xc_t,   y_t = C_t . h_t + D xc_t
// with A = -exp(A_log) per (channel, state) and the state in fp32 registers.
//
// One block per (8-channel group, sequence), 64 threads; thread (c, p) owns states 2p
// and 2p+1 of channel c and updates both with packed f32x2 arithmetic, so a recurrence
// step is two MUFU exp2 and a few FMA-pipe instructions per thread, and the only serial
// dependency is one FMA per state. Time is walked in chunks of 64 rows, each thread
// staging one row with cp.async while the previous chunk is scanned:
//   unpack   thread t: conv + SiLU of row t for the 8 channels, Delta * xc, B/C pairs;
//   scan     thread (c, p): 64 steps, its partial C.h sums written to shared memory;
//   reduce   thread t: y of row t = the 8 partial sums + D xc, one 16-byte store.
// The sum over the threads of a channel is thus never on the recurrence's path.
#include "kernels.h"

namespace hymba {

namespace {

constexpr int CPB = 8;   // channels per block
constexpr int TPC = 8;   // threads per channel (2 states each)
constexpr int NTH = CPB * TPC;
constexpr int TC = 64;   // rows per chunk (= threads: one row each when staging)
constexpr int KC = 4;    // conv taps
constexpr int PSTR = TC + 4;  // padded row of the partial-sum buffer
constexpr float LOG2E = 1.4426950408889634f;
static_assert(TC == NTH, "staging maps one row per thread");

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

// Thread t queues the copies of row t0 + t of the sequence (rows past Tp repeat the
// last row; their results are never stored and their Delta is zeroed when unpacked).
template <typename T>
__device__ __forceinline__ void stage_row(Raw<T>& r, const T* P, long long ldP, int col_x, int col_B, int col_C,
                                          const float* delta, int di, int c0, long long row0, int t0, int Tp) {
    const int tt = threadIdx.x;
    const long long row = row0 + min(t0 + tt, Tp - 1);
    const T* prow = P + row * ldP;
    constexpr int XV = CPB * (int)sizeof(T) / 16;
    constexpr int BV = 16 * (int)sizeof(T) / 16;
#pragma unroll
    for (int k = 0; k < XV; ++k)
        cp_async16(reinterpret_cast<char*>(&r.x[tt][0]) + 16 * k, reinterpret_cast<const char*>(prow + col_x + c0) + 16 * k);
#pragma unroll
    for (int k = 0; k < CPB * 4 / 16; ++k)
        cp_async16(reinterpret_cast<char*>(&r.d[tt][0]) + 16 * k,
                   reinterpret_cast<const char*>(delta + row * di + c0) + 16 * k);
#pragma unroll
    for (int k = 0; k < BV; ++k) {
        cp_async16(reinterpret_cast<char*>(&r.b[tt][0]) + 16 * k, reinterpret_cast<const char*>(prow + col_B) + 16 * k);
        cp_async16(reinterpret_cast<char*>(&r.c[tt][0]) + 16 * k, reinterpret_cast<const char*>(prow + col_C) + 16 * k);
    }
}

template <typename T>
struct ScanSmem {
    Raw<T> raw[2];
    alignas(16) float2 dd[TC][CPB];            // (Delta, Delta * xc)
    alignas(16) float4 bc[TC][TPC];            // (B_2p, B_2p+1, C_2p, C_2p+1)
    alignas(16) float xd[TC][CPB];             // D * xc
    alignas(16) float part[CPB][TPC][PSTR];    // partial C.h sums
};

template <typename T>
__global__ void __launch_bounds__(NTH)
conv_scan_prefill_kernel(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C,
                         const float* __restrict__ delta, const float* __restrict__ conv_w,
                         const float* __restrict__ conv_b, const float* __restrict__ A_log,
                         const float* __restrict__ Dp, T* __restrict__ ypre, float* __restrict__ h_out,
                         float* __restrict__ conv_out, int Tp, int di) {
    extern __shared__ __align__(16) uint8_t scan_smem[];
    ScanSmem<T>& sm = *reinterpret_cast<ScanSmem<T>*>(scan_smem);
    Raw<T>* raw = sm.raw;
    float2 (*dd)[CPB] = sm.dd;
    float4 (*bc)[TPC] = sm.bc;
    float (*xd)[CPB] = sm.xd;
    float (*part)[TPC][PSTR] = sm.part;
    __shared__ float halo[KC - 1][CPB];
    __shared__ float wconv[CPB][KC + 1];
    __shared__ float dch[CPB];

    const int b = blockIdx.y, c0 = blockIdx.x * CPB;
    const int tid = threadIdx.x, cl = tid / TPC, p = tid % TPC, c = c0 + cl;
    const long long row0 = (long long)b * Tp;
    const float2 A2 = make_float2(-expf(A_log[(long long)c * 16 + 2 * p]) * LOG2E,
                                  -expf(A_log[(long long)c * 16 + 2 * p + 1]) * LOG2E);
    if (tid < (KC - 1) * CPB) halo[tid / CPB][tid % CPB] = 0.f;
    if (tid < CPB) {
        for (int k = 0; k < KC; ++k) wconv[tid][k] = conv_w[(long long)(c0 + tid) * KC + k];
        wconv[tid][KC] = conv_b[c0 + tid];
        dch[tid] = Dp[c0 + tid];
    }
    float2 h = make_float2(0.f, 0.f);
    const int nchunk = (Tp + TC - 1) / TC;

    stage_row<T>(raw[0], P, ldP, col_x, col_B, col_C, delta, di, c0, row0, 0, Tp);
    cp_async_commit();
    for (int k = 0; k < nchunk; ++k) {
        const int t0 = k * TC, nt = min(TC, Tp - t0);
        if (k + 1 < nchunk) stage_row<T>(raw[(k + 1) & 1], P, ldP, col_x, col_B, col_C, delta, di, c0, row0, t0 + TC, Tp);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();  // chunk k staged; previous chunk's reduce done
        const Raw<T>& r = raw[k & 1];
        {
            // unpack row tid
            const int tt = tid;
            float xs[KC][CPB];
#pragma unroll
            for (int q = 0; q < KC; ++q) {
                const int src = tt - (KC - 1) + q;
#pragma unroll
                for (int cc = 0; cc < CPB; ++cc) xs[q][cc] = src >= 0 ? to_f(r.x[src][cc]) : halo[src + KC - 1][cc];
            }
#pragma unroll
            for (int cc = 0; cc < CPB; ++cc) {
                float acc = wconv[cc][KC];
#pragma unroll
                for (int q = 0; q < KC; ++q) acc = fmaf(wconv[cc][q], xs[q][cc], acc);
                const float xc = __fdividef(acc, 1.0f + __expf(-acc));
                // rows past the end of the sequence get Delta = 0: exp2(0) = 1 and a zero
                // input leave the state exactly as it is after the last row
                const float d = tt < nt ? r.d[tt][cc] : 0.f;
                dd[tt][cc] = make_float2(d, d * xc);
                xd[tt][cc] = dch[cc] * xc;
            }
#pragma unroll
            for (int q = 0; q < TPC; ++q)
                bc[tt][q] = make_float4(to_f(r.b[tt][2 * q]), to_f(r.b[tt][2 * q + 1]), to_f(r.c[tt][2 * q]),
                                        to_f(r.c[tt][2 * q + 1]));
            if (k + 1 == nchunk && conv_out && tt < KC) {
                // conv state: the last KC inputs of the sequence, oldest first
                const int src = nt - KC + tt;
#pragma unroll
                for (int cc = 0; cc < CPB; ++cc)
                    conv_out[((long long)b * di + c0 + cc) * KC + tt] =
                        src >= 0 ? to_f(r.x[src][cc]) : (src + KC - 1 >= 0 ? halo[src + KC - 1][cc] : 0.f);
            }
        }
        __syncthreads();  // unpacked; halo readers done
        if (k + 1 < nchunk && tid < (KC - 1) * CPB) {
            const int q = tid / CPB, cc = tid % CPB;
            halo[q][cc] = to_f(r.x[TC - (KC - 1) + q][cc]);
        }
        // scan the chunk in groups of 8 steps, software-pipelined: the shared-memory
        // operands of group g+1 are loaded while group g's exp2s and FMAs run, so each
        // step waits only on its own recurrence FMA
        {
            constexpr int GS = 8;
            float2 dvb[2][GS];
            float4 qb[2][GS];
#pragma unroll
            for (int u = 0; u < GS; ++u) {
                dvb[0][u] = dd[u][cl];
                qb[0][u] = bc[u][p];
            }
#pragma unroll
            for (int g8 = 0; g8 < TC / GS; ++g8) {
                const int cur = g8 & 1;
                if (g8 + 1 < TC / GS) {
#pragma unroll
                    for (int u = 0; u < GS; ++u) {
                        dvb[cur ^ 1][u] = dd[(g8 + 1) * GS + u][cl];
                        qb[cur ^ 1][u] = bc[(g8 + 1) * GS + u][p];
                    }
                }
                float2 a[GS];
#pragma unroll
                for (int u = 0; u < GS; ++u) {
                    const float2 arg = mul2(make_float2(dvb[cur][u].x, dvb[cur][u].x), A2);
                    a[u] = make_float2(fast_exp2(arg.x), fast_exp2(arg.y));
                }
                float yp[GS];
#pragma unroll
                for (int u = 0; u < GS; ++u) {
                    const float4 q = qb[cur][u];
                    h = fma2(a[u], h, mul2(make_float2(dvb[cur][u].y, dvb[cur][u].y), make_float2(q.x, q.y)));
                    const float2 ch = mul2(make_float2(q.z, q.w), h);
                    yp[u] = ch.x + ch.y;
                }
                *reinterpret_cast<float4*>(&part[cl][p][g8 * GS]) = make_float4(yp[0], yp[1], yp[2], yp[3]);
                *reinterpret_cast<float4*>(&part[cl][p][g8 * GS + 4]) = make_float4(yp[4], yp[5], yp[6], yp[7]);
            }
        }
        __syncthreads();  // partial sums complete
        if (tid < nt) {
            const int tt = tid;
            float y[CPB];
#pragma unroll
            for (int cc = 0; cc < CPB; ++cc) {
                float s = xd[tt][cc];
#pragma unroll
                for (int q = 0; q < TPC; ++q) s += part[cc][q][tt];
                y[cc] = s;
            }
            T* dst = ypre + (row0 + t0 + tt) * di + c0;
            if constexpr (sizeof(T) == 2) {
                uint4 v;
                v.x = pack2<T>(y[0], y[1]);
                v.y = pack2<T>(y[2], y[3]);
                v.z = pack2<T>(y[4], y[5]);
                v.w = pack2<T>(y[6], y[7]);
                *reinterpret_cast<uint4*>(dst) = v;
            } else {
                *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[1], y[2], y[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(y[4], y[5], y[6], y[7]);
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
    const size_t smem = sizeof(ScanSmem<T>);
    auto kern = conv_scan_prefill_kernel<T>;
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return HYMBA_ERR_CUDA;
        attr_set = true;
    }
    HYMBA_LAUNCH(ctx, "conv_scan_prefill", kern, grid, NTH, smem, P, ldP, col_x, col_B, col_C, delta, conv_w, conv_b,
                 A_log, D, ypre, h_out, conv_out, Tp, di);
    return HYMBA_OK;
}

template int launch_conv_scan_prefill<float>(const Ctx&, const float*, long long, int, int, int, const float*,
                                             const float*, const float*, const float*, const float*, float*, float*,
                                             float*, int, int, int);
template int launch_conv_scan_prefill<f16>(const Ctx&, const f16*, long long, int, int, int, const float*,
                                           const float*, const float*, const float*, const float*, f16*, float*,
                                           float*, int, int, int);

}  // namespace hymba
