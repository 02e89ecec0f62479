// Mamba heads of the mixer, prefill: depthwise causal conv + SiLU, then the
// selective scan ("Jamba: Hybrid SSM-Transformer", How It Actually Works section 1;
// "Lecture 04", section 2):
//     h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) xc_t,   y_t = C_t . h_t + D xc_t
// with A = -exp(A_log) per (channel, state) and the state in fp32 registers.
//
// One block per (8-channel group, sequence), 64 threads; thread (c, p) owns states 2p
// and 2p+1 of channel c and updates both with packed f32x2 arithmetic (__ffma2_rn and
// friends), so a recurrence step is two MUFU exp2 and four FMA-pipe instructions, and
// the only serial dependency is one FFMA2 per step. Time is walked in chunks of 64
// rows; while a chunk is processed the next one is staged with cp.async:
//   unpack   thread t: conv + SiLU of row t for the 8 channels (as 4 channel pairs),
//            (Delta, Delta, Delta*xc, Delta*xc) quads and (B, B, C, C) quads, so the
//            scan reads each operand pair ready-made with one 16-byte load;
//   scan     thread (c, p): 64 steps, its partial C.h sum of each step to shared memory;
//   reduce   thread t: y of row t = the 8 partial sums + D xc, one 16-byte store.
// The chunk's x rows sit after three halo rows (the previous chunk's last three rows,
// zero before the sequence), so the causal conv needs no branches. Shared-memory rows
// are padded so that the unpack's per-row stores spread over all banks.
#include "kernels.h"

namespace hymba {

namespace {

constexpr int CPB = 8;             // channels per block
constexpr int TPC = 8;             // threads per channel (2 states each)
constexpr int NTH = CPB * TPC;
constexpr int TC = 64;             // rows per chunk (one row per thread in unpack and reduce)
constexpr int KC = 4;              // conv taps
constexpr int GS = 4;              // steps per software-pipelined group of the scan
constexpr int PCS = TC * TPC + 8;  // channel stride of the partial-sum buffer (floats)
constexpr float LOG2E = 1.4426950408889634f;
static_assert(TC == NTH, "unpack and reduce map one row per thread");

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 exp2_pair(float2 a) { return make_float2(fast_exp2(a.x), fast_exp2(a.y)); }

template <typename T>
struct Raw {  // one chunk as copied from global memory
    alignas(16) T x[TC + KC - 1][CPB];   // rows 0..2: the three rows before the chunk
    alignas(16) float d[TC][CPB];
    alignas(16) T b[TC][16];
    alignas(16) T c[TC][16];
};

template <typename T>
struct ScanSmem {
    Raw<T> raw[2];
    alignas(16) float4 dd[TC][CPB + 1];      // (Delta, Delta, Delta*xc, Delta*xc), padded rows
    alignas(16) float4 bc[TC][TPC + 1];      // (B_2p, B_2p+1, C_2p, C_2p+1), padded rows
    alignas(16) float xd[TC][12];            // D * xc (8 used), padded rows
    alignas(16) float part[CPB * PCS];       // [channel][row][p] partial C.h sums
    alignas(16) float2 w2[KC + 2][CPB / 2];  // conv taps, conv bias and D as channel pairs
};

// 8 consecutive values as 4 float pairs
template <typename T>
__device__ __forceinline__ void load8x2(const T* p, float2* v) {
    if constexpr (sizeof(T) == 2) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        v[0] = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        v[1] = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        v[2] = __half22float2(*reinterpret_cast<const __half2*>(&u.z));
        v[3] = __half22float2(*reinterpret_cast<const __half2*>(&u.w));
    } else {
        const float4 a = reinterpret_cast<const float4*>(p)[0];
        const float4 b = reinterpret_cast<const float4*>(p)[1];
        v[0] = make_float2(a.x, a.y);
        v[1] = make_float2(a.z, a.w);
        v[2] = make_float2(b.x, b.y);
        v[3] = make_float2(b.z, b.w);
    }
}

// Queue the copies of rows t0 .. t0+TC-1 of the sequence (rows past Tp repeat the last
// row; their results are never stored and their Delta is zeroed when unpacked).
template <typename T>
__device__ __forceinline__ void stage_chunk(Raw<T>& r, const T* P, long long ldP, int col_x, int col_B, int col_C,
                                            const float* delta, int di, int c0, long long row0, int t0, int Tp) {
    constexpr int XV = CPB * (int)sizeof(T) / 16;  // 16-byte pieces per row
    constexpr int DV = CPB * 4 / 16;
    constexpr int BV = 16 * (int)sizeof(T) / 16;
    const int tid = threadIdx.x;
#pragma unroll
    for (int j = tid; j < TC * XV; j += NTH) {
        const int rr = j / XV, k = j % XV;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp_async16(reinterpret_cast<char*>(&r.x[rr + KC - 1][0]) + 16 * k,
                   reinterpret_cast<const char*>(P + row * ldP + col_x + c0) + 16 * k);
    }
#pragma unroll
    for (int j = tid; j < TC * DV; j += NTH) {
        const int rr = j / DV, k = j % DV;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp_async16(reinterpret_cast<char*>(&r.d[rr][0]) + 16 * k,
                   reinterpret_cast<const char*>(delta + row * di + c0) + 16 * k);
    }
#pragma unroll
    for (int j = tid; j < TC * BV; j += NTH) {
        const int rr = j / BV, k = j % BV;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp_async16(reinterpret_cast<char*>(&r.b[rr][0]) + 16 * k,
                   reinterpret_cast<const char*>(P + row * ldP + col_B) + 16 * k);
        cp_async16(reinterpret_cast<char*>(&r.c[rr][0]) + 16 * k,
                   reinterpret_cast<const char*>(P + row * ldP + col_C) + 16 * k);
    }
}

template <typename T>
__global__ void __launch_bounds__(NTH)
conv_scan_prefill_kernel(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C,
                         const float* __restrict__ delta, const float* __restrict__ conv_w,
                         const float* __restrict__ conv_b, const float* __restrict__ A_log,
                         const float* __restrict__ Dp, T* __restrict__ ypre, float* __restrict__ h_out,
                         float* __restrict__ conv_out, int Tp, int di) {
    griddep_sync();
    extern __shared__ __align__(16) uint8_t scan_smem[];
    ScanSmem<T>& sm = *reinterpret_cast<ScanSmem<T>*>(scan_smem);
    const int b = blockIdx.y, c0 = blockIdx.x * CPB;
    const int tid = threadIdx.x, cl = tid / TPC, p = tid % TPC;
    const long long row0 = (long long)b * Tp;
    // A * log2(e) for the thread's two states: exp(Delta A) = exp2(Delta * A2)
    const float2 A2 = make_float2(-expf(A_log[(long long)(c0 + cl) * 16 + 2 * p]) * LOG2E,
                                  -expf(A_log[(long long)(c0 + cl) * 16 + 2 * p + 1]) * LOG2E);
    if (tid < (KC + 2) * (CPB / 2)) {
        const int q = tid / (CPB / 2), j = tid % (CPB / 2);
        const int ca = c0 + 2 * j, cb = ca + 1;
        float2 v;
        if (q < KC) v = make_float2(conv_w[(long long)ca * KC + q], conv_w[(long long)cb * KC + q]);
        else if (q == KC) v = make_float2(conv_b[ca], conv_b[cb]);
        else v = make_float2(Dp[ca], Dp[cb]);
        sm.w2[q][j] = v;
    }
    if (tid < (KC - 1) * CPB) sm.raw[0].x[tid / CPB][tid % CPB] = from_f<T>(0.f);
    float2 h = make_float2(0.f, 0.f);
    const int nchunk = (Tp + TC - 1) / TC;

    stage_chunk<T>(sm.raw[0], P, ldP, col_x, col_B, col_C, delta, di, c0, row0, 0, Tp);
    cp_async_commit();
    for (int k = 0; k < nchunk; ++k) {
        const int t0 = k * TC, nt = min(TC, Tp - t0);
        if (k + 1 < nchunk)
            stage_chunk<T>(sm.raw[(k + 1) & 1], P, ldP, col_x, col_B, col_C, delta, di, c0, row0, t0 + TC, Tp);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();  // chunk k staged; previous chunk's reduce done
        const Raw<T>& r = sm.raw[k & 1];
        {
            // unpack row t
            const int t = tid;
            float2 acc[CPB / 2];
#pragma unroll
            for (int j = 0; j < CPB / 2; ++j) acc[j] = sm.w2[KC][j];
#pragma unroll
            for (int q = 0; q < KC; ++q) {
                float2 xv[CPB / 2];
                load8x2<T>(&r.x[t + q][0], xv);
#pragma unroll
                for (int j = 0; j < CPB / 2; ++j) acc[j] = __ffma2_rn(sm.w2[q][j], xv[j], acc[j]);
            }
            const float4 da = *reinterpret_cast<const float4*>(&r.d[t][0]);
            const float4 db = *reinterpret_cast<const float4*>(&r.d[t][4]);
            // rows past the end of the sequence get Delta = 0: exp2(0) = 1 and a zero
            // input leave the state exactly as it is after the last row
            const float keep = t < nt ? 1.f : 0.f;
            const float2 dl[CPB / 2] = {make_float2(da.x, da.y), make_float2(da.z, da.w), make_float2(db.x, db.y),
                                        make_float2(db.z, db.w)};
            float2 xdv[CPB / 2];
#pragma unroll
            for (int j = 0; j < CPB / 2; ++j) {
                // SiLU(u) = u / (1 + exp(-u))
                const float2 e = exp2_pair(__fmul2_rn(acc[j], make_float2(-LOG2E, -LOG2E)));
                const float2 den = __fadd2_rn(e, make_float2(1.f, 1.f));
                const float2 xc = __fmul2_rn(acc[j], make_float2(rcp_approx(den.x), rcp_approx(den.y)));
                const float2 d = __fmul2_rn(dl[j], make_float2(keep, keep));
                const float2 dv = __fmul2_rn(d, xc);
                sm.dd[t][2 * j] = make_float4(d.x, d.x, dv.x, dv.x);
                sm.dd[t][2 * j + 1] = make_float4(d.y, d.y, dv.y, dv.y);
                xdv[j] = __fmul2_rn(sm.w2[KC + 1][j], xc);
            }
            *reinterpret_cast<float4*>(&sm.xd[t][0]) = make_float4(xdv[0].x, xdv[0].y, xdv[1].x, xdv[1].y);
            *reinterpret_cast<float4*>(&sm.xd[t][4]) = make_float4(xdv[2].x, xdv[2].y, xdv[3].x, xdv[3].y);
            float2 bv[8], cv[8];
            load8x2<T>(&r.b[t][0], bv);
            load8x2<T>(&r.b[t][8], bv + 4);
            load8x2<T>(&r.c[t][0], cv);
            load8x2<T>(&r.c[t][8], cv + 4);
#pragma unroll
            for (int q = 0; q < TPC; ++q) sm.bc[t][q] = make_float4(bv[q].x, bv[q].y, cv[q].x, cv[q].y);
        }
        if (k + 1 < nchunk) {
            if (tid < KC - 1) {
                // halo of the next chunk: this chunk's last three rows of x (the next
                // chunk's copies write rows 3.. of that buffer only)
                const uint4* src = reinterpret_cast<const uint4*>(&r.x[TC + tid][0]);
                uint4* dst = reinterpret_cast<uint4*>(&sm.raw[(k + 1) & 1].x[tid][0]);
#pragma unroll
                for (int i = 0; i < CPB * (int)sizeof(T) / 16; ++i) dst[i] = src[i];
            }
        } else if (conv_out && tid < KC * CPB) {
            // conv state: the last KC inputs of the sequence, oldest first (zero rows
            // stand before the sequence start)
            const int q = tid / CPB, cc = tid % CPB;
            conv_out[((long long)b * di + c0 + cc) * KC + q] = to_f(r.x[nt - 1 + q][cc]);
        }
        __syncthreads();  // unpacked
        {
            // scan in groups of GS steps; the next group's operands load while the
            // current group's exp2s and FMAs run
            float* pw = sm.part + cl * PCS + p;
            float4 qd[2][GS], qb[2][GS];
#pragma unroll
            for (int u = 0; u < GS; ++u) {
                qd[0][u] = sm.dd[u][cl];
                qb[0][u] = sm.bc[u][p];
            }
#pragma unroll
            for (int g = 0; g < TC / GS; ++g) {
                const int cur = g & 1;
                if (g + 1 < TC / GS) {
#pragma unroll
                    for (int u = 0; u < GS; ++u) {
                        qd[cur ^ 1][u] = sm.dd[(g + 1) * GS + u][cl];
                        qb[cur ^ 1][u] = sm.bc[(g + 1) * GS + u][p];
                    }
                }
                float2 a[GS];
#pragma unroll
                for (int u = 0; u < GS; ++u) a[u] = exp2_pair(__fmul2_rn(make_float2(qd[cur][u].x, qd[cur][u].y), A2));
#pragma unroll
                for (int u = 0; u < GS; ++u) {
                    const float4 q = qb[cur][u];
                    h = __ffma2_rn(a[u], h, __fmul2_rn(make_float2(qd[cur][u].z, qd[cur][u].w), make_float2(q.x, q.y)));
                    const float2 ch = __fmul2_rn(make_float2(q.z, q.w), h);
                    pw[(g * GS + u) * TPC] = ch.x + ch.y;
                }
            }
        }
        __syncthreads();  // partial sums complete
        if (tid < nt) {
            const int t = tid;
            float y[CPB];
#pragma unroll
            for (int cc = 0; cc < CPB; ++cc) {
                const float4 a = *reinterpret_cast<const float4*>(sm.part + cc * PCS + t * TPC);
                const float4 e = *reinterpret_cast<const float4*>(sm.part + cc * PCS + t * TPC + 4);
                const float2 s = __fadd2_rn(__fadd2_rn(make_float2(a.x, a.y), make_float2(a.z, a.w)),
                                            __fadd2_rn(make_float2(e.x, e.y), make_float2(e.z, e.w)));
                y[cc] = (s.x + s.y) + sm.xd[t][cc];
            }
            T* dst = ypre + (row0 + t0 + t) * di + c0;
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
        float* dst = h_out + ((long long)b * di + c0 + cl) * 16 + 2 * p;
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
