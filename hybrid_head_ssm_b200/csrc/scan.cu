// Mamba heads of the mixer, prefill: depthwise causal conv + SiLU, then the
// selective scan ("Jamba: Hybrid SSM-Transformer", How It Actually Works section 1;
// "Lecture 04", section 2):
//     h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) xc_t,   y_t = C_t . h_t + D xc_t
// with A = -exp(A_log) per (channel, state) and the state in fp32 registers.
//
// One block per (8-channel group, sequence), four warps in two roles:
//   scan warps (64 threads): thread (c, p) owns states 2p and 2p+1 of channel c and
//       updates both with packed f32x2 arithmetic (__ffma2_rn and friends), so a step is
//       two MUFU exp2 and four FMA-pipe instructions and the only serial dependency is
//       one FFMA2; each step's partial C.h sum goes to shared memory;
//   helper warps (64 threads, two per row): cp.async staging of the rows, conv + SiLU,
//       the scan's operands and the reduction y = sum of the 8 partial sums + D xc.
// The scan warps are bound by shared-memory bandwidth (a 16-byte load costs four
// wavefronts even when it is a broadcast), so the operands are packed for the fewest
// wavefronts per step: one 16-byte (Delta_t, Delta_t xc_t, Delta_t+1, Delta_t+1 xc_t+1)
// load serves two steps, and B_2p, B_2p+1, C_2p, C_2p+1 stay the fp16 values of the
// projection (one 8-byte load, converted in registers).
// Time is walked in chunks of 32 rows with one block barrier per chunk: while the scan
// warps scan chunk k, the helpers stage chunk k+2, reduce chunk k-1 and unpack chunk
// k+1, so the recurrence never waits for the preparation or the reduction. Raw rows are
// triple-buffered, operands and partial sums double-buffered. A chunk's x rows sit after
// three halo rows (the previous chunk's last three, zero before the sequence), so the
// causal conv needs no branches; shared-memory rows are padded against bank conflicts.
#include <type_traits>

#include "kernels.h"

namespace hymba {

namespace {

constexpr int CPB = 8;             // channels per block
constexpr int TPC = 8;             // scan threads per channel (2 states each)
constexpr int NSCAN = CPB * TPC;   // 64 scan threads
constexpr int NHELP = 64;          // helper threads
constexpr int NTH = NSCAN + NHELP;
constexpr int TC = 32;             // rows per chunk
constexpr int KC = 4;
constexpr int GS = 4;
constexpr int NRAW = 3;            // raw chunk buffers (stage k+2 while unpacking k+1)
constexpr int PCS = TC * TPC + 8;  // channel stride of the partial-sum buffer
constexpr float LOG2E = 1.4426950408889634f;
static_assert(NHELP == 2 * TC, "two helper threads per row");

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 exp2_pair(float2 a) { return make_float2(fast_exp2(a.x), fast_exp2(a.y)); }

template <typename T>
struct Raw {
    alignas(16) T x[TC + KC - 1][CPB];   // rows 0..2: the three rows before the chunk
    alignas(16) float d[TC][CPB];
    alignas(16) T b[TC][16];
    alignas(16) T c[TC][16];
};

// (B_2p, B_2p+1, C_2p, C_2p+1) of a row: fp16 inputs keep their four halves (8 bytes,
// converted in the scan), fp32 inputs four floats
template <typename T>
using BcEl = typename std::conditional<sizeof(T) == 2, uint2, float4>::type;

template <typename T>
struct Smem {
    Raw<T> raw[NRAW];
    alignas(16) float4 dd[2][TC / 2][CPB + 1];  // (d_t, dv_t, d_t+1, dv_t+1) per row pair
    alignas(16) BcEl<T> bc[2][TC][TPC + 1];
    alignas(16) float xd[2][TC][12];
    alignas(16) float part[2][CPB * PCS];
    alignas(16) float2 w2[KC + 2][CPB / 2];
};

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

// Helper thread h (0..63) queues its share of the copies of rows t0 .. t0+TC-1 (rows
// past Tp repeat the last row; their results are never stored and their Delta is
// zeroed when unpacked).
template <typename T>
__device__ __forceinline__ void stage_chunk(Raw<T>& r, int h, const T* P, long long ldP, int col_x, int col_B,
                                            int col_C, const float* delta, int di, int hp, int c0, long long row0,
                                            int t0, int Tp) {
    constexpr int XV = CPB * (int)sizeof(T) / 16;
    constexpr int DV = CPB * 4 / 16;
    constexpr int BV = 16 * (int)sizeof(T) / 16;
#pragma unroll
    for (int j = h; j < TC * XV; j += NHELP) {
        const int rr = j / XV, k = j % XV;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp_async16(reinterpret_cast<char*>(&r.x[rr + KC - 1][0]) + 16 * k,
                   reinterpret_cast<const char*>(P + row * ldP + col_x + c0) + 16 * k);
    }
    if (hp > 0) {
        // SSD form: one Delta per row for the block's head ([rows, di / hp])
        for (int j = h; j < TC; j += NHELP) {
            const long long row = row0 + min(t0 + j, Tp - 1);
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                             static_cast<uint32_t>(__cvta_generic_to_shared(&r.d[j][0]))),
                         "l"(delta + row * (di / hp) + c0 / hp)
                         : "memory");
        }
    } else {
#pragma unroll
        for (int j = h; j < TC * DV; j += NHELP) {
            const int rr = j / DV, k = j % DV;
            const long long row = row0 + min(t0 + rr, Tp - 1);
            cp_async16(reinterpret_cast<char*>(&r.d[rr][0]) + 16 * k,
                       reinterpret_cast<const char*>(delta + row * di + c0) + 16 * k);
        }
    }
#pragma unroll
    for (int j = h; j < TC * BV; j += NHELP) {
        const int rr = j / BV, k = j % BV;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp_async16(reinterpret_cast<char*>(&r.b[rr][0]) + 16 * k,
                   reinterpret_cast<const char*>(P + row * ldP + col_B) + 16 * k);
        cp_async16(reinterpret_cast<char*>(&r.c[rr][0]) + 16 * k,
                   reinterpret_cast<const char*>(P + row * ldP + col_C) + 16 * k);
    }
}

// Helper thread h: unpack row h >> 1 of the chunk in r, for channels (and state pairs)
// 4 * (h & 1) .. +3: conv + SiLU, the (Delta, Delta*xc) pairs, D xc and the B/C quads
// into operand buffer `buf`.
template <typename T>
__device__ __forceinline__ void unpack_chunk(Smem<T>& sm, const Raw<T>& r, int buf, int h, int nt, int hp) {
    const int t = h >> 1, hf = h & 1;
    float2 acc[2] = {sm.w2[KC][2 * hf], sm.w2[KC][2 * hf + 1]};
#pragma unroll
    for (int q = 0; q < KC; ++q) {
        float2 xv[CPB / 2];
        load8x2<T>(&r.x[t + q][0], xv);
#pragma unroll
        for (int j = 0; j < 2; ++j) acc[j] = __ffma2_rn(sm.w2[q][2 * hf + j], hf ? xv[2 + j] : xv[j], acc[j]);
    }
    const float4 dq = hp > 0 ? make_float4(r.d[t][0], r.d[t][0], r.d[t][0], r.d[t][0])
                             : *reinterpret_cast<const float4*>(&r.d[t][4 * hf]);
    const float keep = t < nt ? 1.f : 0.f;
    const float2 dl[2] = {make_float2(dq.x * keep, dq.y * keep), make_float2(dq.z * keep, dq.w * keep)};
    float2 xdv[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float2 e = exp2_pair(__fmul2_rn(acc[j], make_float2(-LOG2E, -LOG2E)));
        const float2 den = __fadd2_rn(e, make_float2(1.f, 1.f));
        const float2 xc = __fmul2_rn(acc[j], make_float2(rcp_approx(den.x), rcp_approx(den.y)));
        const float2 dv = __fmul2_rn(dl[j], xc);
        float2* d2 = reinterpret_cast<float2*>(&sm.dd[buf][t >> 1][0]) + (t & 1);
        d2[2 * (4 * hf + 2 * j)] = make_float2(dl[j].x, dv.x);
        d2[2 * (4 * hf + 2 * j + 1)] = make_float2(dl[j].y, dv.y);
        xdv[j] = __fmul2_rn(sm.w2[KC + 1][2 * hf + j], xc);
    }
    *reinterpret_cast<float4*>(&sm.xd[buf][t][4 * hf]) = make_float4(xdv[0].x, xdv[0].y, xdv[1].x, xdv[1].y);
    if constexpr (sizeof(T) == 2) {
        const uint4 bw = *reinterpret_cast<const uint4*>(&r.b[t][8 * hf]);
        const uint4 cw = *reinterpret_cast<const uint4*>(&r.c[t][8 * hf]);
        sm.bc[buf][t][4 * hf + 0] = make_uint2(bw.x, cw.x);
        sm.bc[buf][t][4 * hf + 1] = make_uint2(bw.y, cw.y);
        sm.bc[buf][t][4 * hf + 2] = make_uint2(bw.z, cw.z);
        sm.bc[buf][t][4 * hf + 3] = make_uint2(bw.w, cw.w);
    } else {
        float2 bv[4], cv[4];
        load8x2<T>(&r.b[t][8 * hf], bv);
        load8x2<T>(&r.c[t][8 * hf], cv);
#pragma unroll
        for (int q = 0; q < 4; ++q) sm.bc[buf][t][4 * hf + q] = make_float4(bv[q].x, bv[q].y, cv[q].x, cv[q].y);
    }
}

// Helper thread h: y of row h >> 1 for channels 4 * (h & 1) .. +3 = the 8 partial C.h
// sums + D xc.
template <typename T>
__device__ __forceinline__ void reduce_chunk(Smem<T>& sm, int buf, int h, int nt, T* ypre, long long row0, int t0,
                                             int di, int c0) {
    const int t = h >> 1, hf = h & 1;
    if (t >= nt) return;
    float y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int cc = 4 * hf + i;
        const float* pp = sm.part[buf] + cc * PCS + t * TPC;
        const float4 a = *reinterpret_cast<const float4*>(pp);
        const float4 e = *reinterpret_cast<const float4*>(pp + 4);
        const float2 s2 = __fadd2_rn(__fadd2_rn(make_float2(a.x, a.y), make_float2(a.z, a.w)),
                                     __fadd2_rn(make_float2(e.x, e.y), make_float2(e.z, e.w)));
        y[i] = (s2.x + s2.y) + sm.xd[buf][t][cc];
    }
    T* dst = ypre + (row0 + t0 + t) * di + c0 + 4 * hf;
    if constexpr (sizeof(T) == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(pack2<T>(y[0], y[1]), pack2<T>(y[2], y[3]));
    else *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[1], y[2], y[3]);
}

template <typename T>
__global__ void __launch_bounds__(NTH)
conv_scan_prefill_kernel(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C, const float* __restrict__ delta,
            const float* __restrict__ conv_w, const float* __restrict__ conv_b, const float* __restrict__ A_log,
            const float* __restrict__ Dp, T* __restrict__ ypre, float* __restrict__ h_out,
            float* __restrict__ conv_out, int Tp, int di, int hp) {
    griddep_sync();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem<T>& sm = *reinterpret_cast<Smem<T>*>(smem_raw);
    const int b = blockIdx.y, c0 = blockIdx.x * CPB;
    const int tid = threadIdx.x;
    const bool scanner = tid < NSCAN;
    const int h = tid - NSCAN;  // helper index
    const long long row0 = (long long)b * Tp;
    const int nchunk = (Tp + TC - 1) / TC;
    auto nt_of = [&](int k) { return min(TC, Tp - k * TC); };

    if (tid < (KC + 2) * (CPB / 2)) {
        const int q = tid / (CPB / 2), j = tid % (CPB / 2);
        const int ca = c0 + 2 * j, cb = ca + 1;
        float2 v;
        if (q < KC) v = make_float2(conv_w[(long long)ca * KC + q], conv_w[(long long)cb * KC + q]);
        else if (q == KC) v = make_float2(conv_b[ca], conv_b[cb]);
        else v = make_float2(Dp[ca], Dp[cb]);
        sm.w2[q][j] = v;
    }
    // prologue (helpers): stage chunks 0 and 1, zero halo of chunk 0
    if (!scanner) {
        if (h < (KC - 1) * CPB) sm.raw[0].x[h / CPB][h % CPB] = from_f<T>(0.f);
        stage_chunk<T>(sm.raw[0], h, P, ldP, col_x, col_B, col_C, delta, di, hp, c0, row0, 0, Tp);
        if (nchunk > 1) stage_chunk<T>(sm.raw[1], h, P, ldP, col_x, col_B, col_C, delta, di, hp, c0, row0, TC, Tp);
        cp_async_commit();
        cp_async_wait0();
    }
    __syncthreads();  // conv weights, chunks 0 and 1 visible
    if (!scanner) {
        if (nchunk > 1 && h < KC - 1) {
            const uint4* src = reinterpret_cast<const uint4*>(&sm.raw[0].x[TC + h][0]);
            uint4* dst = reinterpret_cast<uint4*>(&sm.raw[1].x[h][0]);
#pragma unroll
            for (int i = 0; i < CPB * (int)sizeof(T) / 16; ++i) dst[i] = src[i];
        }
        unpack_chunk<T>(sm, sm.raw[0], 0, h, nt_of(0), hp);
    }
    __syncthreads();  // chunk 0 unpacked, chunk 1's halo in place

    const int cl = tid / TPC, p = tid % TPC;
    float2 A2 = make_float2(0.f, 0.f), hs = make_float2(0.f, 0.f);
    if (scanner) {
        if (hp > 0) {  // SSD form: one A per head, for every state
            const float a = -expf(A_log[(c0 + cl) / hp]) * LOG2E;
            A2 = make_float2(a, a);
        } else {
            A2 = make_float2(-expf(A_log[(long long)(c0 + cl) * 16 + 2 * p]) * LOG2E,
                             -expf(A_log[(long long)(c0 + cl) * 16 + 2 * p + 1]) * LOG2E);
        }
    }
    for (int k = 0; k < nchunk; ++k) {
        const int buf = k & 1;
        if (scanner) {
            float* pw = sm.part[buf] + cl * PCS + p;
            float4 qd[2][GS / 2];
            BcEl<T> qb[2][GS];
#pragma unroll
            for (int u = 0; u < GS; ++u) qb[0][u] = sm.bc[buf][u][p];
#pragma unroll
            for (int u = 0; u < GS / 2; ++u) qd[0][u] = sm.dd[buf][u][cl];
#pragma unroll
            for (int g = 0; g < TC / GS; ++g) {
                const int cur = g & 1;
                if (g + 1 < TC / GS) {
#pragma unroll
                    for (int u = 0; u < GS; ++u) qb[cur ^ 1][u] = sm.bc[buf][(g + 1) * GS + u][p];
#pragma unroll
                    for (int u = 0; u < GS / 2; ++u) qd[cur ^ 1][u] = sm.dd[buf][(g + 1) * (GS / 2) + u][cl];
                }
                float dstep[GS], dvstep[GS];
#pragma unroll
                for (int u = 0; u < GS / 2; ++u) {
                    dstep[2 * u] = qd[cur][u].x;
                    dvstep[2 * u] = qd[cur][u].y;
                    dstep[2 * u + 1] = qd[cur][u].z;
                    dvstep[2 * u + 1] = qd[cur][u].w;
                }
                float2 a[GS];
#pragma unroll
                for (int u = 0; u < GS; ++u) a[u] = exp2_pair(__fmul2_rn(make_float2(dstep[u], dstep[u]), A2));
#pragma unroll
                for (int u = 0; u < GS; ++u) {
                    float2 Bq, Cq;
                    if constexpr (sizeof(T) == 2) {
                        Bq = __half22float2(*reinterpret_cast<const __half2*>(&qb[cur][u].x));
                        Cq = __half22float2(*reinterpret_cast<const __half2*>(&qb[cur][u].y));
                    } else {
                        Bq = make_float2(qb[cur][u].x, qb[cur][u].y);
                        Cq = make_float2(qb[cur][u].z, qb[cur][u].w);
                    }
                    hs = __ffma2_rn(a[u], hs, __fmul2_rn(make_float2(dvstep[u], dvstep[u]), Bq));
                    const float2 ch = __fmul2_rn(Cq, hs);
                    pw[(g * GS + u) * TPC] = ch.x + ch.y;
                }
            }
        } else {
            // stage k+2, halo of k+2, unpack k+1, reduce k-1
            if (k + 2 < nchunk)
                stage_chunk<T>(sm.raw[(k + 2) % NRAW], h, P, ldP, col_x, col_B, col_C, delta, di, hp, c0, row0,
                               (k + 2) * TC, Tp);
            cp_async_commit();
            if (k + 2 < nchunk && h < KC - 1) {
                const uint4* src = reinterpret_cast<const uint4*>(&sm.raw[(k + 1) % NRAW].x[TC + h][0]);
                uint4* dst = reinterpret_cast<uint4*>(&sm.raw[(k + 2) % NRAW].x[h][0]);
#pragma unroll
                for (int i = 0; i < CPB * (int)sizeof(T) / 16; ++i) dst[i] = src[i];
            }
            // reduce k-1 before unpacking k+1 into the same buffers (each helper reads and
            // then rewrites only its own row and channels of xd)
            if (k >= 1) reduce_chunk<T>(sm, buf ^ 1, h, nt_of(k - 1), ypre, row0, (k - 1) * TC, di, c0);
            if (k + 1 < nchunk) unpack_chunk<T>(sm, sm.raw[(k + 1) % NRAW], buf ^ 1, h, nt_of(k + 1), hp);
            if (k + 1 == nchunk && conv_out && h < KC * CPB) {
                // conv state: the last KC inputs of the sequence, oldest first
                const int q = h / CPB, cc = h % CPB;
                const int ntl = nt_of(k);
                conv_out[((long long)b * di + c0 + cc) * KC + q] = to_f(sm.raw[k % NRAW].x[ntl - 1 + q][cc]);
            }
            cp_async_wait0();
        }
        __syncthreads();
    }
    if (!scanner) reduce_chunk<T>(sm, (nchunk - 1) & 1, h, nt_of(nchunk - 1), ypre, row0, (nchunk - 1) * TC, di, c0);
    if (scanner && h_out) {
        float* dst = h_out + ((long long)b * di + c0 + cl) * 16 + 2 * p;
        dst[0] = hs.x;
        dst[1] = hs.y;
    }
}

}  // namespace

template <typename T>
int launch_conv_scan_prefill(const Ctx& ctx, const T* P, long long ldP, int col_x, int col_B, int col_C,
                             const float* delta, const float* conv_w, const float* conv_b, const float* A_log,
                             const float* D, T* ypre, float* h_out, float* conv_out, int B, int Tp, int di,
                             int hp) {
    if (di % CPB || (col_x % 8) || (col_B % 8) || (col_C % 8) || (ldP % 8) || hp < 0 ||
        (hp > 0 && (hp % CPB || di % hp)))
        return HYMBA_ERR_UNSUPPORTED;
    dim3 grid(di / CPB, B);
    const size_t smem = sizeof(Smem<T>);
    auto kern = conv_scan_prefill_kernel<T>;
    static std::atomic<unsigned long long> smem_set{0};
    if (!smem_opt_in_once(smem_set, kern, smem, ctx)) return HYMBA_ERR_CUDA;
    HYMBA_LAUNCH(ctx, "conv_scan_prefill", kern, grid, NTH, smem, P, ldP, col_x, col_B, col_C, delta, conv_w, conv_b,
                 A_log, D, ypre, h_out, conv_out, Tp, di, hp);
    return HYMBA_OK;
}

template int launch_conv_scan_prefill<float>(const Ctx&, const float*, long long, int, int, int, const float*,
                                             const float*, const float*, const float*, const float*, float*, float*,
                                             float*, int, int, int, int);
template int launch_conv_scan_prefill<f16>(const Ctx&, const f16*, long long, int, int, int, const float*,
                                           const float*, const float*, const float*, const float*, f16*, float*,
                                           float*, int, int, int, int);

}  // namespace hymba
