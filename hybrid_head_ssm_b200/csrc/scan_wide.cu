// Mamba heads of the mixer, prefill, for batches with many (sequence, channel) pairs:
// depthwise causal conv + SiLU, Delta = softplus(dt_low W_dt^T + b_dt), and the selective
// scan ("Jamba: Hybrid SSM-Transformer", How It Actually Works section 1; "Lecture 04",
// section 2):
//     h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) xc_t,   y_t = C_t . h_t + D xc_t
// with A = -exp(A_log) per (channel, state), the state in fp32 registers.
//
// The work per (row, channel) is set by the method: 16 exponentials of the state decays
// on the 16-per-clock MUFU unit (plus the SiLU's and the softplus's) and about 48 fp32
// instructions around them. Everything that does not depend on the state is done for a
// whole chunk of rows in parallel before the recurrence runs, so the recurrence issues
// little besides its own arithmetic.
//
// One block of 128 threads per (64-channel group, sequence). Rows are walked in chunks of
// 32; cp.async stages chunk k+1 (x with a three-row halo, dt_low, B, C) while chunk k is
// worked on in three phases separated by block barriers:
//   A1: Delta of the chunk from warp-level tensor-core MMAs (m16n8k16, fp16 dt_low rows x
//       the W_dt rows of the warp's 16 channels, which stay in registers, fp32
//       accumulate) plus a branch-free softplus, stored in conflict-free 8-byte pairs;
//       B and C converted to fp32;
//   A2: conv + SiLU of every (row, channel), two adjacent channels per thread as fp32
//       pairs (FFMA2), stored with Delta as the pairs (Delta, Delta xc) the recurrence
//       consumes, and D xc;
//   B:  the recurrence. Thread (channel c, half s) holds states 8s .. 8s+7 of c as four
//       fp32 pairs: per row one 8-byte load of (Delta, Delta xc), B_t and C_t of its half
//       as fp32 quads shared by the warp, four (FMUL2, 2 ex2, FMUL2, FFMA2, FFMA2) groups,
//       and the next row's decays computed ahead so the exponentials overlap the FMA
//       chain; the halves add their partial C.h with one shuffle and both store y.
// Two threads per channel keep enough warps per SM to hide the latencies; this kernel is
// used when B * d_inner fills the GPU. Smaller batches use the kernel that splits a
// channel's states over 8 threads (scan.cu).
#include "kernels.h"

namespace hymba {

namespace {

constexpr int WCH = 64;            // channels per block
constexpr int WTH = 128;           // threads per block: 64 channels x 2 state halves
constexpr int WTC = 32;            // rows per chunk
constexpr int WHALO = 3;           // conv history rows staged before each chunk
constexpr int WXR = WTC + WHALO;   // staged x rows per chunk
constexpr int WRMAX = 128;         // dt_rank <= WRMAX
constexpr int WKS = WRMAX / 16;    // MMA k-steps at most
constexpr int WDLD = WRMAX + 8;    // staged dt_low row stride (fp16): conflict-free ldmatrix rows
constexpr int WDD = WCH + 8;       // Delta row stride (fp32): conflict-free 8-byte stores of the MMA pairs
constexpr float WLOG2E = 1.4426950408889634f;

struct WideSmem {
    alignas(16) f16 x[2][WXR][WCH];        // pre-conv inputs of the block's channels, rows t0-3 ..
    alignas(16) f16 dtl[2][WTC][WDLD];     // dt_low rows
    alignas(16) f16 bc[2][WTC][32];        // B (16) then C (16) of each row, as staged
    alignas(16) float bcf[WTC][32];        // the same in fp32, current chunk
    alignas(16) float dlt[WTC][WDD];       // Delta of the current chunk
    alignas(16) float2 dd[WTC][WCH];       // (Delta, Delta xc)
    alignas(16) float dx[WTC][WCH];        // D xc
};

__device__ __forceinline__ void cp16(void* dst, const void* src, bool zero = false) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src), "r"(zero ? 0 : 16)
                 : "memory");
}
__device__ __forceinline__ void cp8(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ float rcp_fast(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_fast(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// softplus of a pair (two adjacent channels), the arithmetic on fp32 pairs:
// softplus(u) = max(u, 0) + log(1 + e), e = exp(-|u|), branch-free: the series
// e - e^2/2 + e^3/3 where 1 + e would drop e's low bits (e < 2^-10), the MUFU log2 above.
__device__ __forceinline__ float2 softplus_bf2(float2 u) {
    const float2 na = __fmul2_rn(make_float2(fabsf(u.x), fabsf(u.y)), make_float2(-WLOG2E, -WLOG2E));
    const float2 e = make_float2(fast_exp2(na.x), fast_exp2(na.y));
    // e (1 - e (1/2 - e / 3)) = e (1 + e (e / 3 - 1/2))
    const float2 a = __ffma2_rn(e, make_float2(1.0f / 3.0f, 1.0f / 3.0f), make_float2(-0.5f, -0.5f));
    const float2 series = __fmul2_rn(e, __ffma2_rn(e, a, make_float2(1.f, 1.f)));
    const float2 ope = __fadd2_rn(e, make_float2(1.f, 1.f));
    const float2 lg = __fmul2_rn(make_float2(lg2_fast(ope.x), lg2_fast(ope.y)),
                                 make_float2(0.69314718055994531f, 0.69314718055994531f));
    return __fadd2_rn(make_float2(fmaxf(u.x, 0.0f), fmaxf(u.y, 0.0f)),
                      make_float2(e.x < 9.765625e-4f ? series.x : lg.x, e.y < 9.765625e-4f ? series.y : lg.y));
}

// The dt_low pieces (r_dt / 4 per row) a thread copies: j = tid, tid + WTH, ... as (row,
// piece), the first one and the step, so that each chunk's copies need no division.
struct DtPieces {
    int pieces, rr0, k0, drr, dk;
    __device__ void init(int tid, int r_dt) {
        pieces = r_dt / 4;
        rr0 = tid / pieces;
        k0 = tid - rr0 * pieces;
        drr = WTH / pieces;
        dk = WTH - drr * pieces;
    }
};

// Stage rows t0 .. t0+WTC-1 of sequence b into buffer buf: x of the block's channels with
// the WHALO rows before t0 (zeros before the first row), dt_low (r_dt values in 8-byte
// pieces), B and C. Rows past Tp repeat the last one; they are never scanned.
__device__ __forceinline__ void stage(WideSmem& sm, int buf, int tid, const f16* P, long long ldP, int col_x,
                                     int col_B, int col_dt, const DtPieces& dp, int c0, long long row0, int t0,
                                     int Tp) {
    for (int j = tid; j < WXR * (WCH / 8); j += WTH) {
        const int rr = j / (WCH / 8), k = j % (WCH / 8);
        const int t = t0 - WHALO + rr;
        const long long row = row0 + min(max(t, 0), Tp - 1);
        cp16(&sm.x[buf][rr][8 * k], P + row * ldP + col_x + c0 + 8 * k, t < 0);
    }
    {
        const int rr = tid / 4, k = tid % 4;  // B and C: 32 fp16 = 4 pieces of 16 bytes per row
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp16(&sm.bc[buf][rr][8 * k], P + row * ldP + col_B + 8 * k);
    }
    for (int rr = dp.rr0, k = dp.k0; rr < WTC;) {
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp8(&sm.dtl[buf][rr][4 * k], P + row * ldP + col_dt + 4 * k);
        rr += dp.drr;
        k += dp.dk;
        if (k >= dp.pieces) {
            k -= dp.pieces;
            ++rr;
        }
    }
}

__global__ void __launch_bounds__(WTH, 3)
conv_scan_wide_kernel(const f16* __restrict__ P, long long ldP, int col_x, int col_B, int col_dt, int r_dt,
                      const f16* __restrict__ wdt, int ld_wdt, const float* __restrict__ b_dt,
                      const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                      const float* __restrict__ A_log, const float* __restrict__ Dp, f16* __restrict__ ypre,
                      float* __restrict__ h_out, float* __restrict__ conv_out, int Tp, int di) {
    griddep_sync();
    extern __shared__ __align__(16) uint8_t wsmem[];
    WideSmem& sm = *reinterpret_cast<WideSmem*>(wsmem);
    const int b = blockIdx.y, c0 = blockIdx.x * WCH;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long row0 = (long long)b * Tp;
    const int nchunk = (Tp + WTC - 1) / WTC;
    const int ks = (r_dt + 15) / 16;

    // zero tails of the dt_low buffers (columns the copies never write, read by the MMAs)
    for (int j = tid; j < 2 * WTC * (WDLD - r_dt); j += WTH) {
        const int bsel = j / (WTC * (WDLD - r_dt)), rem = j - bsel * WTC * (WDLD - r_dt);
        sm.dtl[bsel][rem / (WDLD - r_dt)][r_dt + rem % (WDLD - r_dt)] = __float2half_rn(0.f);
    }
    DtPieces dp;
    dp.init(tid, r_dt);
    stage(sm, 0, tid, P, ldP, col_x, col_B, col_dt, dp, c0, row0, 0, Tp);
    cp_commit();

    // A1 constants: this lane's B fragments of the warp's 16 channels (n-tiles j = 0, 1;
    // W_dt is zero-padded to 16 ks columns) and the bias of its output columns
    // 8 j + 2 (lane % 4), +1
    const int g = lane >> 2, q = lane & 3;
    uint32_t bfr[WKS][2][2];
#pragma unroll
    for (int st = 0; st < WKS; ++st)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            bfr[st][j][0] = bfr[st][j][1] = 0u;
            if (st < ks) {
                const f16* wr = wdt + (long long)(c0 + warp * 16 + 8 * j + g) * ld_wdt + 16 * st + 2 * q;
                bfr[st][j][0] = *reinterpret_cast<const uint32_t*>(wr);
                bfr[st][j][1] = *reinterpret_cast<const uint32_t*>(wr + 8);
            }
        }
    float2 bdt[2];
#pragma unroll
    for (int j = 0; j < 2; ++j)
        bdt[j] = *reinterpret_cast<const float2*>(b_dt + c0 + warp * 16 + 8 * j + 2 * q);
    // A2: conv of channels 2 cp, 2 cp + 1 over rows rh .. rh+7 of each chunk
    constexpr int A2R = WTC / (WTH / (WCH / 2));  // rows per thread: 8
    const int cp = tid & (WCH / 2 - 1), rh = (tid / (WCH / 2)) * A2R;
    float2 w2[4];  // tap k of the two channels
    {
        const float4 wa = *reinterpret_cast<const float4*>(conv_w + (long long)(c0 + 2 * cp) * 4);
        const float4 wb = *reinterpret_cast<const float4*>(conv_w + (long long)(c0 + 2 * cp + 1) * 4);
        w2[0] = make_float2(wa.x, wb.x);
        w2[1] = make_float2(wa.y, wb.y);
        w2[2] = make_float2(wa.z, wb.z);
        w2[3] = make_float2(wa.w, wb.w);
    }
    const float2 cb2 = *reinterpret_cast<const float2*>(conv_b + c0 + 2 * cp);
    const float2 D2 = *reinterpret_cast<const float2*>(Dp + c0 + 2 * cp);

    // B: channel cl of the block, states 8 s .. 8 s + 7 as pairs
    const int cl = warp * 16 + (lane >> 1), s = lane & 1;
    float2 A2[4], h[4];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float4 a4 = *reinterpret_cast<const float4*>(A_log + (long long)(c0 + cl) * 16 + 8 * s + 4 * k);
        A2[2 * k] = make_float2(-expf(a4.x) * WLOG2E, -expf(a4.y) * WLOG2E);
        A2[2 * k + 1] = make_float2(-expf(a4.z) * WLOG2E, -expf(a4.w) * WLOG2E);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) h[k] = make_float2(0.f, 0.f);

    for (int kc = 0; kc < nchunk; ++kc) {
        const int buf = kc & 1;
        cp_wait0();
        __syncthreads();  // chunk kc staged; everyone is past chunk kc-1's phase B
        if (kc + 1 < nchunk) stage(sm, buf ^ 1, tid, P, ldP, col_x, col_B, col_dt, dp, c0, row0, (kc + 1) * WTC, Tp);
        cp_commit();

        // ---- A1: Delta (rows 16 i + g (+8), channels warp*16 + 8 j + 2 q (+1)), B/C to fp32 ----
        {
            float acc[2][2][4];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
#pragma unroll
            for (int st = 0; st < WKS; ++st) {
                if (st < ks) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        uint32_t a[4];
                        ldmatrix_x4(a, &sm.dtl[buf][16 * i + (lane & 15)][16 * st + 8 * (lane >> 4)]);
#pragma unroll
                        for (int j = 0; j < 2; ++j) mma16816(acc[i][j], a, bfr[st][j][0], bfr[st][j][1]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int col = warp * 16 + 8 * j + 2 * q;
                    *reinterpret_cast<float2*>(&sm.dlt[16 * i + g][col]) =
                        softplus_bf2(__fadd2_rn(make_float2(acc[i][j][0], acc[i][j][1]), bdt[j]));
                    *reinterpret_cast<float2*>(&sm.dlt[16 * i + g + 8][col]) =
                        softplus_bf2(__fadd2_rn(make_float2(acc[i][j][2], acc[i][j][3]), bdt[j]));
                }
        }
#pragma unroll
        for (int j = tid; j < WTC * 32; j += WTH) sm.bcf[j / 32][j % 32] = __half2float(sm.bc[buf][j / 32][j % 32]);
        __syncthreads();

        // ---- A2: conv + SiLU of channels 2 cp, 2 cp + 1, rows rh .. rh+7 (x row t sits at
        // staged row t + WHALO) ----
        {
            const float2 nl2 = make_float2(-WLOG2E, -WLOG2E), one2 = make_float2(1.f, 1.f);
            auto xpair = [&](int row) {
                return __half22float2(*reinterpret_cast<const __half2*>(&sm.x[buf][row][2 * cp]));
            };
            float2 x3 = xpair(rh), x2 = xpair(rh + 1), x1 = xpair(rh + 2);
#pragma unroll
            for (int t = rh; t < rh + A2R; ++t) {
                const float2 xt = xpair(t + WHALO);
                float2 u = __ffma2_rn(w2[0], x3, cb2);
                u = __ffma2_rn(w2[1], x2, u);
                u = __ffma2_rn(w2[2], x1, u);
                u = __ffma2_rn(w2[3], xt, u);
                x3 = x2;
                x2 = x1;
                x1 = xt;
                const float2 ne = __fmul2_rn(u, nl2);
                const float2 den = __fadd2_rn(make_float2(fast_exp2(ne.x), fast_exp2(ne.y)), one2);
                const float2 xc = __fmul2_rn(u, make_float2(rcp_fast(den.x), rcp_fast(den.y)));
                const float2 d = *reinterpret_cast<const float2*>(&sm.dlt[t][2 * cp]);
                const float2 dxc = __fmul2_rn(d, xc);
                *reinterpret_cast<float4*>(&sm.dd[t][2 * cp]) = make_float4(d.x, dxc.x, d.y, dxc.y);
                *reinterpret_cast<float2*>(&sm.dx[t][2 * cp]) = __fmul2_rn(D2, xc);
            }
        }
        __syncthreads();

        // ---- B: the recurrence ----
        const int nt = min(WTC, Tp - kc * WTC);
        f16* yrow = ypre + (row0 + (long long)kc * WTC) * di + c0 + cl;
        const float2* ddc = &sm.dd[0][cl];
        const float* bcs = &sm.bcf[0][8 * s];
        const float* dxc = &sm.dx[0][cl];
        float2 dv = ddc[0];
        float2 a[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 ad = __fmul2_rn(make_float2(dv.x, dv.x), A2[k]);
            a[k] = make_float2(fast_exp2(ad.x), fast_exp2(ad.y));
        }
        auto step = [&](int t) {
            // the next row's decays first: they depend only on its Delta
            const float2 dn = ddc[min(t + 1, WTC - 1) * WCH];
            float2 an[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 ad = __fmul2_rn(make_float2(dn.x, dn.x), A2[k]);
                an[k] = make_float2(fast_exp2(ad.x), fast_exp2(ad.y));
            }
            const float4* bq = reinterpret_cast<const float4*>(bcs + t * 32);
            const float4 b0 = bq[0], b1 = bq[1], q0 = bq[4], q1 = bq[5];
            const float2 xx = make_float2(dv.y, dv.y);
            h[0] = __ffma2_rn(a[0], h[0], __fmul2_rn(xx, make_float2(b0.x, b0.y)));
            h[1] = __ffma2_rn(a[1], h[1], __fmul2_rn(xx, make_float2(b0.z, b0.w)));
            h[2] = __ffma2_rn(a[2], h[2], __fmul2_rn(xx, make_float2(b1.x, b1.y)));
            h[3] = __ffma2_rn(a[3], h[3], __fmul2_rn(xx, make_float2(b1.z, b1.w)));
            float2 y0 = __fmul2_rn(make_float2(q0.x, q0.y), h[0]);
            float2 y1 = __fmul2_rn(make_float2(q0.z, q0.w), h[1]);
            y0 = __ffma2_rn(make_float2(q1.x, q1.y), h[2], y0);
            y1 = __ffma2_rn(make_float2(q1.z, q1.w), h[3], y1);
            const float2 y2 = __fadd2_rn(y0, y1);
            float ys = y2.x + y2.y;
            ys += __shfl_xor_sync(0xffffffffu, ys, 1);  // the other half's states
            // both halves hold y and store the same value (no divergent branch per row)
            yrow[(long long)t * di] = __float2half_rn(ys + dxc[t * WCH]);
#pragma unroll
            for (int k = 0; k < 4; ++k) a[k] = an[k];
            dv = dn;
        };
        if (nt == WTC) {
            // fully unrolled: every shared-memory address is the base plus a constant
#pragma unroll
            for (int t = 0; t < WTC; ++t) step(t);
        } else {
            for (int t = 0; t < nt; ++t) step(t);
        }
    }
    if (conv_out && tid < WCH) {
        // conv state: the last four inputs of the sequence, oldest first (staged rows of
        // the last chunk; the halo holds zeros before the first row)
        const int tl = Tp - (nchunk - 1) * WTC + WHALO;  // staged index of row Tp
        const int lb = (nchunk - 1) & 1;
        *reinterpret_cast<float4*>(conv_out + ((long long)b * di + c0 + tid) * 4) =
            make_float4(__half2float(sm.x[lb][tl - 4][tid]), __half2float(sm.x[lb][tl - 3][tid]),
                        __half2float(sm.x[lb][tl - 2][tid]), __half2float(sm.x[lb][tl - 1][tid]));
    }
    if (h_out) {
        float* hp = h_out + ((long long)b * di + c0 + cl) * 16 + 8 * s;
#pragma unroll
        for (int k = 0; k < 4; ++k) *reinterpret_cast<float2*>(hp + 2 * k) = h[k];
    }
}

}  // namespace

bool scan_wide_applies(int B, int di, int dt_rank, int sm_count) {
    // two threads per channel: the GPU needs a few blocks of 128 per SM
    return di % WCH == 0 && dt_rank > 0 && dt_rank <= WRMAX && dt_rank % 4 == 0 &&
           (long long)B * (di / WCH) >= 2LL * sm_count;
}

int launch_conv_scan_wide(const Ctx& ctx, const f16* P, long long ldP, int col_x, int col_B, int col_dt, int dt_rank,
                          const f16* wdt, int ld_wdt, const float* b_dt, const float* conv_w, const float* conv_b,
                          const float* A_log, const float* D, f16* ypre, float* h_out, float* conv_out, int B, int Tp,
                          int di) {
    if (di % WCH || dt_rank <= 0 || dt_rank > WRMAX || dt_rank % 4 || col_x % 8 || col_B % 8 || col_dt % 4 ||
        ldP % 8 || ld_wdt % 8 || ld_wdt < 16 * ((dt_rank + 15) / 16) || Tp <= 0 ||
        (reinterpret_cast<uintptr_t>(P) & 15) || (reinterpret_cast<uintptr_t>(wdt) & 15) ||
        (reinterpret_cast<uintptr_t>(b_dt) & 7) || (reinterpret_cast<uintptr_t>(conv_w) & 15) ||
        (reinterpret_cast<uintptr_t>(A_log) & 15) || (h_out && (reinterpret_cast<uintptr_t>(h_out) & 7)) ||
        (conv_out && (reinterpret_cast<uintptr_t>(conv_out) & 15)))
        return HYMBA_ERR_UNSUPPORTED;
    dim3 grid(di / WCH, B);
    const size_t smem = sizeof(WideSmem);
    static std::atomic<unsigned long long> smem_set{0};
    if (!smem_opt_in_once(smem_set, conv_scan_wide_kernel, smem, ctx)) return HYMBA_ERR_CUDA;
    HYMBA_LAUNCH(ctx, "conv_scan_prefill", conv_scan_wide_kernel, grid, WTH, smem, P, ldP, col_x, col_B, col_dt,
                 dt_rank, wdt, ld_wdt, b_dt, conv_w, conv_b, A_log, D, ypre, h_out, conv_out, Tp, di);
    return HYMBA_OK;
}

}  // namespace hymba
