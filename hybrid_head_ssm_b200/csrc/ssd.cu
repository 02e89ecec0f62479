// Mamba heads of the mixer in the SSD form, prefill, on the tensor cores ("Lecture 04 -
// Beyond the Dense Transformer", section 3: with A a scalar times the identity per SSM
// head, the selective scan equals a masked product with a semiseparable matrix and can
// be computed as blocks of matmuls). Per head h (P = 64 consecutive channels, scalar
// a = -exp(A_log[h]), Delta_t per head) and chunk of Q = 64 rows, with
// cs_i = a * (Delta_1 + .. + Delta_i) counted from the chunk start:
//     y_i = sum_{j<=i} exp(cs_i - cs_j) (C_i . B_j) Delta_j xc_j      (within the chunk)
//         + exp(cs_i) C_i . S                                          (earlier chunks)
//         + D xc_i
//     S  <- exp(cs_Q) S + sum_j exp(cs_Q - cs_j) Delta_j B_j xc_j^T    (state [N, P])
// which is the recurrence h_t = exp(Delta_t a) h_{t-1} + Delta_t B_t xc_t, y_t = C_t . h_t
// + D xc_t grouped by chunks. The conv + SiLU of x runs first in the same kernel.
//
// One CTA of 4 warps per (head, sequence) walks the chunks in order, carrying S (fp32, in
// the registers of the warps that own its columns). cp.async stages chunk k+1 (x with a
// three-row halo, B and C, the head's Delta) while chunk k is worked on:
//   phase 1: conv + SiLU -> xc and Delta xc as fp16 MMA operands; warp 0 forms the
//            cumulative decay cs (a warp scan, in log2 units) and the state weights;
//   phase 2: warp w owns rows 16w .. 16w+15: G = C B^T (m16n8k16 MMAs, fp32), masked and
//            scaled by exp2(cs_i - cs_j) in registers, reused as the A operand of
//            (L o G)(Delta xc) without a round trip through shared memory; the
//            earlier-chunk term as (exp(cs_i) C_i) S from the fp16 copy of S; + D xc;
//            the chunk's state update as one more MMA group into the fp32 state;
//   then the fp16 y rows leave through shared memory as 16-byte stores.
// The work is bound by the HBM traffic of x and y (4 bytes per row and channel); the
// tensor cores do about 330 flops per (row, channel).
#include "kernels.h"
#include "warp_mma.cuh"

namespace hymba {

namespace {

constexpr int SQ = 64;              // rows per chunk
constexpr int SP = 64;              // channels per SSM head
constexpr int SN = 16;              // states
constexpr int STH = 128;            // 4 warps
constexpr int SHALO = 3;
constexpr int SXR = SQ + SHALO;
constexpr int SLD = SP + 8;         // fp16 row stride of the operand tiles (144 bytes: ldmatrix conflict-free)
constexpr int SBC = 40;             // fp16 row stride of the staged B | C rows (80 bytes)
constexpr float SLOG2E = 1.4426950408889634f;

struct SsdSmem {
    alignas(16) f16 x[2][SXR][SP];      // pre-conv x of the head's channels, rows t0-3 ..
    alignas(16) f16 bc[2][SQ][SBC];     // B (0..15) | C (16..31) per row
    alignas(16) float dl[2][SQ];        // the head's Delta per row
    alignas(16) f16 xh[SQ][SLD];        // xc
    alignas(16) f16 dxh[SQ][SLD];       // Delta_j xc_j
    alignas(16) f16 yo[SQ][SLD];        // y rows on their way out
    alignas(16) f16 sh[SN][SLD];        // S of the earlier chunks, fp16
    alignas(16) float cs[SQ];           // cumulative decay (log2 units)
    alignas(16) float wj[SQ];           // state weights exp2(cs_Q - cs_j) Delta_j
    alignas(16) float Dv[SP];
};

using wm::cpa16;
using wm::cpa4;
using wm::cpa_commit;
using wm::cpa_wait0;
using wm::ldsm_x4;
using wm::ldsm_x4_t;
using wm::mma_f16;
using wm::pack_h2;

__device__ __forceinline__ uint32_t scale_h2(uint32_t v, float lo, float hi) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&v), __floats2half2_rn(lo, hi));
    return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_a(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// rows t0 .. t0+SQ-1 of sequence b (rows past Tp repeat the last one and are masked)
__device__ __forceinline__ void ssd_stage(SsdSmem& sm, int buf, int tid, const f16* P, long long ldP, int col_x,
                                          int col_B, const float* delta, int ld_delta, int h, int c0,
                                          long long row0, int t0, int Tp) {
    for (int j = tid; j < SXR * (SP / 8); j += STH) {
        const int rr = j / (SP / 8), k = j % (SP / 8);
        const int t = t0 - SHALO + rr;
        const long long row = row0 + min(max(t, 0), Tp - 1);
        cpa16(&sm.x[buf][rr][8 * k], P + row * ldP + col_x + c0 + 8 * k, t < 0);
    }
    for (int j = tid; j < SQ * 4; j += STH) {
        const int rr = j / 4, k = j % 4;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cpa16(&sm.bc[buf][rr][8 * k], P + row * ldP + col_B + 8 * k);
    }
    if (tid < SQ) {
        const long long row = row0 + min(t0 + tid, Tp - 1);
        cpa4(&sm.dl[buf][tid], delta + row * ld_delta + h);
    }
}

__global__ void __launch_bounds__(STH, 3)
ssd_scan_kernel(const f16* __restrict__ P, long long ldP, int col_x, int col_B, const float* __restrict__ delta,
                int ld_delta, const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                const float* __restrict__ A_log, const float* __restrict__ Dp, f16* __restrict__ ypre,
                float* __restrict__ h_out, float* __restrict__ conv_out, int Tp, int di) {
    griddep_sync();
    extern __shared__ __align__(16) uint8_t ssd_smem_raw[];
    SsdSmem& sm = *reinterpret_cast<SsdSmem*>(ssd_smem_raw);
    const int h = blockIdx.x, b = blockIdx.y, c0 = h * SP;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const long long row0 = (long long)b * Tp;
    const int nchunk = (Tp + SQ - 1) / SQ;

    ssd_stage(sm, 0, tid, P, ldP, col_x, col_B, delta, ld_delta, h, c0, row0, 0, Tp);
    cpa_commit();
    for (int j = tid; j < SN * SLD; j += STH) (&sm.sh[0][0])[j] = __float2half_rn(0.f);
    if (tid < SP) sm.Dv[tid] = Dp[c0 + tid];
    const float a2 = -expf(A_log[h]) * SLOG2E;  // a in log2 units
    // conv of channel cp over rows rh .. rh+31 of each chunk
    const int cp = tid & (SP - 1), rh = (tid / SP) * (SQ / 2);
    const float4 w4 = *reinterpret_cast<const float4*>(conv_w + (long long)(c0 + cp) * 4);
    const float cbias = conv_b[c0 + cp];
    // the state S[n][p] for p in this warp's columns 16 w + 8 t + 2 q (+1), n = g (+8)
    float st[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[t][e] = 0.f;

    for (int kc = 0; kc < nchunk; ++kc) {
        const int buf = kc & 1;
        const int t0 = kc * SQ, nt = min(SQ, Tp - t0);
        cpa_wait0();
        __syncthreads();  // chunk kc staged; chunk kc-1 fully consumed
        if (kc + 1 < nchunk)
            ssd_stage(sm, buf ^ 1, tid, P, ldP, col_x, col_B, delta, ld_delta, h, c0, row0, t0 + SQ, Tp);
        cpa_commit();

        // ---- phase 1 ----
        if (warp == 0) {
            // cs (inclusive prefix of a Delta, rows past nt hold Delta = 0) and the state weights
            const float d0 = 2 * lane < nt ? sm.dl[buf][2 * lane] : 0.f;
            const float d1 = 2 * lane + 1 < nt ? sm.dl[buf][2 * lane + 1] : 0.f;
            const float v0 = a2 * d0, v1 = a2 * d1;
            float s = v0 + v1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += u;
            }
            const float tot = __shfl_sync(0xffffffffu, s, 31);
            sm.cs[2 * lane] = s - v1;
            sm.cs[2 * lane + 1] = s;
            sm.wj[2 * lane] = ex2(tot - (s - v1)) * d0;
            sm.wj[2 * lane + 1] = ex2(tot - s) * d1;
        }
        {
            float x3 = __half2float(sm.x[buf][rh][cp]);
            float x2 = __half2float(sm.x[buf][rh + 1][cp]);
            float x1 = __half2float(sm.x[buf][rh + 2][cp]);
#pragma unroll 8
            for (int i = rh; i < rh + SQ / 2; ++i) {
                const float xt = __half2float(sm.x[buf][i + SHALO][cp]);
                const float u = fmaf(w4.w, xt, fmaf(w4.z, x1, fmaf(w4.y, x2, fmaf(w4.x, x3, cbias))));
                x3 = x2;
                x2 = x1;
                x1 = xt;
                const float xc = u * rcp_a(1.0f + ex2(-u * SLOG2E));
                const float dli = i < nt ? sm.dl[buf][i] : 0.f;
                sm.xh[i][cp] = __float2half_rn(xc);
                sm.dxh[i][cp] = __float2half_rn(dli * xc);
            }
        }
        __syncthreads();

        // ---- phase 2: rows 16 w .. 16 w + 15 ----
        const int r0 = 16 * warp;
        const float csg = sm.cs[r0 + g], csg8 = sm.cs[r0 + g + 8];
        const float csQ = sm.cs[SQ - 1];
        uint32_t cf[4];  // C rows as the A operand (k = state)
        ldsm_x4(cf, &sm.bc[buf][r0 + (lane & 15)][16 + 8 * (lane >> 4)]);
        float y[8][4];
#pragma unroll
        for (int pt = 0; pt < 8; ++pt)
#pragma unroll
            for (int e = 0; e < 4; ++e) y[pt][e] = 0.f;
        // within the chunk: k-steps kk <= warp over the keys j = 16 kk .. 16 kk + 15
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk <= warp) {
                uint32_t bq[4];  // B rows j as the "col" operand of two 8-key tiles
                ldsm_x4(bq, &sm.bc[buf][16 * kk + (lane & 7) + 8 * (lane >> 4)][8 * ((lane >> 3) & 1)]);
                float gl[2][4];
#pragma unroll
                for (int e = 0; e < 4; ++e) gl[0][e] = gl[1][e] = 0.f;
                mma_f16(gl[0], cf[0], cf[1], cf[2], cf[3], bq[0], bq[1]);
                mma_f16(gl[1], cf[0], cf[1], cf[2], cf[3], bq[2], bq[3]);
                // mask j <= i and scale by exp2(cs_i - cs_j)
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int j = 16 * kk + 8 * t + 2 * q;
                    const float csj0 = sm.cs[j], csj1 = sm.cs[j + 1];
                    const int i0 = r0 + g, i1 = r0 + g + 8;
                    gl[t][0] = j <= i0 ? gl[t][0] * ex2(csg - csj0) : 0.f;
                    gl[t][1] = j + 1 <= i0 ? gl[t][1] * ex2(csg - csj1) : 0.f;
                    gl[t][2] = j <= i1 ? gl[t][2] * ex2(csg8 - csj0) : 0.f;
                    gl[t][3] = j + 1 <= i1 ? gl[t][3] * ex2(csg8 - csj1) : 0.f;
                }
                const uint32_t a0 = pack_h2(gl[0][0], gl[0][1]), a1 = pack_h2(gl[0][2], gl[0][3]);
                const uint32_t a2r = pack_h2(gl[1][0], gl[1][1]), a3 = pack_h2(gl[1][2], gl[1][3]);
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    uint32_t bx[4];  // (Delta xc)[j][p] as the "col" operand of p-tiles 2 pp, 2 pp + 1
                    ldsm_x4_t(bx, &sm.dxh[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][16 * pp + 8 * (lane >> 4)]);
                    mma_f16(y[2 * pp], a0, a1, a2r, a3, bx[0], bx[1]);
                    mma_f16(y[2 * pp + 1], a0, a1, a2r, a3, bx[2], bx[3]);
                }
            }
        }
        // earlier chunks: (exp2(cs_i) C_i) . S
        {
            const float e0 = ex2(csg), e1 = ex2(csg8);
            const uint32_t s0 = scale_h2(cf[0], e0, e0), s1 = scale_h2(cf[1], e1, e1);
            const uint32_t s2 = scale_h2(cf[2], e0, e0), s3 = scale_h2(cf[3], e1, e1);
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                uint32_t bs[4];
                ldsm_x4_t(bs, &sm.sh[(lane & 7) + 8 * ((lane >> 3) & 1)][16 * pp + 8 * (lane >> 4)]);
                mma_f16(y[2 * pp], s0, s1, s2, s3, bs[0], bs[1]);
                mma_f16(y[2 * pp + 1], s0, s1, s2, s3, bs[2], bs[3]);
            }
        }
        // + D xc, to the output tile
#pragma unroll
        for (int pt = 0; pt < 8; ++pt) {
            const int p = 8 * pt + 2 * q;
            const float D0 = sm.Dv[p], D1 = sm.Dv[p + 1];
            const float2 xa = __half22float2(*reinterpret_cast<const __half2*>(&sm.xh[r0 + g][p]));
            const float2 xb = __half22float2(*reinterpret_cast<const __half2*>(&sm.xh[r0 + g + 8][p]));
            *reinterpret_cast<uint32_t*>(&sm.yo[r0 + g][p]) = pack_h2(fmaf(D0, xa.x, y[pt][0]), fmaf(D1, xa.y, y[pt][1]));
            *reinterpret_cast<uint32_t*>(&sm.yo[r0 + g + 8][p]) = pack_h2(fmaf(D0, xb.x, y[pt][2]), fmaf(D1, xb.y, y[pt][3]));
        }
        // state update of this warp's columns p = 16 w .. 16 w + 15:
        // S <- exp2(csQ) S + sum_j (exp2(csQ - cs_j) Delta_j B_j) xc_j^T
        {
            const float dec = ex2(csQ);
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) st[t][e] *= dec;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t wa[4];  // B^T (state x key) as the A operand
                ldsm_x4_t(wa, &sm.bc[buf][16 * kk + (lane & 7) + 8 * (lane >> 4)][8 * ((lane >> 3) & 1)]);
                const int j = 16 * kk + 2 * q;
                const float w0 = sm.wj[j], w1 = sm.wj[j + 1], w8 = sm.wj[j + 8], w9 = sm.wj[j + 9];
                wa[0] = scale_h2(wa[0], w0, w1);
                wa[1] = scale_h2(wa[1], w0, w1);
                wa[2] = scale_h2(wa[2], w8, w9);
                wa[3] = scale_h2(wa[3], w8, w9);
                uint32_t bx[4];
                ldsm_x4_t(bx, &sm.xh[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][16 * warp + 8 * (lane >> 4)]);
                mma_f16(st[0], wa[0], wa[1], wa[2], wa[3], bx[0], bx[1]);
                mma_f16(st[1], wa[0], wa[1], wa[2], wa[3], bx[2], bx[3]);
            }
        }
        __syncthreads();  // every warp has read S (fp16) and written its y rows
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int p = 16 * warp + 8 * t + 2 * q;
            *reinterpret_cast<uint32_t*>(&sm.sh[g][p]) = pack_h2(st[t][0], st[t][1]);
            *reinterpret_cast<uint32_t*>(&sm.sh[g + 8][p]) = pack_h2(st[t][2], st[t][3]);
        }
        for (int j = tid; j < SQ * (SP / 8); j += STH) {
            const int rr = j / (SP / 8), k = j % (SP / 8);
            if (rr < nt)
                *reinterpret_cast<uint4*>(ypre + (row0 + t0 + rr) * di + c0 + 8 * k) =
                    *reinterpret_cast<const uint4*>(&sm.yo[rr][8 * k]);
        }
    }
    if (conv_out && tid < SP) {
        const int tl = Tp - (nchunk - 1) * SQ + SHALO;  // staged index of row Tp
        const int lb = (nchunk - 1) & 1;
        *reinterpret_cast<float4*>(conv_out + ((long long)b * di + c0 + tid) * 4) =
            make_float4(__half2float(sm.x[lb][tl - 4][tid]), __half2float(sm.x[lb][tl - 3][tid]),
                        __half2float(sm.x[lb][tl - 2][tid]), __half2float(sm.x[lb][tl - 1][tid]));
    }
    if (h_out) {
        // h[c][n] of channel c = c0 + p
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int p = 16 * warp + 8 * t + 2 * q;
            float* hp0 = h_out + ((long long)b * di + c0 + p) * SN;
            float* hp1 = hp0 + SN;
            hp0[g] = st[t][0];
            hp1[g] = st[t][1];
            hp0[g + 8] = st[t][2];
            hp1[g + 8] = st[t][3];
        }
    }
}

}  // namespace

bool ssd_scan_applies(int di, int ssm_heads) { return ssm_heads > 0 && di == ssm_heads * SP; }

int launch_ssd_scan(const Ctx& ctx, const f16* P, long long ldP, int col_x, int col_B, const float* delta,
                    int ld_delta, const float* conv_w, const float* conv_b, const float* A_log, const float* D,
                    f16* ypre, float* h_out, float* conv_out, int B, int Tp, int di, int ssm_heads) {
    if (!ssd_scan_applies(di, ssm_heads) || col_x % 8 || col_B % 8 || ldP % 8 || ld_delta < ssm_heads || Tp <= 0 ||
        (reinterpret_cast<uintptr_t>(P) & 15) || (reinterpret_cast<uintptr_t>(ypre) & 15) || di % 8 ||
        (reinterpret_cast<uintptr_t>(conv_w) & 15) || (reinterpret_cast<uintptr_t>(delta) & 3) ||
        (conv_out && (reinterpret_cast<uintptr_t>(conv_out) & 15)))
        return HYMBA_ERR_UNSUPPORTED;
    dim3 grid(ssm_heads, B);
    const size_t smem = sizeof(SsdSmem);
    static std::atomic<unsigned long long> smem_set{0};
    if (!smem_opt_in_once(smem_set, ssd_scan_kernel, smem, ctx)) return HYMBA_ERR_CUDA;
    HYMBA_LAUNCH(ctx, "ssd_scan_prefill", ssd_scan_kernel, grid, STH, smem, P, ldP, col_x, col_B, delta, ld_delta,
                 conv_w, conv_b, A_log, D, ypre, h_out, conv_out, Tp, di);
    return HYMBA_OK;
}

}  // namespace hymba
