// Mamba heads of the mixer, prefill, for batches with many (sequence, channel) pairs:
// depthwise causal conv + SiLU, Delta = softplus(dt_low W_dt^T + b_dt), and the selective
// scan ("Jamba: Hybrid SSM-Transformer", How It Actually Works section 1; "Lecture 04",
// section 2):
//     h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) xc_t,   y_t = C_t . h_t + D xc_t
// with A = -exp(A_log) per (channel, state), the state in fp32 registers.
//
// One block of 64 threads per (64-channel group, sequence); thread (pair p, half s) of a
// warp holds states 8s .. 8s+7 of the two channels 2p, 2p+1 as fp32 pairs, so one step is
// 8 packed (FMUL2, FMUL2, FFMA2, FFMA2) groups and 16 exp2 for 16 (row, channel, state)
// updates. B_t and C_t are the same for every channel: a thread reads only its half (two
// 16-byte loads of fp16 values per step) and each value serves two channels. Half s runs
// the conv and SiLU of channel 2p+s (the last three inputs stay in registers, so the
// conv needs no halo), the two halves swap xc and add their partial C.h sums with one
// shuffle each, and half s stores y of channel 2p+s (a warp writes 32 consecutive
// channels). Delta of a 32-row chunk comes from warp-level tensor-core MMAs (m16n8k16,
// fp16 in, fp32 out) of the staged dt_low rows against the block's W_dt rows, each warp
// computing its own 32 channels; no Delta tensor goes through memory.
// Rows are walked in chunks of 32: cp.async stages chunk k+1 (x, dt_low, B, C) while
// chunk k is scanned; one block barrier per chunk.
// Parallelism is one thread per channel of every sequence, so this kernel is used when
// B * d_inner is large enough to fill the GPU; smaller batches use the kernel that splits
// a channel's states over 8 threads (scan.cu).
#include "kernels.h"

namespace hymba {

namespace {

constexpr int WCH = 64;            // channels per block
constexpr int WTH = 64;            // threads per block: 32 channel pairs x 2 state halves
constexpr int WTC = 32;            // rows per chunk
constexpr int WRMAX = 128;         // dt_rank <= WRMAX
constexpr int WDLD = WRMAX + 8;    // staged dt_low / W_dt row stride (fp16): conflict-free fragments
constexpr int WDD = WCH + 4;       // Delta row stride (fp32)
constexpr float WLOG2E = 1.4426950408889634f;

struct WideSmem {
    alignas(16) f16 x[2][WTC][WCH];        // pre-conv inputs of the block's channels
    alignas(16) f16 dtl[2][WTC][WDLD];     // dt_low rows
    alignas(16) f16 bc[2][WTC][32];        // B (16) then C (16) of each row
    alignas(16) float dlt[WTC][WDD];       // Delta of the current chunk
    alignas(16) f16 w[WCH][WDLD];          // the block's W_dt rows (fp16, zero-padded)
};

__device__ __forceinline__ void cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
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
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Stage rows t0 .. t0+WTC-1 of sequence b (rows past Tp repeat the last one; they are
// never scanned): x of the block's channels, dt_low (r_dt values in 8-byte pieces), B, C.
__device__ __forceinline__ void stage(WideSmem& sm, int buf, int tid, const f16* P, long long ldP, int col_x,
                                     int col_B, int col_dt, int r_dt, int c0, long long row0, int t0, int Tp) {
    for (int j = tid; j < WTC * (WCH / 8); j += WTH) {
        const int rr = j / (WCH / 8), k = j % (WCH / 8);
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp16(&sm.x[buf][rr][8 * k], P + row * ldP + col_x + c0 + 8 * k);
    }
    for (int j = tid; j < WTC * 4; j += WTH) {  // B and C: 32 fp16 = 4 pieces of 16 bytes
        const int rr = j / 4, k = j % 4;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp16(&sm.bc[buf][rr][8 * k], P + row * ldP + col_B + 8 * k);
    }
    const int pieces = r_dt / 4;
    for (int j = tid; j < WTC * pieces; j += WTH) {
        const int rr = j / pieces, k = j - rr * pieces;
        const long long row = row0 + min(t0 + rr, Tp - 1);
        cp8(&sm.dtl[buf][rr][4 * k], P + row * ldP + col_dt + 4 * k);
    }
}

__global__ void __launch_bounds__(WTH)
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
    const int p = lane >> 1, s = lane & 1;          // channel pair of the warp, state half
    const int cl = warp * 32 + 2 * p;                // first channel of the pair (block-local)
    const int cs = cl + s;                           // the channel whose conv this thread runs
    const long long row0 = (long long)b * Tp;
    const int nchunk = (Tp + WTC - 1) / WTC;
    const int ks = (r_dt + 15) / 16;

    // W_dt rows of the block (zero-padded to a multiple of 16 columns) and zero tails of
    // the dt_low buffers (columns the copies never write, read by the last MMA)
    for (int j = tid; j < WCH * (WDLD / 8); j += WTH) {
        const int rr = j / (WDLD / 8), k = j % (WDLD / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (8 * k < ld_wdt) v = *reinterpret_cast<const uint4*>(wdt + (long long)(c0 + rr) * ld_wdt + 8 * k);
        *reinterpret_cast<uint4*>(&sm.w[rr][8 * k]) = v;
    }
    for (int j = tid; j < 2 * WTC * (WDLD - r_dt); j += WTH) {
        const int bsel = j / (WTC * (WDLD - r_dt)), rem = j - bsel * WTC * (WDLD - r_dt);
        sm.dtl[bsel][rem / (WDLD - r_dt)][r_dt + rem % (WDLD - r_dt)] = __float2half_rn(0.f);
    }
    stage(sm, 0, tid, P, ldP, col_x, col_B, col_dt, r_dt, c0, row0, 0, Tp);
    cp_commit();

    // per-thread constants: A of the pair's states (as exp2 factors), conv taps of channel cs
    float2 A2[8];
#pragma unroll
    for (int n = 0; n < 8; ++n)
        A2[n] = make_float2(-expf(A_log[(long long)(c0 + cl) * 16 + 8 * s + n]) * WLOG2E,
                            -expf(A_log[(long long)(c0 + cl + 1) * 16 + 8 * s + n]) * WLOG2E);
    const float4 w4 = *reinterpret_cast<const float4*>(conv_w + (long long)(c0 + cs) * 4);
    const float cb = conv_b[c0 + cs], Dc = Dp[c0 + cs];
    // this lane's output columns of the Delta MMAs: channels 8 j + 2 (lane % 4), +1 of
    // the warp's 32, for n-tiles j = 0..3
    float2 bdt[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        bdt[j] = make_float2(b_dt[c0 + warp * 32 + 8 * j + 2 * (lane & 3)],
                             b_dt[c0 + warp * 32 + 8 * j + 2 * (lane & 3) + 1]);
    float2 h[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) h[n] = make_float2(0.f, 0.f);
    float x1 = 0.f, x2 = 0.f, x3 = 0.f, x4 = 0.f;  // x_{t-1} .. x_{t-4} of channel cs

    for (int k = 0; k < nchunk; ++k) {
        const int buf = k & 1;
        cp_wait0();
        __syncthreads();  // chunk k staged; everyone is past chunk k-1
        if (k + 1 < nchunk) stage(sm, buf ^ 1, tid, P, ldP, col_x, col_B, col_dt, r_dt, c0, row0, (k + 1) * WTC, Tp);
        cp_commit();
        // Delta of the chunk for this warp's 32 channels: rows 16 i + g (+8), channels
        // 8 j + 2 q (+1) of the warp, i = 0..1, j = 0..3
        {
            const int g = lane >> 2, q = lane & 3;
            float acc[2][4][4];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
#pragma unroll
            for (int st = 0; st < WRMAX / 16; ++st) {
                if (st < ks) {
                    uint32_t a[2][4];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const f16* r0 = sm.dtl[buf][16 * i + g];
                        const f16* r1 = sm.dtl[buf][16 * i + g + 8];
                        a[i][0] = *reinterpret_cast<const uint32_t*>(r0 + 16 * st + 2 * q);
                        a[i][1] = *reinterpret_cast<const uint32_t*>(r1 + 16 * st + 2 * q);
                        a[i][2] = *reinterpret_cast<const uint32_t*>(r0 + 16 * st + 8 + 2 * q);
                        a[i][3] = *reinterpret_cast<const uint32_t*>(r1 + 16 * st + 8 + 2 * q);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const f16* wr = sm.w[warp * 32 + 8 * j + g];
                        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wr + 16 * st + 2 * q);
                        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wr + 16 * st + 8 + 2 * q);
#pragma unroll
                        for (int i = 0; i < 2; ++i) mma16816(acc[i][j], a[i][0], a[i][1], a[i][2], a[i][3], b0, b1);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int col = warp * 32 + 8 * j + 2 * q;
                    *reinterpret_cast<float2*>(&sm.dlt[16 * i + g][col]) =
                        make_float2(softplus_fast(acc[i][j][0] + bdt[j].x), softplus_fast(acc[i][j][1] + bdt[j].y));
                    *reinterpret_cast<float2*>(&sm.dlt[16 * i + g + 8][col]) =
                        make_float2(softplus_fast(acc[i][j][2] + bdt[j].x), softplus_fast(acc[i][j][3] + bdt[j].y));
                }
        }
        __syncwarp();  // a warp's threads read only the Delta of the warp's own channels
        const int nt = min(WTC, Tp - k * WTC);
        f16* yrow = ypre + (row0 + (long long)k * WTC) * di + c0 + cs;
#pragma unroll 2
        for (int t = 0; t < nt; ++t) {
            // conv + SiLU of channel cs, swapped with the partner's channel
            const float xt = __half2float(sm.x[buf][t][cs]);
            const float u = fmaf(w4.w, xt, fmaf(w4.z, x1, fmaf(w4.y, x2, fmaf(w4.x, x3, cb))));
            x4 = x3;
            x3 = x2;
            x2 = x1;
            x1 = xt;
            const float xc_s = u * rcp_fast(1.0f + fast_exp2(-u * WLOG2E));
            const float xc_o = __shfl_xor_sync(0xffffffffu, xc_s, 1);
            const float2 xc = s ? make_float2(xc_o, xc_s) : make_float2(xc_s, xc_o);
            const float2 d = *reinterpret_cast<const float2*>(&sm.dlt[t][cl]);
            const float2 dx = __fmul2_rn(d, xc);
            // B, C of this half's 8 states (fp16 in shared memory)
            const uint4 bq = *reinterpret_cast<const uint4*>(&sm.bc[buf][t][8 * s]);
            const uint4 cq = *reinterpret_cast<const uint4*>(&sm.bc[buf][t][16 + 8 * s]);
            const uint32_t bw[4] = {bq.x, bq.y, bq.z, bq.w};
            const uint32_t cw[4] = {cq.x, cq.y, cq.z, cq.w};
            float2 y = make_float2(0.f, 0.f);
#pragma unroll
            for (int n2 = 0; n2 < 4; ++n2) {
                const float2 Bv = __half22float2(*reinterpret_cast<const __half2*>(&bw[n2]));
                const float2 Cv = __half22float2(*reinterpret_cast<const __half2*>(&cw[n2]));
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int n = 2 * n2 + e;
                    const float bn = e ? Bv.y : Bv.x, cn = e ? Cv.y : Cv.x;
                    const float2 ad = __fmul2_rn(d, A2[n]);
                    const float2 a = make_float2(fast_exp2(ad.x), fast_exp2(ad.y));
                    h[n] = __ffma2_rn(a, h[n], __fmul2_rn(dx, make_float2(bn, bn)));
                    y = __ffma2_rn(make_float2(cn, cn), h[n], y);
                }
            }
            // the other half's states
            y.x += __shfl_xor_sync(0xffffffffu, y.x, 1);
            y.y += __shfl_xor_sync(0xffffffffu, y.y, 1);
            const float ys = (s ? y.y : y.x) + Dc * xc_s;
            yrow[(long long)t * di] = __float2half_rn(ys);
        }
        if (k + 1 == nchunk && conv_out) {
            // conv state: the last four inputs of the sequence, oldest first
            *reinterpret_cast<float4*>(conv_out + ((long long)b * di + c0 + cs) * 4) = make_float4(x4, x3, x2, x1);
        }
    }
    if (h_out) {
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            h_out[((long long)b * di + c0 + cl) * 16 + 8 * s + n] = h[n].x;
            h_out[((long long)b * di + c0 + cl + 1) * 16 + 8 * s + n] = h[n].y;
        }
    }
}

}  // namespace

bool scan_wide_applies(int B, int di, int dt_rank, int sm_count) {
    // one thread per channel: the GPU needs a few blocks of 64 per SM
    return di % WCH == 0 && dt_rank > 0 && dt_rank <= WRMAX && dt_rank % 4 == 0 &&
           (long long)B * (di / WCH) >= 2LL * sm_count;
}

int launch_conv_scan_wide(const Ctx& ctx, const f16* P, long long ldP, int col_x, int col_B, int col_dt, int dt_rank,
                          const f16* wdt, int ld_wdt, const float* b_dt, const float* conv_w, const float* conv_b,
                          const float* A_log, const float* D, f16* ypre, float* h_out, float* conv_out, int B, int Tp,
                          int di) {
    if (di % WCH || dt_rank <= 0 || dt_rank > WRMAX || dt_rank % 4 || col_x % 8 || col_B % 8 || col_dt % 4 ||
        ldP % 8 || ld_wdt % 8 || ld_wdt < 16 * ((dt_rank + 15) / 16) || ld_wdt > WDLD ||
        (reinterpret_cast<uintptr_t>(P) & 15) || (reinterpret_cast<uintptr_t>(wdt) & 15) ||
        (reinterpret_cast<uintptr_t>(conv_w) & 15) || (conv_out && (reinterpret_cast<uintptr_t>(conv_out) & 15)))
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
