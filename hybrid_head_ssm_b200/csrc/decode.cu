// Decode step kernels: attention of one new query per (sequence, head) over the
// meta block + KV ring ("Lecture 04", section 1: decode reads every cached K, V of
// the span; "Hymba Guide", Cross-Layer KV Cache Sharing: the consumer layer reads
// the producer's cache), and the O(1) SSM step on the fixed-size state ("Lecture
// 04", section 2).
//
// Cache layout: k_cache [B, G, cap, dh], v_cache [B, G, cap, dv]; position p < n_meta
// in slot p, position p >= n_meta in slot n_meta + (p - n_meta) mod (cap - n_meta).
#include "kernels.h"

namespace hymba {

namespace {

constexpr int DH = 64;
constexpr int MAX_R = 8;        // query heads per KV head handled by one block
constexpr int MAX_CHUNK = 256;  // keys per split
constexpr float LOG2E = 1.4426950408889634f;

// Visible key list of the query at position p: meta positions [0, min(n_meta, p+1)),
// then positions [lo, p]. Returns false when the ring cannot hold the span.
__device__ __forceinline__ bool decode_span(int p, int n_meta, int window, int ring, int* meta_n,
                                            int* lo) {
    *meta_n = min(n_meta, p + 1);
    *lo = window > 0 ? max(n_meta, p - window + 1) : n_meta;
    const int span = p + 1 - *lo;
    return p >= 0 && span <= ring;
}

// 8 consecutive elements of a K or V row as fp32 (one or two 16-byte loads).
template <typename T>
__device__ __forceinline__ void load_row8(const T* p, float* v) {
    if constexpr (sizeof(T) == 2) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = to_f(h[i]);
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p));
        const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

constexpr int KGROUPS = 8;  // key groups of the PV phase (128 threads = 8 groups x 16 pieces of 8)

// One block per (key split, KV head, sequence) serves the R query heads of the KV head.
// Scores: four lanes per key, each holding its 16 dimensions of the R queries in
// registers and reading 32 bytes of the K row, joined by two shuffles per head. P V:
// thread (key group, 8-dimension piece) walks its keys four at a time with the V pieces
// loaded ahead of use and all R heads' weights read as two 16-byte loads per key
// (P stored [key][head]); the products are packed f32x2 FMAs.
template <typename T, int DV, int R>
__global__ void __launch_bounds__(128)
attn_decode_kernel(const T* __restrict__ P, long long ldP, const T* __restrict__ k_cache,
                   const T* __restrict__ v_cache, int cap, const int* __restrict__ len,
                   int pos_offset, float* __restrict__ part, int n_split, int H, int G,
                   int n_meta, int window, int* status) {
    griddep_sync();
    static_assert(DV == 16 * 8, "PV phase covers a V row with 16 pieces of 8");
    static_assert(R >= 1 && R <= 8, "query heads per KV head");
    __shared__ __align__(16) float ps[MAX_CHUNK][8];
    __shared__ int slots[MAX_CHUNK];
    __shared__ float stat[R][2];
    __shared__ __align__(16) float red[KGROUPS][R][DV];
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p = len[b] + pos_offset;
    const int ring = cap - n_meta;
    int meta_n, lo;
    const bool ok = decode_span(p, n_meta, window, ring, &meta_n, &lo);
    if (!ok && s == 0 && g == 0 && tid == 0) set_status(status, HYMBA_ERR_DEVICE_RANGE);
    const int L = ok ? meta_n + (p + 1 - lo) : 0;
    const int chunk = (L + n_split - 1) / n_split;
    const int k0 = min(L, s * chunk), k1 = min(L, k0 + chunk);
    const int nk = k1 - k0;
    const long long kvbase = ((long long)b * G + g) * cap;

    for (int kk = tid; kk < nk; kk += blockDim.x) {
        const int idx = k0 + kk;
        const int j = idx < meta_n ? idx : lo + (idx - meta_n);
        slots[kk] = j < n_meta ? j : n_meta + (j - n_meta) % ring;
    }
    // this lane's quarter of the head dimension (16 of 64) for the R queries, scaled by
    // log2(e) / sqrt(64)
    const int qq = lane & 3, kl = lane >> 2;
    float2 qr[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float qv[16];
        const T* qp = P + (long long)b * ldP + (g * R + r) * DH + 16 * qq;
        load_row8<T>(qp, qv);
        load_row8<T>(qp + 8, qv + 8);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            qr[r][i] = make_float2(qv[2 * i] * (LOG2E * 0.125f), qv[2 * i + 1] * (LOG2E * 0.125f));
    }
    __syncthreads();
    // scores: warp w takes keys w*8 .. w*8+7 of every 32, lane (key kl, quarter qq)
    for (int kb = warp * 8; kb < nk; kb += 32) {
        const int kk = kb + kl;
        float2 acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = make_float2(0.f, 0.f);
        if (kk < nk) {
            const T* kr = k_cache + (kvbase + slots[kk]) * DH + 16 * qq;
            float kv[16];
            load_row8<T>(kr, kv);
            load_row8<T>(kr + 8, kv + 8);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 k2 = make_float2(kv[2 * i], kv[2 * i + 1]);
#pragma unroll
                for (int r = 0; r < R; ++r) acc[r] = __ffma2_rn(qr[r][i], k2, acc[r]);
            }
        }
        float sc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float a = acc[r].x + acc[r].y;
            a += __shfl_xor_sync(0xffffffffu, a, 1);
            a += __shfl_xor_sync(0xffffffffu, a, 2);
            sc[r] = a;
        }
        if (kk < nk && qq == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r) ps[kk][r] = sc[r];
        }
    }
    __syncthreads();
    // per-head max and sum over this split's keys: warp w handles heads w, w+4, ...
    for (int r = warp; r < R; r += 4) {
        float mx = -INFINITY;
        for (int kk = lane; kk < nk; kk += 32) mx = fmaxf(mx, ps[kk][r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        for (int kk = lane; kk < nk; kk += 32) {
            const float e = exp2f(ps[kk][r] - mx);
            ps[kk][r] = e;
            sum += e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) { stat[r][0] = mx; stat[r][1] = sum; }
    }
    __syncthreads();
    // P V: thread (key group kg, piece eb) adds keys kg, kg + 8, ... for V elements eb*8..+7
    {
        const int eb = tid % 16, kg = tid / 16;
        float2 acc[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][i] = make_float2(0.f, 0.f);
        constexpr int U = 4;
        for (int kk0 = kg; kk0 < nk; kk0 += KGROUPS * U) {
            float v[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int kk = kk0 + u * KGROUPS;
                if (kk < nk) {
                    load_row8<T>(v_cache + (kvbase + slots[kk]) * DV + eb * 8, v[u]);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int kk = kk0 + u * KGROUPS;
                if (kk < nk) {
                    const float4 pa = *reinterpret_cast<const float4*>(&ps[kk][0]);
                    const float4 pb = *reinterpret_cast<const float4*>(&ps[kk][4]);
                    const float pw[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float2 pr = make_float2(pw[r], pw[r]);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            acc[r][i] = __ffma2_rn(pr, make_float2(v[u][2 * i], v[u][2 * i + 1]), acc[r][i]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            *reinterpret_cast<float4*>(&red[kg][r][eb * 8]) = make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
            *reinterpret_cast<float4*>(&red[kg][r][eb * 8 + 4]) = make_float4(acc[r][2].x, acc[r][2].y, acc[r][3].x, acc[r][3].y);
        }
    }
    __syncthreads();
    for (int i = tid; i < R * DV; i += blockDim.x) {
        const int r = i / DV, e = i % DV;
        float sum = 0.f;
#pragma unroll
        for (int k = 0; k < KGROUPS; ++k) sum += red[k][r][e];
        part[(((long long)b * H + g * R + r) * n_split + s) * (DV + 2) + e] = sum;
    }
    if (tid < R) {
        float* st = part + (((long long)b * H + g * R + tid) * n_split + s) * (DV + 2) + DV;
        st[0] = nk > 0 ? stat[tid][0] : -INFINITY;
        st[1] = nk > 0 ? stat[tid][1] : 0.f;
    }
}

template <typename T, int DV>
__global__ void __launch_bounds__(DV)
attn_decode_combine_kernel(const float* __restrict__ part, int n_split, T* __restrict__ O, int H) {
    griddep_sync();
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
    const float* base = part + ((long long)b * H + h) * n_split * (DV + 2);
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, base[s * (DV + 2) + DV]);
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < n_split; ++s) {
            const float ms = base[s * (DV + 2) + DV];
            const float w = exp2f(ms - M);
            num = fmaf(w, base[s * (DV + 2) + e], num);
            den = fmaf(w, base[s * (DV + 2) + DV + 1], den);
        }
    }
    O[((long long)b * H + h) * DV + e] = from_f<T>(den > 0.f ? num / den : 0.f);
}

template <typename T>
__global__ void __launch_bounds__(128)
ssm_decode_kernel(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C,
                  const float* __restrict__ delta, const float* __restrict__ conv_w,
                  const float* __restrict__ conv_b, const float* __restrict__ A_log,
                  const float* __restrict__ Dp, float* __restrict__ h, float* __restrict__ conv,
                  T* __restrict__ ypre, int B, int di) {
    griddep_sync();
    constexpr int NS = 16, KC = 4;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)B * di) return;
    const int b = (int)(idx / di), c = (int)(idx % di);
    const T* prow = P + (long long)b * ldP;
    // shift the new input into the conv state (oldest first), then convolve; every
    // per-channel and per-row vector below is read with 16-byte loads
    float4* cst = reinterpret_cast<float4*>(conv + idx * KC);
    const float4 c4 = *cst;
    const float cs[KC] = {c4.y, c4.z, c4.w, to_f(prow[col_x + c])};
    const float4 w4 = *reinterpret_cast<const float4*>(conv_w + (long long)c * KC);
    float acc = conv_b[c];
    acc = fmaf(w4.x, cs[0], acc);
    acc = fmaf(w4.y, cs[1], acc);
    acc = fmaf(w4.z, cs[2], acc);
    acc = fmaf(w4.w, cs[3], acc);
    *cst = make_float4(cs[0], cs[1], cs[2], cs[3]);
    const float xc = silu_f(acc);
    const float d = delta[idx];
    const float dx = d * xc;
    float Bv[NS], Cv[NS], Al[NS];
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint4 ub = *reinterpret_cast<const uint4*>(prow + col_B + 8 * k);
            const uint4 uc = *reinterpret_cast<const uint4*>(prow + col_C + 8 * k);
            const T* hb = reinterpret_cast<const T*>(&ub);
            const T* hc = reinterpret_cast<const T*>(&uc);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                Bv[8 * k + i] = to_f(hb[i]);
                Cv[8 * k + i] = to_f(hc[i]);
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 fb = *reinterpret_cast<const float4*>(prow + col_B + 4 * k);
            const float4 fc = *reinterpret_cast<const float4*>(prow + col_C + 4 * k);
            Bv[4 * k] = fb.x; Bv[4 * k + 1] = fb.y; Bv[4 * k + 2] = fb.z; Bv[4 * k + 3] = fb.w;
            Cv[4 * k] = fc.x; Cv[4 * k + 1] = fc.y; Cv[4 * k + 2] = fc.z; Cv[4 * k + 3] = fc.w;
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 a4 = *reinterpret_cast<const float4*>(A_log + (long long)c * NS + 4 * k);
        Al[4 * k] = a4.x; Al[4 * k + 1] = a4.y; Al[4 * k + 2] = a4.z; Al[4 * k + 3] = a4.w;
    }
    float4* hp = reinterpret_cast<float4*>(h + idx * NS);
    float hv[NS];
#pragma unroll
    for (int q = 0; q < NS / 4; ++q) {
        float4 t = hp[q];
        hv[4 * q] = t.x; hv[4 * q + 1] = t.y; hv[4 * q + 2] = t.z; hv[4 * q + 3] = t.w;
    }
    float y = 0.f;
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        // exp(Delta A) with A = -exp(A_log): exp2(-Delta * 2^(A_log log2 e) * log2 e)
        const float a = fast_exp2(-d * fast_exp2(Al[n] * LOG2E) * LOG2E);
        hv[n] = fmaf(a, hv[n], dx * Bv[n]);
        y = fmaf(Cv[n], hv[n], y);
    }
#pragma unroll
    for (int q = 0; q < NS / 4; ++q) hp[q] = make_float4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
    ypre[idx] = from_f<T>(fmaf(Dp[c], xc, y));
}

}  // namespace

template <typename T>
int launch_attn_decode(const Ctx& ctx, const T* P, long long ldP, const T* k_cache,
                       const T* v_cache, int cache_cap, const int* len, int pos_offset,
                       float* part, int n_split, T* O, int B, int H, int G, int dv, int n_meta,
                       int window) {
    if (H / G > MAX_R || dv != 128) return HYMBA_ERR_UNSUPPORTED;
    if ((cache_cap + n_split - 1) / n_split > MAX_CHUNK) return HYMBA_ERR_INVALID_ARG;
    dim3 grid(n_split, G, B);
    // 16-byte loads of q, K and V rows
    if ((reinterpret_cast<uintptr_t>(P) | reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15 ||
        ldP % (16 / (long long)sizeof(T)))
        return HYMBA_ERR_UNSUPPORTED;
    void (*k1)(const T*, long long, const T*, const T*, int, const int*, int, float*, int, int, int, int, int, int*);
    switch (H / G) {
        case 1: k1 = attn_decode_kernel<T, 128, 1>; break;
        case 2: k1 = attn_decode_kernel<T, 128, 2>; break;
        case 3: k1 = attn_decode_kernel<T, 128, 3>; break;
        case 4: k1 = attn_decode_kernel<T, 128, 4>; break;
        case 5: k1 = attn_decode_kernel<T, 128, 5>; break;
        case 6: k1 = attn_decode_kernel<T, 128, 6>; break;
        case 7: k1 = attn_decode_kernel<T, 128, 7>; break;
        default: k1 = attn_decode_kernel<T, 128, 8>; break;
    }
    HYMBA_LAUNCH(ctx, "attn_decode", k1, grid, 128, 0, P, ldP, k_cache, v_cache, cache_cap, len,
                 pos_offset, part, n_split, H, G, n_meta, window, ctx.status);
    dim3 g2(H, B);
    auto k2 = attn_decode_combine_kernel<T, 128>;
    HYMBA_LAUNCH(ctx, "attn_decode_combine", k2, g2, 128, 0, part, n_split, O, H);
    return HYMBA_OK;
}

template <typename T>
int launch_ssm_decode(const Ctx& ctx, const T* P, long long ldP, int col_x, int col_B, int col_C,
                      const float* delta, const float* conv_w, const float* conv_b,
                      const float* A_log, const float* D, float* h, float* conv, T* ypre, int B,
                      int di) {
    const long long n = (long long)B * di;
    // 16-byte loads: the B/C columns of every projection row, conv taps, A_log and conv state
    constexpr int V = 16 / (int)sizeof(T);
    if (ldP % V || col_B % V || col_C % V || (reinterpret_cast<uintptr_t>(conv_w) & 15) ||
        (reinterpret_cast<uintptr_t>(A_log) & 15) || (reinterpret_cast<uintptr_t>(conv) & 15) ||
        (reinterpret_cast<uintptr_t>(h) & 15) || (reinterpret_cast<uintptr_t>(P) & 15))
        return HYMBA_ERR_UNSUPPORTED;
    HYMBA_LAUNCH(ctx, "ssm_decode", ssm_decode_kernel<T>, ceil_div(n, 128), 128, 0, P, ldP, col_x,
                 col_B, col_C, delta, conv_w, conv_b, A_log, D, h, conv, ypre, B, di);
    return HYMBA_OK;
}

template int launch_attn_decode<float>(const Ctx&, const float*, long long, const float*,
                                       const float*, int, const int*, int, float*, int, float*,
                                       int, int, int, int, int, int);
template int launch_attn_decode<f16>(const Ctx&, const f16*, long long, const f16*, const f16*,
                                     int, const int*, int, float*, int, f16*, int, int, int, int,
                                     int, int);
template int launch_ssm_decode<float>(const Ctx&, const float*, long long, int, int, int,
                                      const float*, const float*, const float*, const float*,
                                      const float*, float*, float*, float*, int, int);
template int launch_ssm_decode<f16>(const Ctx&, const f16*, long long, int, int, int,
                                    const float*, const float*, const float*, const float*,
                                    const float*, float*, float*, f16*, int, int);

}  // namespace hymba
