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

template <typename T, int DV>
__global__ void __launch_bounds__(128)
attn_decode_kernel(const T* __restrict__ P, long long ldP, const T* __restrict__ k_cache,
                   const T* __restrict__ v_cache, int cap, const int* __restrict__ len,
                   int pos_offset, float* __restrict__ part, int n_split, int H, int G,
                   int n_meta, int window, int* status) {
    griddep_sync();
    static_assert(DV == 16 * 8, "PV phase covers a V row with 16 pieces of 8");
    __shared__ __align__(16) float qs[MAX_R][DH];
    __shared__ float ps[MAX_R][MAX_CHUNK];
    __shared__ int slots[MAX_CHUNK];
    __shared__ float stat[MAX_R][2];
    __shared__ __align__(16) float red[KGROUPS][MAX_R][DV];
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int R = H / G;
    const int tid = threadIdx.x;
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

    for (int i = tid; i < R * DH; i += blockDim.x) {
        const int r = i / DH, e = i % DH;
        qs[r][e] = to_f(P[(long long)b * ldP + (g * R + r) * DH + e]) * (LOG2E * 0.125f);
    }
    for (int kk = tid; kk < nk; kk += blockDim.x) {
        const int idx = k0 + kk;
        const int j = idx < meta_n ? idx : lo + (idx - meta_n);
        slots[kk] = j < n_meta ? j : n_meta + (j - n_meta) % ring;
    }
    __syncthreads();
    // scores: one key per thread, its K row (128 bytes) loaded whole before any use so
    // that all eight 16-byte loads are in flight together; q broadcast from smem
    for (int kk = tid; kk < nk; kk += blockDim.x) {
        const T* kr = k_cache + (kvbase + slots[kk]) * DH;
        float kv[DH];
#pragma unroll
        for (int e = 0; e < DH; e += 8) load_row8<T>(kr + e, kv + e);
        float acc[MAX_R];
#pragma unroll
        for (int r = 0; r < MAX_R; ++r) acc[r] = 0.f;
#pragma unroll
        for (int e = 0; e < DH; e += 4) {
#pragma unroll
            for (int r = 0; r < MAX_R; ++r) {
                if (r < R) {
                    const float4 qa = *reinterpret_cast<const float4*>(&qs[r][e]);
                    acc[r] = fmaf(qa.x, kv[e], acc[r]);
                    acc[r] = fmaf(qa.y, kv[e + 1], acc[r]);
                    acc[r] = fmaf(qa.z, kv[e + 2], acc[r]);
                    acc[r] = fmaf(qa.w, kv[e + 3], acc[r]);
                }
            }
        }
        for (int r = 0; r < R; ++r) ps[r][kk] = acc[r];
    }
    __syncthreads();
    // per-head max and sum over this split's keys: warp w handles heads w, w+4, ...
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < R; r += 4) {
        float mx = -INFINITY;
        for (int kk = lane; kk < nk; kk += 32) mx = fmaxf(mx, ps[r][kk]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        for (int kk = lane; kk < nk; kk += 32) {
            const float e = exp2f(ps[r][kk] - mx);
            ps[r][kk] = e;
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
        float acc[MAX_R][8];
#pragma unroll
        for (int r = 0; r < MAX_R; ++r)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[r][i] = 0.f;
        // four keys per round, their V pieces loaded before any is used, so that four
        // loads per thread are in flight instead of one
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
#pragma unroll
                    for (int r = 0; r < MAX_R; ++r) {
                        if (r < R) {
                            const float pr = ps[r][kk];
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[r][i] = fmaf(pr, v[u][i], acc[r][i]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < MAX_R; ++r) {
            if (r < R) {
                *reinterpret_cast<float4*>(&red[kg][r][eb * 8]) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
                *reinterpret_cast<float4*>(&red[kg][r][eb * 8 + 4]) = make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
            }
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
    auto k1 = attn_decode_kernel<T, 128>;
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
