// Decode step kernels: attention of one new query per (sequence, head) over the
// meta block + KV ring ("Lecture 04", section 1: decode reads every cached K, V of
// the span; "Hymba Guide", Cross-Layer KV Cache Sharing: the consumer layer reads
// the producer's cache), and the O(1) SSM step on the fixed-size state ("Lecture
// 04", section 2).
//
// Cache layout: k_cache [B, G, cap, dh], v_cache [B, G, cap, dv]; position p < n_meta
// in slot p, position p >= n_meta in slot n_meta + (p - n_meta) mod (cap - n_meta).
#include <algorithm>

#include "kernels.h"
#include "tc.cuh"
#include "warp_mma.cuh"

namespace hymba {

namespace {

constexpr int DH = 64;
constexpr int MAX_R = 8;        // query heads per KV head handled by one block
constexpr int MAX_CHUNK = 256;  // keys per split
constexpr float LOG2E = 1.4426950408889634f;

// Visible key list of the query at position p: meta positions [0, min(n_meta, p+1)),
// then the n_win positions [lo, p] (none while p is inside the meta block). Returns
// false when the ring cannot hold the span.
__device__ __forceinline__ bool decode_span(int p, int n_meta, int window, int ring, int* meta_n,
                                            int* lo, int* n_win) {
    *meta_n = min(n_meta, p + 1);
    *lo = window > 0 ? max(n_meta, p - window + 1) : n_meta;
    *n_win = max(0, p + 1 - *lo);
    return p >= 0 && *n_win <= ring;
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

// An fp16 pair (the raw bits of two f16) as two floats.
__device__ __forceinline__ float2 x2float(uint32_t v) {
    __half2 h;
    memcpy(&h, &v, 4);
    return __half22float2(h);
}

// PV phase of the register-streaming kernel: 128 threads = (DV / 8 pieces of 8 V elements)
// x (128 / (DV / 8) key groups)
template <int DV>
constexpr int kgroups() { return 128 / (DV / 8); }

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
    static_assert(DV == 64 || DV == 128, "V head dim");
    constexpr int KGROUPS = kgroups<DV>();
    constexpr int PIECES = DV / 8;
    static_assert(R >= 1 && R <= 8, "query heads per KV head");
    __shared__ __align__(16) float ps[MAX_CHUNK][8];
    __shared__ int slots[MAX_CHUNK];
    __shared__ float stat[R][2];
    __shared__ __align__(16) float red[KGROUPS][R][DV];
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p = len[b] + pos_offset;
    const int ring = cap - n_meta;
    int meta_n, lo, n_win;
    const bool ok = decode_span(p, n_meta, window, ring, &meta_n, &lo, &n_win);
    if (!ok && s == 0 && g == 0 && tid == 0) set_status(status, HYMBA_ERR_DEVICE_RANGE);
    const int L = ok ? meta_n + n_win : 0;
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
        const int eb = tid % PIECES, kg = tid / PIECES;
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
        part[(((long long)b * H + g * R + r) * n_split + s) * (DV + 4) + e] = sum;
    }
    if (tid < R) {
        float* st = part + (((long long)b * H + g * R + tid) * n_split + s) * (DV + 4) + DV;
        st[0] = nk > 0 ? stat[tid][0] : -INFINITY;
        st[1] = nk > 0 ? stat[tid][1] : 0.f;
    }
}

// ---------------------------------------------------------------------------
// 16-bit K/V: the split's K and V rows in shared memory, scores and P V on the tensor
// cores (warp-level m16n8k16 MMAs, fp16 operands, fp32 accumulators)
// ---------------------------------------------------------------------------
// Shared memory of one block for splits of up to max_chunk keys: K [NKP][64] and
// V [NKP][DV] fp16 rows (16-byte chunks XOR-swizzled by the row's low three bits, so
// that the eight rows an ldmatrix reads fall in eight different bank groups), P as two
// fp16 parts [2][8 heads][NKP + 8], the slot of every key, and the per-warp partial
// maxima and sums. NKP = max_chunk rounded up to 64.
__host__ __device__ constexpr int mma_nkp(int max_chunk) { return (max_chunk + 63) / 64 * 64; }
__host__ __device__ constexpr size_t mma_smem_bytes(int max_chunk, int dv) {
    return (size_t)mma_nkp(max_chunk) * (DH + dv) * 2 + 2 * 8 * ((size_t)mma_nkp(max_chunk) + 8) * 2 +
           (size_t)mma_nkp(max_chunk) * 4 + 2 * 4 * 8 * 4;
}

// One block (four warps) per (key split, KV head, sequence) serves the R <= 8 query
// heads of the KV head. Every K and V row of the split is requested up front by 16-byte
// asynchronous copies (K, then V, as two commit groups), so the block's whole share of
// the cache is in flight while it waits. Scores S^T = K q^T: the 16-key tiles of K are
// the MMA's A operand (ldmatrix), the R queries (padded to 8) its B operand, held in
// registers for the block's life; warp w takes key tiles w, w + 4, ... The split's
// max per head meets across the warps in shared memory. p = exp2(s - max) enters P V as
// two fp16 parts, p = p_hi + p_lo (p_hi = p rounded to fp16, p_lo the rounded remainder),
// two MMAs against the same V fragment, so the weights keep about 22 bits (a single
// fp16 rounding of p costs up to 2^-11 of every weight). P V: O^T = V^T P^T, V^T 16-row
// tiles by transposing ldmatrix, P^T from shared memory; warp w takes the V columns
// [w DV / 4, (w + 1) DV / 4) over all keys, so no reduction across warps.
template <int R, int DV>
__device__ __forceinline__ void
attn_decode_mma_body(const f16* __restrict__ P, long long ldP, const f16* __restrict__ k_cache,
                     const f16* __restrict__ v_cache, int cap, const int* __restrict__ len, int pos_offset,
                     float* __restrict__ part, int n_split, int H, int G, int n_meta, int window, int max_chunk,
                     int* status, int s, int g, int b, unsigned char* smem) {
    griddep_sync();
    static_assert(DV == 64 || DV == 128, "V head dim");
    static_assert(R >= 1 && R <= 8, "query heads per KV head");
    constexpr int VCH = DV / 8;         // 16-byte chunks per V row
    constexpr int MTW = DV / 64;        // 16-column V^T tiles per warp
    const int NKP = mma_nkp(max_chunk);
    const int PST = NKP + 8;            // fp16 elements per P row (bank-conflict-free B loads)
    unsigned char* Ks = smem;
    unsigned char* Vs = smem + (size_t)NKP * DH * 2;
    f16* Ps = reinterpret_cast<f16*>(Vs + (size_t)NKP * DV * 2);
    f16* Pl = Ps + 8 * PST;
    int* slots = reinterpret_cast<int*>(Pl + 8 * PST);
    float* red = reinterpret_cast<float*>(slots + NKP);  // [2][4 warps][8 heads]
    float* Os = reinterpret_cast<float*>(Ks);            // [R][DV + 4] once K is no longer read
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;            // MMA fragment row group and column pair
    const int p = len[b] + pos_offset;
    const int ring = cap - n_meta;
    int meta_n, lo, n_win;
    const bool span_ok = decode_span(p, n_meta, window, ring, &meta_n, &lo, &n_win);
    if (!span_ok && s == 0 && g == 0 && tid == 0) set_status(status, HYMBA_ERR_DEVICE_RANGE);
    const int L = span_ok ? meta_n + n_win : 0;
    const int chunk = (L + n_split - 1) / n_split;
    const int k0 = min(L, s * chunk), k1 = min(L, k0 + chunk);
    const int nk = k1 - k0;
    const int nkt = (nk + 15) / 16;  // 16-key tiles
    const int nk16 = nkt * 16;
    float* const rec = part + (((long long)b * H + g * R) * n_split + s) * (DV + 4);
    const long long rec_head = (long long)n_split * (DV + 4);
    if (nk == 0) {
        for (int i = tid; i < R * (DV + 4); i += blockDim.x) {
            const int r = i / (DV + 4), e = i - r * (DV + 4);
            rec[r * rec_head + e] = e == DV ? -INFINITY : 0.f;
        }
        return;
    }
    // cache slot of every key of the split (keys past nk repeat the first, masked below)
    for (int kk = tid; kk < nk16; kk += blockDim.x) {
        const int idx = k0 + (kk < nk ? kk : 0);
        const int j = idx < meta_n ? idx : lo + (idx - meta_n);
        slots[kk] = j < n_meta ? j : n_meta + (j - n_meta) % ring;
    }
    __syncthreads();
    const long long kvbase = ((long long)b * G + g) * cap;
    const unsigned char* kb = reinterpret_cast<const unsigned char*>(k_cache + kvbase * DH);
    const unsigned char* vb = reinterpret_cast<const unsigned char*>(v_cache + kvbase * DV);
    {
        // K: eight threads per 128-byte row, rows tid / 8 + 16 i (the swizzle term is fixed)
        const int c = tid & 7, r0 = tid >> 3, sw = ((c ^ (r0 & 7)) << 4);
        for (int r = r0; r < nk16; r += 16)
            wm::cpa16(Ks + r * (DH * 2) + sw, kb + (long long)slots[r] * (DH * 2) + c * 16);
        wm::cpa_commit();
        // V: VCH threads per row
        constexpr int RPI = 128 / VCH;  // rows per pass
        const int cv = tid % VCH, rv0 = tid / VCH, swv = ((cv ^ (rv0 & 7)) << 4);
        for (int r = rv0; r < nk16; r += RPI)
            wm::cpa16(Vs + r * (DV * 2) + swv, vb + (long long)slots[r] * (DV * 2) + cv * 16);
        wm::cpa_commit();
    }
    // B operand of the scores: q^T, lane (gq, tq) holds dims 16 ks + 2 tq (+1, +8, +9) of
    // query head gq (zero past R)
    uint32_t qb[4][2];
    {
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(P + (long long)b * ldP + (g * R + gq) * DH);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            qb[ks][0] = gq < R ? qrow[8 * ks + tq] : 0u;
            qb[ks][1] = gq < R ? qrow[8 * ks + tq + 4] : 0u;
        }
    }
    wm::cpa_wait1();
    __syncthreads();
    // scores of the warp's key tiles: c[0..1] keys 16 t + gq, heads 2 tq, 2 tq + 1;
    // c[2..3] the same heads at key 16 t + gq + 8
    constexpr int MAXT = MAX_CHUNK / 64;  // key tiles per warp
    float sc[MAXT][4];
    const float qk_scale = LOG2E * 0.125f;  // log2(e) / sqrt(64)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int i = 0; i < MAXT; ++i) {
        const int t = warp + 4 * i;
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[i][e] = 0.f;
        if (t < nkt) {
            const int row = 16 * t + (lane & 15);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4];
                wm::ldsm_x4(a, Ks + row * (DH * 2) + (((2 * ks + (lane >> 4)) ^ (row & 7)) << 4));
                wm::mma_f16(sc[i], a[0], a[1], a[2], a[3], qb[ks][0], qb[ks][1]);
            }
            const bool v0 = 16 * t + gq < nk, v1 = 16 * t + gq + 8 < nk;
            sc[i][0] = v0 ? sc[i][0] * qk_scale : -INFINITY;
            sc[i][1] = v0 ? sc[i][1] * qk_scale : -INFINITY;
            sc[i][2] = v1 ? sc[i][2] * qk_scale : -INFINITY;
            sc[i][3] = v1 ? sc[i][3] * qk_scale : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(sc[i][0], sc[i][2]));
            mx1 = fmaxf(mx1, fmaxf(sc[i][1], sc[i][3]));
        }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (gq == 0) {
        red[warp * 8 + 2 * tq] = mx0;
        red[warp * 8 + 2 * tq + 1] = mx1;
    }
    __syncthreads();
    const float M0 = fmaxf(fmaxf(red[2 * tq], red[8 + 2 * tq]), fmaxf(red[16 + 2 * tq], red[24 + 2 * tq]));
    const float M1 =
        fmaxf(fmaxf(red[2 * tq + 1], red[9 + 2 * tq]), fmaxf(red[17 + 2 * tq], red[25 + 2 * tq]));
    // p = exp2(s - max) (every head sees every key, so the max is finite) as p_hi + p_lo
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int i = 0; i < MAXT; ++i) {
        const int t = warp + 4 * i;
        if (t < nkt) {
            const int key = 16 * t + gq;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pe = fast_exp2(sc[i][e] - ((e & 1) ? M1 : M0));
                const __half hi = __float2half_rn(pe);
                const __half lo = __float2half_rn(pe - __half2float(hi));
                const int at = (2 * tq + (e & 1)) * PST + key + ((e & 2) ? 8 : 0);
                Ps[at] = hi;
                Pl[at] = lo;
                if (e & 1) l1 += pe; else l0 += pe;
            }
        }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (gq == 0) {
        red[32 + warp * 8 + 2 * tq] = l0;
        red[32 + warp * 8 + 2 * tq + 1] = l1;
    }
    wm::cpa_wait0();
    __syncthreads();
    // P V over all keys for the warp's V columns
    float oc[MTW][4];
#pragma unroll
    for (int m = 0; m < MTW; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) oc[m][e] = 0.f;
    const uint32_t* Pw = reinterpret_cast<const uint32_t*>(Ps) + gq * (PST / 2);
    const uint32_t* Plw = reinterpret_cast<const uint32_t*>(Pl) + gq * (PST / 2);
    const int vrow = (lane & 7) + ((lane >> 4) << 3);  // key within the 16-key step
    const int vch = (lane >> 3) & 1;                   // chunk within the 16-column tile
    for (int t = 0; t < nkt; ++t) {
        const uint32_t b0 = Pw[8 * t + tq], b1 = Pw[8 * t + tq + 4];
        const uint32_t c0 = Plw[8 * t + tq], c1 = Plw[8 * t + tq + 4];
        const int key = 16 * t + vrow;
        const unsigned char* vr = Vs + key * (DV * 2);
#pragma unroll
        for (int m = 0; m < MTW; ++m) {
            const int c = 2 * (warp * MTW + m) + vch;
            uint32_t a[4];
            wm::ldsm_x4_t(a, vr + ((c ^ (key & 7)) << 4));
            wm::mma_f16(oc[m], a[0], a[1], a[2], a[3], b0, b1);
            wm::mma_f16(oc[m], a[0], a[1], a[2], a[3], c0, c1);
        }
    }
    // (Os reuses K, whose last reads came before the two barriers above)
#pragma unroll
    for (int m = 0; m < MTW; ++m) {
        const int col = 16 * (warp * MTW + m) + gq;
        if (2 * tq < R) {
            Os[(2 * tq) * (DV + 4) + col] = oc[m][0];
            Os[(2 * tq) * (DV + 4) + col + 8] = oc[m][2];
        }
        if (2 * tq + 1 < R) {
            Os[(2 * tq + 1) * (DV + 4) + col] = oc[m][1];
            Os[(2 * tq + 1) * (DV + 4) + col + 8] = oc[m][3];
        }
    }
    __syncthreads();
    for (int i = tid; i < R * (DV / 4); i += blockDim.x) {
        const int r = i / (DV / 4), q = i - r * (DV / 4);
        *reinterpret_cast<float4*>(rec + r * rec_head + 4 * q) =
            *reinterpret_cast<const float4*>(Os + r * (DV + 4) + 4 * q);
    }
    if (tid < R) {
        const float mx = fmaxf(fmaxf(red[tid], red[8 + tid]), fmaxf(red[16 + tid], red[24 + tid]));
        const float sum = red[32 + tid] + red[40 + tid] + red[48 + tid] + red[56 + tid];
        rec[tid * rec_head + DV] = mx;
        rec[tid * rec_head + DV + 1] = sum;
    }
}

template <int R, int DV>
__global__ void __launch_bounds__(128, 4)
attn_decode_mma_kernel(const f16* __restrict__ P, long long ldP, const f16* __restrict__ k_cache,
                       const f16* __restrict__ v_cache, int cap, const int* __restrict__ len, int pos_offset,
                       float* __restrict__ part, int n_split, int H, int G, int n_meta, int window, int max_chunk,
                       int* status) {
    extern __shared__ __align__(128) unsigned char mm_smem[];
    attn_decode_mma_body<R, DV>(P, ldP, k_cache, v_cache, cap, len, pos_offset, part, n_split, H, G, n_meta, window,
                                max_chunk, status, blockIdx.x, blockIdx.y, blockIdx.z, mm_smem);
}

template <typename T, int DV>
__global__ void __launch_bounds__(DV)
attn_decode_combine_kernel(const float* __restrict__ part, int n_split, T* __restrict__ O, int H) {
    griddep_sync();
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
    const float* base = part + ((long long)b * H + h) * n_split * (DV + 4);
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, base[s * (DV + 4) + DV]);
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < n_split; ++s) {
            const float ms = base[s * (DV + 4) + DV];
            const float w = exp2f(ms - M);
            num = fmaf(w, base[s * (DV + 4) + e], num);
            den = fmaf(w, base[s * (DV + 4) + DV + 1], den);
        }
    }
    O[((long long)b * H + h) * DV + e] = from_f<T>(den > 0.f ? num / den : 0.f);
}

constexpr int SSM_WARPS = 4;   // warps per block
constexpr int SSM_RPT = 2;     // sequences per thread: rows warp and warp + 4 of the block's 8
constexpr int SSM_ROWS = SSM_WARPS * SSM_RPT;
constexpr int SSM_CH = 32;     // channels per block, one per lane
constexpr int SSM_PAIRS = 128; // W_dt column pairs staged per pass (dt_rank <= 256 in one pass)
constexpr int SSM_WLD = 4;     // 16-byte W_dt loads per thread in the wide staging (32 rows x <= 64 pairs)
constexpr int SSM_XLD = 4;     // 4-byte dt_low loads per thread in the wide staging (8 rows x <= 64 pairs)

// A pair of adjacent W_dt entries of one channel as held in shared memory: the raw
// bits of two bf16 (exact on unpacking), or two floats.
template <typename TW> struct WSlot { using type = float2; };
template <> struct WSlot<bf16> { using type = uint32_t; };
__device__ __forceinline__ float2 wunpack(float2 v) { return v; }
__device__ __forceinline__ float2 wunpack(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ float2 wpack(float lo, float hi) { return make_float2(lo, hi); }
__device__ __forceinline__ uint32_t wpack(bf16 lo, bf16 hi) {
    return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// One decode step of the selective SSM for (sequence b, channel c), with the Delta
// projection of the new token folded in: Delta = softplus(dt_low . W_dt[c] + b_dt[c])
// ("Hymba Guide", Parallel Hybrid-Head Layer Formulation: the SSM heads take Delta,
// B, C from the shared input projection). Block = 8 sequences x 32 channels, each
// thread one channel of two sequences (the W_dt row and the per-channel constants are
// read once for both). The block's 32 rows of W_dt and 8 dt_low rows are staged in
// shared memory (rows padded to an odd number of slots, so that the per-lane row reads
// hit distinct banks); with 16-bit operands and an even dt_rank <= 128 the staging is
// a few wide loads per thread. Every load that does not depend on Delta (the state rows,
// the conv state, x, the per-channel constants, and the rows' B and C, copied once per
// block into shared memory) is issued before the staging, so the block waits for one
// round trip to memory rather than one per stage.
template <typename T, typename TW>
__device__ __forceinline__ void
ssm_decode_body(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C,
                int col_dtl, const TW* __restrict__ w_dt, const float* __restrict__ b_dt, int r,
                int wide, const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                const float* __restrict__ A_log, const float* __restrict__ Dp,
                float* __restrict__ h, float* __restrict__ conv, T* __restrict__ ypre, int B,
                int di, int hp, int bx, int by, unsigned char* ssm_smem) {
    griddep_sync();
    using Slot = typename WSlot<TW>::type;
    constexpr int NS = 16, KC = 4;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c0 = bx * SSM_CH, b0 = by * SSM_ROWS;
    const int c = c0 + lane;
    const bool cok = c < di;
    int bs[SSM_RPT];
    bool ok[SSM_RPT];
#pragma unroll
    for (int u = 0; u < SSM_RPT; ++u) {
        bs[u] = b0 + warp + u * SSM_WARPS;
        ok[u] = cok && bs[u] < B;
    }
    const int npairs = (r + 1) / 2;
    const int cp = min(npairs, SSM_PAIRS);
    const int RS = cp | 1;
    Slot* Ws = reinterpret_cast<Slot*>(ssm_smem);
    float2* xs = reinterpret_cast<float2*>(ssm_smem + ((SSM_CH * RS * sizeof(Slot) + 15) & ~size_t(15)));
    // B and C of the block's rows: [SSM_ROWS][2][NS] in the projection's type
    T* bcs = reinterpret_cast<T*>(xs + SSM_ROWS * cp);
    {
        constexpr int CH16 = NS * (int)sizeof(T) / 16;  // 16-byte pieces of one B or C row
        if (tid < SSM_ROWS * 2 * CH16) {
            const int row = tid / (2 * CH16), w = (tid / CH16) & 1, k = tid % CH16;
            if (b0 + row < B)
                wm::cpa16(bcs + (row * 2 + w) * NS + k * (16 / (int)sizeof(T)),
                          P + (long long)(b0 + row) * ldP + (w ? col_C : col_B) + k * (16 / (int)sizeof(T)));
        }
        wm::cpa_commit();
    }
    // the state rows, the conv state, x and the per-channel constants
    float hv[SSM_RPT][NS];
    float4 cst4[SSM_RPT];
    float xin[SSM_RPT];
#pragma unroll
    for (int u = 0; u < SSM_RPT; ++u) {
        const long long idx = (long long)bs[u] * di + c;
        const float4* hp4 = reinterpret_cast<const float4*>(h + idx * NS);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
            const float4 t = ok[u] ? hp4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
            hv[u][4 * q] = t.x; hv[u][4 * q + 1] = t.y; hv[u][4 * q + 2] = t.z; hv[u][4 * q + 3] = t.w;
        }
        cst4[u] = ok[u] ? *reinterpret_cast<const float4*>(conv + idx * KC) : make_float4(0.f, 0.f, 0.f, 0.f);
        xin[u] = ok[u] ? to_f(P[(long long)bs[u] * ldP + col_x + c]) : 0.f;
    }
    float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
    float cb = 0.f, bdt = 0.f, Dc = 0.f;
    float Ae[NS];  // -exp(A_log) log2(e): exp(Delta A) = exp2(Delta Ae)
    if (cok) {
        w4 = *reinterpret_cast<const float4*>(conv_w + (long long)c * KC);
        cb = conv_b[c];
        bdt = b_dt[hp > 0 ? c / hp : c];
        Dc = Dp[c];
        if (hp > 0) {
            // SSD form: one A per head, for every state
            const float a = -fast_exp2(A_log[c / hp] * LOG2E) * LOG2E;
#pragma unroll
            for (int n = 0; n < NS; ++n) Ae[n] = a;
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 a4 = *reinterpret_cast<const float4*>(A_log + (long long)c * NS + 4 * k);
                Ae[4 * k] = -fast_exp2(a4.x * LOG2E) * LOG2E;
                Ae[4 * k + 1] = -fast_exp2(a4.y * LOG2E) * LOG2E;
                Ae[4 * k + 2] = -fast_exp2(a4.z * LOG2E) * LOG2E;
                Ae[4 * k + 3] = -fast_exp2(a4.w * LOG2E) * LOG2E;
            }
        }
    }
    float2 dacc[SSM_RPT];
#pragma unroll
    for (int u = 0; u < SSM_RPT; ++u) dacc[u] = make_float2(0.f, 0.f);
    if constexpr (sizeof(TW) == 2) {
        if (wide) {
            // one pass: the block's W_dt rows are one contiguous run of 32 * r entries
            // (16-byte aligned), the dt_low rows r/2 fp16 pairs each
            const int n4 = SSM_CH * npairs / 4;
            const uint4* wsrc = reinterpret_cast<const uint4*>(w_dt + (long long)c0 * r);
            uint4 wb[SSM_WLD];
#pragma unroll
            for (int k = 0; k < SSM_WLD; ++k)
                if (tid + k * SSM_WARPS * 32 < n4) wb[k] = __ldg(wsrc + tid + k * SSM_WARPS * 32);
            const int nx = SSM_ROWS * npairs;
            uint32_t xb[SSM_XLD];
#pragma unroll
            for (int k = 0; k < SSM_XLD; ++k) {
                const int i = tid + k * SSM_WARPS * 32;
                xb[k] = 0u;
                if (i < nx) {
                    const int row = i / npairs, q = i - row * npairs;
                    if (b0 + row < B)
                        xb[k] = *reinterpret_cast<const uint32_t*>(P + (long long)(b0 + row) * ldP + col_dtl + 2 * q);
                }
            }
#pragma unroll
            for (int k = 0; k < SSM_WLD; ++k) {
                const int i4 = tid + k * SSM_WARPS * 32;
                if (i4 < n4) {
                    int row = (4 * i4) / npairs, q = 4 * i4 - row * npairs;
                    const uint32_t wv[4] = {wb[k].x, wb[k].y, wb[k].z, wb[k].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        Ws[row * RS + q] = wv[j];
                        if (++q == npairs) { q = 0; ++row; }
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < SSM_XLD; ++k) {
                const int i = tid + k * SSM_WARPS * 32;
                if (i < nx) {
                    const int row = i / npairs, q = i - row * npairs;
                    xs[row * cp + q] = x2float(xb[k]);
                }
            }
            __syncthreads();
#pragma unroll 4
            for (int q = 0; q < npairs; ++q) {
                const float2 wv = wunpack(Ws[lane * RS + q]);
#pragma unroll
                for (int u = 0; u < SSM_RPT; ++u)
                    dacc[u] = __ffma2_rn(wv, xs[(warp + u * SSM_WARPS) * cp + q], dacc[u]);
            }
        }
    }
    if (!(sizeof(TW) == 2 && wide)) {
        // general staging: any dt_rank and weight type, in passes of SSM_PAIRS pairs
        const TW wz = from_f<TW>(0.f);
        for (int q0 = 0; q0 < npairs; q0 += cp) {
            const int nq = min(cp, npairs - q0);
            if (q0) __syncthreads();
            for (int cc = warp; cc < SSM_CH; cc += SSM_WARPS) {
                const int ch = c0 + cc;
                const long long wrow = hp > 0 ? ch / hp : ch;  // SSD form: the head's row
                for (int q = lane; q < nq; q += 32) {
                    const int j = 2 * (q0 + q);
                    TW lo = wz, hi = wz;
                    if (ch < di) {
                        lo = w_dt[wrow * r + j];
                        if (j + 1 < r) hi = w_dt[wrow * r + j + 1];
                    }
                    Ws[cc * RS + q] = wpack(lo, hi);
                }
            }
            for (int row = warp; row < SSM_ROWS; row += SSM_WARPS) {
                for (int q = lane; q < nq; q += 32) {
                    const int j = 2 * (q0 + q);
                    float lo = 0.f, hi = 0.f;
                    if (b0 + row < B) {
                        const T* xr = P + (long long)(b0 + row) * ldP + col_dtl;
                        lo = to_f(xr[j]);
                        if (j + 1 < r) hi = to_f(xr[j + 1]);
                    }
                    xs[row * cp + q] = make_float2(lo, hi);
                }
            }
            __syncthreads();
            for (int q = 0; q < nq; ++q) {
                const float2 wv = wunpack(Ws[lane * RS + q]);
#pragma unroll
                for (int u = 0; u < SSM_RPT; ++u)
                    dacc[u] = __ffma2_rn(wv, xs[(warp + u * SSM_WARPS) * cp + q], dacc[u]);
            }
        }
    }
    wm::cpa_wait0();
    __syncthreads();  // B and C are in
    if (!cok) return;
#pragma unroll
    for (int u = 0; u < SSM_RPT; ++u) {
        if (!ok[u]) continue;
        const long long idx = (long long)bs[u] * di + c;
        const float d = softplus_fast(dacc[u].x + dacc[u].y + bdt);
        // shift the new input into the conv state (oldest first), then convolve
        float4* cst = reinterpret_cast<float4*>(conv + idx * KC);
        const float4 c4 = cst4[u];
        const float cs[KC] = {c4.y, c4.z, c4.w, xin[u]};
        float acc = cb;
        acc = fmaf(w4.x, cs[0], acc);
        acc = fmaf(w4.y, cs[1], acc);
        acc = fmaf(w4.z, cs[2], acc);
        acc = fmaf(w4.w, cs[3], acc);
        *cst = make_float4(cs[0], cs[1], cs[2], cs[3]);
        const float xc = silu_f(acc);
        const float dx = d * xc;
        const T* Bs = bcs + (warp + u * SSM_WARPS) * 2 * NS;  // this row's B, then C
        float y = 0.f;
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            const float a = fast_exp2(d * Ae[n]);
            hv[u][n] = fmaf(a, hv[u][n], dx * to_f(Bs[n]));
            y = fmaf(to_f(Bs[NS + n]), hv[u][n], y);
        }
        float4* hp = reinterpret_cast<float4*>(h + idx * NS);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q)
            hp[q] = make_float4(hv[u][4 * q], hv[u][4 * q + 1], hv[u][4 * q + 2], hv[u][4 * q + 3]);
        ypre[idx] = from_f<T>(fmaf(Dc, xc, y));
    }
}


template <typename T, typename TW>
__global__ void __launch_bounds__(SSM_WARPS * 32, 4)
ssm_decode_kernel(const T* __restrict__ P, long long ldP, int col_x, int col_B, int col_C,
                  int col_dtl, const TW* __restrict__ w_dt, const float* __restrict__ b_dt, int r,
                  int wide, const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                  const float* __restrict__ A_log, const float* __restrict__ Dp,
                  float* __restrict__ h, float* __restrict__ conv, T* __restrict__ ypre, int B,
                  int di, int hp) {
    extern __shared__ __align__(16) unsigned char ssm_smem[];
    ssm_decode_body<T, TW>(P, ldP, col_x, col_B, col_C, col_dtl, w_dt, b_dt, r, wide, conv_w, conv_b, A_log, Dp, h,
                           conv, ypre, B, di, hp, blockIdx.x, blockIdx.y, ssm_smem);
}

// The decode attention and the SSM step of a layer in one launch (both read only the
// in-projection's rows and write disjoint outputs): n_ssm blocks, spread evenly through
// the grid, run the SSM step and the rest the attention's (split, KV head, sequence)
// blocks, so the SSM's loads of the state overlap the attention's stream of the cache.
struct DecodeAttnArgs {
    const f16* P;
    long long ldP;
    const f16* k_cache;
    const f16* v_cache;
    int cap;
    const int* len;
    int pos_offset;
    float* part;
    int n_split, H, G, n_meta, window, max_chunk;
};
template <typename TW>
struct DecodeSsmArgs {
    const f16* P;
    long long ldP;
    int col_x, col_B, col_C, col_dtl;
    const TW* w_dt;
    const float* b_dt;
    int r, wide;
    const float *conv_w, *conv_b, *A_log, *D;
    float *h, *conv;
    f16* ypre;
    int B, di, hp, gx;
};

template <int R, int DV, typename TW>
__global__ void __launch_bounds__(128, 4)
decode_attn_ssm_kernel(const DecodeAttnArgs a, const DecodeSsmArgs<TW> m, int n_ssm, int* status) {
    extern __shared__ __align__(128) unsigned char dsm[];
    // the SSM blocks are spread evenly through the grid: block bid is the SSM block
    // floor(bid * n_ssm / n) when that count steps at bid, else attention block
    // bid - floor(bid * n_ssm / n)
    const long long n = (long long)gridDim.x, bid = blockIdx.x;
    const int k0 = (int)(bid * n_ssm / n), k1 = (int)((bid + 1) * n_ssm / n);
    if (k1 > k0) {
        ssm_decode_body<f16, TW>(m.P, m.ldP, m.col_x, m.col_B, m.col_C, m.col_dtl, m.w_dt, m.b_dt, m.r, m.wide,
                                 m.conv_w, m.conv_b, m.A_log, m.D, m.h, m.conv, m.ypre, m.B, m.di, m.hp,
                                 k0 % m.gx, k0 / m.gx, dsm);
    } else {
        const int q = (int)bid - k0;
        attn_decode_mma_body<R, DV>(a.P, a.ldP, a.k_cache, a.v_cache, a.cap, a.len, a.pos_offset, a.part, a.n_split,
                                     a.H, a.G, a.n_meta, a.window, a.max_chunk, status, q % a.n_split,
                                     (q / a.n_split) % a.G, q / (a.n_split * a.G), dsm);
    }
}

template <int DV, typename TW>
static void (*fused_kernel(int R))(const DecodeAttnArgs, const DecodeSsmArgs<TW>, int, int*) {
    switch (R) {
        case 1: return decode_attn_ssm_kernel<1, DV, TW>;
        case 2: return decode_attn_ssm_kernel<2, DV, TW>;
        case 3: return decode_attn_ssm_kernel<3, DV, TW>;
        case 4: return decode_attn_ssm_kernel<4, DV, TW>;
        case 5: return decode_attn_ssm_kernel<5, DV, TW>;
        case 6: return decode_attn_ssm_kernel<6, DV, TW>;
        case 7: return decode_attn_ssm_kernel<7, DV, TW>;
        default: return decode_attn_ssm_kernel<8, DV, TW>;
    }
}

template <int DV>
static void (*mma_kernel(int R))(const f16*, long long, const f16*, const f16*, int, const int*, int, float*, int,
                                  int, int, int, int, int, int*) {
    switch (R) {
        case 1: return attn_decode_mma_kernel<1, DV>;
        case 2: return attn_decode_mma_kernel<2, DV>;
        case 3: return attn_decode_mma_kernel<3, DV>;
        case 4: return attn_decode_mma_kernel<4, DV>;
        case 5: return attn_decode_mma_kernel<5, DV>;
        case 6: return attn_decode_mma_kernel<6, DV>;
        case 7: return attn_decode_mma_kernel<7, DV>;
        default: return attn_decode_mma_kernel<8, DV>;
    }
}

template <typename T, int DV>
static void (*stream_kernel(int R))(const T*, long long, const T*, const T*, int, const int*, int, float*, int, int,
                                    int, int, int, int*) {
    switch (R) {
        case 1: return attn_decode_kernel<T, DV, 1>;
        case 2: return attn_decode_kernel<T, DV, 2>;
        case 3: return attn_decode_kernel<T, DV, 3>;
        case 4: return attn_decode_kernel<T, DV, 4>;
        case 5: return attn_decode_kernel<T, DV, 5>;
        case 6: return attn_decode_kernel<T, DV, 6>;
        case 7: return attn_decode_kernel<T, DV, 7>;
        default: return attn_decode_kernel<T, DV, 8>;
    }
}

template <typename T, int DV>
static int attn_decode_dv(const Ctx& ctx, const T* P, long long ldP, const T* k_cache, const T* v_cache,
                          int cache_cap, const int* len, int pos_offset, float* part, int n_split, T* O, int B,
                          int H, int G, int n_meta, int window) {
    dim3 grid(n_split, G, B);
    if constexpr (std::is_same<T, f16>::value) {
        const int max_chunk = (cache_cap + n_split - 1) / n_split;
        const size_t smem = mma_smem_bytes(max_chunk, DV);
        auto kern = mma_kernel<DV>(H / G);
        if (smem > 48 * 1024) {
            static std::atomic<unsigned long long> smem_set[8];
            if (!smem_opt_in_once(smem_set[H / G - 1], kern, mma_smem_bytes(MAX_CHUNK, DV), ctx)) return HYMBA_ERR_CUDA;
        }
        HYMBA_LAUNCH(ctx, "attn_decode", kern, grid, 128, smem, P, ldP, k_cache, v_cache, cache_cap, len, pos_offset,
                     part, n_split, H, G, n_meta, window, max_chunk, ctx.status);
    } else {
        HYMBA_LAUNCH(ctx, "attn_decode", (stream_kernel<T, DV>(H / G)), grid, 128, 0, P, ldP, k_cache, v_cache,
                     cache_cap, len, pos_offset, part, n_split, H, G, n_meta, window, ctx.status);
    }
    if (!O) return HYMBA_OK;  // the caller merges the splits itself
    dim3 g2(H, B);
    auto k2 = attn_decode_combine_kernel<T, DV>;
    HYMBA_LAUNCH(ctx, "attn_decode_combine", k2, g2, DV, 0, part, n_split, O, H);
    return HYMBA_OK;
}

}  // namespace

template <typename T>
int launch_attn_decode(const Ctx& ctx, const T* P, long long ldP, const T* k_cache,
                       const T* v_cache, int cache_cap, const int* len, int pos_offset,
                       float* part, int n_split, T* O, int B, int H, int G, int dv, int n_meta,
                       int window) {
    if (H / G > MAX_R || (dv != 128 && dv != 64)) return HYMBA_ERR_UNSUPPORTED;
    if ((cache_cap + n_split - 1) / n_split > MAX_CHUNK) return HYMBA_ERR_INVALID_ARG;
    // 16-byte loads of q, K and V rows; 16-byte stores of the partial records
    if ((reinterpret_cast<uintptr_t>(P) | reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache) |
         reinterpret_cast<uintptr_t>(part)) & 15 ||
        ldP % (16 / (long long)sizeof(T)))
        return HYMBA_ERR_UNSUPPORTED;
    if (dv == 128)
        return attn_decode_dv<T, 128>(ctx, P, ldP, k_cache, v_cache, cache_cap, len, pos_offset, part, n_split, O, B,
                                      H, G, n_meta, window);
    return attn_decode_dv<T, 64>(ctx, P, ldP, k_cache, v_cache, cache_cap, len, pos_offset, part, n_split, O, B, H,
                                 G, n_meta, window);
}

template <typename T, typename TW>
int launch_ssm_decode(const Ctx& ctx, const T* P, long long ldP, int col_x, int col_B, int col_C,
                      int col_dtl, const TW* w_dt, const float* b_dt, int dt_rank,
                      const float* conv_w, const float* conv_b, const float* A_log, const float* D,
                      float* h, float* conv, T* ypre, int B, int di, int hp) {
    if (B <= 0) return HYMBA_OK;
    if (dt_rank <= 0 || hp < 0 || (hp > 0 && di % hp)) return HYMBA_ERR_INVALID_ARG;
    // 16-byte loads: the B/C columns of every projection row, conv taps, A_log and conv state
    constexpr int V = 16 / (int)sizeof(T);
    if (ldP % V || col_B % V || col_C % V || (reinterpret_cast<uintptr_t>(conv_w) & 15) ||
        (reinterpret_cast<uintptr_t>(A_log) & 15) || (reinterpret_cast<uintptr_t>(conv) & 15) ||
        (reinterpret_cast<uintptr_t>(h) & 15) || (reinterpret_cast<uintptr_t>(P) & 15))
        return HYMBA_ERR_UNSUPPORTED;
    using Slot = typename WSlot<TW>::type;
    const int npairs = (dt_rank + 1) / 2;
    const int cp = npairs < SSM_PAIRS ? npairs : SSM_PAIRS;
    const size_t smem = ((SSM_CH * (size_t)(cp | 1) * sizeof(Slot) + 15) & ~size_t(15)) +
                        (size_t)SSM_ROWS * cp * sizeof(float2) + (size_t)SSM_ROWS * 2 * 16 * sizeof(T);
    // one-pass wide staging: 16-bit W_dt with even dt_rank <= 128 (so the block's run of
    // 32 rows is 16-byte aligned and a whole number of 16-byte pieces, d_inner being a
    // multiple of 32), 4-byte dt_low pairs
    const int wide = hp == 0 && sizeof(TW) == 2 && dt_rank % 2 == 0 && npairs <= SSM_PAIRS && di % SSM_CH == 0 &&
                     (reinterpret_cast<uintptr_t>(w_dt) & 15) == 0 && col_dtl % 2 == 0 &&
                     SSM_CH * npairs / 4 <= SSM_WLD * SSM_WARPS * 32 && SSM_ROWS * npairs <= SSM_XLD * SSM_WARPS * 32;
    dim3 grid(ceil_div(di, SSM_CH), ceil_div(B, SSM_ROWS));
    HYMBA_LAUNCH(ctx, "ssm_decode", (ssm_decode_kernel<T, TW>), grid, SSM_WARPS * 32, smem, P, ldP, col_x,
                 col_B, col_C, col_dtl, w_dt, b_dt, dt_rank, wide, conv_w, conv_b, A_log, D, h, conv, ypre, B,
                 di, hp);
    return HYMBA_OK;
}

template <typename TW>
int launch_decode_attn_ssm(const Ctx& ctx, const f16* P, long long ldP, const f16* k_cache, const f16* v_cache,
                           int cache_cap, const int* len, int pos_offset, float* part, int n_split, int B, int H,
                           int G, int dv, int n_meta, int window, int col_x, int col_B, int col_C, int col_dtl,
                           const TW* w_dt, const float* b_dt, int dt_rank, const float* conv_w, const float* conv_b,
                           const float* A_log, const float* D, float* h, float* conv, f16* ypre, int di, int hp) {
    // anything outside the shapes both halves take goes to the two separate launches, which
    // report their own errors
    if (B <= 0 || dt_rank <= 0 || hp < 0 || (hp > 0 && di % hp) || G <= 0 || H % G || H / G > MAX_R ||
        (dv != 64 && dv != 128) || n_split <= 0 || (cache_cap + n_split - 1) / n_split > MAX_CHUNK)
        return HYMBA_ERR_UNSUPPORTED;
    constexpr int V = 8;  // 16-byte loads of fp16 rows
    if (ldP % V || col_B % V || col_C % V || (reinterpret_cast<uintptr_t>(conv_w) & 15) ||
        (reinterpret_cast<uintptr_t>(A_log) & 15) || (reinterpret_cast<uintptr_t>(conv) & 15) ||
        (reinterpret_cast<uintptr_t>(h) & 15) || (reinterpret_cast<uintptr_t>(P) & 15) ||
        ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache) |
          reinterpret_cast<uintptr_t>(part)) & 15))
        return HYMBA_ERR_UNSUPPORTED;
    using Slot = typename WSlot<TW>::type;
    const int npairs = (dt_rank + 1) / 2;
    const int cp = npairs < SSM_PAIRS ? npairs : SSM_PAIRS;
    const size_t smem_ssm = ((SSM_CH * (size_t)(cp | 1) * sizeof(Slot) + 15) & ~size_t(15)) +
                            (size_t)SSM_ROWS * cp * sizeof(float2) + (size_t)SSM_ROWS * 2 * 16 * sizeof(f16);
    const int wide = hp == 0 && sizeof(TW) == 2 && dt_rank % 2 == 0 && npairs <= SSM_PAIRS && di % SSM_CH == 0 &&
                     (reinterpret_cast<uintptr_t>(w_dt) & 15) == 0 && col_dtl % 2 == 0 &&
                     SSM_CH * npairs / 4 <= SSM_WLD * SSM_WARPS * 32 && SSM_ROWS * npairs <= SSM_XLD * SSM_WARPS * 32;
    const int max_chunk = (cache_cap + n_split - 1) / n_split;
    const size_t smem_attn = mma_smem_bytes(max_chunk, dv);
    const size_t smem = smem_attn > smem_ssm ? smem_attn : smem_ssm;
    DecodeAttnArgs a{P, ldP, k_cache, v_cache, cache_cap, len, pos_offset, part, n_split, H, G, n_meta, window,
                     max_chunk};
    DecodeSsmArgs<TW> m{P, ldP, col_x, col_B, col_C, col_dtl, w_dt, b_dt, dt_rank, wide, conv_w, conv_b, A_log, D,
                        h, conv, ypre, B, di, hp, ceil_div(di, SSM_CH)};
    const int n_ssm = m.gx * ceil_div(B, SSM_ROWS);
    const int n_attn = n_split * G * B;
    auto kern = dv == 128 ? fused_kernel<128, TW>(H / G) : fused_kernel<64, TW>(H / G);
    if (smem > 48 * 1024) {
        // one opt-in per kernel and device, at the largest size any launch asks for
        static std::atomic<unsigned long long> smem_set[2][8];
        const size_t most = std::max(mma_smem_bytes(MAX_CHUNK, dv), smem_ssm);
        if (!smem_opt_in_once(smem_set[dv == 128][H / G - 1], kern, most, ctx)) return HYMBA_ERR_CUDA;
    }
    HYMBA_LAUNCH(ctx, "attn_ssm_decode", kern, n_ssm + n_attn, 128, smem, a, m, n_ssm, ctx.status);
    return HYMBA_OK;
}

template int launch_decode_attn_ssm<bf16>(const Ctx&, const f16*, long long, const f16*, const f16*, int, const int*,
                                          int, float*, int, int, int, int, int, int, int, int, int, int, int,
                                          const bf16*, const float*, int, const float*, const float*, const float*,
                                          const float*, float*, float*, f16*, int, int);

template int launch_attn_decode<float>(const Ctx&, const float*, long long, const float*,
                                       const float*, int, const int*, int, float*, int, float*,
                                       int, int, int, int, int, int);
template int launch_attn_decode<f16>(const Ctx&, const f16*, long long, const f16*, const f16*,
                                     int, const int*, int, float*, int, f16*, int, int, int, int,
                                     int, int);
template int launch_ssm_decode<float, float>(const Ctx&, const float*, long long, int, int, int, int,
                                             const float*, const float*, int, const float*, const float*,
                                             const float*, const float*, float*, float*, float*, int, int, int);
template int launch_ssm_decode<f16, bf16>(const Ctx&, const f16*, long long, int, int, int, int,
                                          const bf16*, const float*, int, const float*, const float*,
                                          const float*, const float*, float*, float*, f16*, int, int, int);

}  // namespace hymba
