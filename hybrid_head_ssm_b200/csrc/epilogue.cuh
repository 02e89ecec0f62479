// Epilogues of the three projections of a mixer layer. Every GEMM of the library
// (SIMT or tcgen05) hands its fp32 accumulators to epi_run64 in runs of 64
// consecutive output columns of one output row, so that RoPE (pairs i, i+32 of a
// 64-wide head) and the per-head scatter of K and V happen before rounding.
#pragma once
#include "common.cuh"

namespace hymba {

enum EpiKind { EPI_INPROJ = 0, EPI_DELTA = 1, EPI_OUT = 2 };

// How GEMM row r maps to rows of the layer's T' = n_meta + T rows per sequence.
enum RowMode {
    ROWS_DIRECT = 0,   // r is already the layer row b*T' + t
    ROWS_META = 1,     // r < n_meta is meta row r, identical for every sequence: write it B times
    ROWS_USER = 2,     // r = b*T + u is user token u of sequence b: layer row b*T' + n_meta + u
    ROWS_DECODE = 3,   // decode: r = b, position pos[b]
};

template <typename T>
struct EpiArgs {
    int kind;
    int row_mode;
    int M, N;              // GEMM output extent
    int B, Tu, Tp, n_meta; // sequences, user tokens, layer rows per sequence, meta rows
    // EPI_INPROJ
    T* P;                  // [B*T', ldP] projection (Q | (K V slots unused) | x | z | B | C | dt_low)
    long long ldP;
    T* k_out;              // producer: K after RoPE [B, G, kcap, dh] (NULL: consumer)
    T* v_out;              // producer: V [B, G, kcap, dv]
    int kcap;
    int H, G, dh, dv;
    const float2* rope;    // [T', dh/2] (cos, sin) of position * theta_i (prefill)
    const int* pos;        // decode: [B] positions held (len); the new token sits at pos[b] + pos_offset
    int pos_offset;        // decode: 0 for a producer (appends), -1 for a consumer
    int n_meta_ring;       // decode: ring length (cache_cap - n_meta)
    float rope_base;       // decode: angles computed on the fly
    // EPI_DELTA
    float* delta;          // [M, N] fp32
    const float* b_dt;
    // EPI_OUT
    T* y;                  // [M, N]
    int res_mode;          // 0: none; 1: residual = res_x row r; 2: residual = X^ row (meta or user)
    const T* res_x;
    const void* res_meta;  // [n_meta, N] of the layer's weight type
    int res_meta_bf16;     // 1: res_meta is bf16; 0: it has type T
    // in-projection GEMMs that also cover the meta rows: GEMM rows [0, meta_pad) are
    // meta rows (valid below meta_M, written for every sequence), the rest follow
    // row_mode after subtracting meta_pad
    int meta_pad;
    int meta_M;
};

// RoPE on one 64-wide head run: pairs (i, i+32) rotated by (cos, sin).
__device__ __forceinline__ void rope_run64(float* v, const float2* cs) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        float2 c = cs[i];
        float a = v[i], b = v[i + 32];
        v[i] = a * c.x - b * c.y;
        v[i + 32] = b * c.x + a * c.y;
    }
}

// cos/sin of position p for pair i of a 64-wide head, angles in double precision.
__device__ __forceinline__ float2 rope_cs_at(int p, int i, int dh, float base) {
    double theta = pow((double)base, -2.0 * (double)i / (double)dh);
    double ang = (double)p * theta;
    double s, c;
    sincos(ang, &s, &c);
    return make_float2((float)c, (float)s);
}

template <typename T>
__device__ void epi_run64(const EpiArgs<T>& e, int r, int c0, float* v) {
    int mode = e.row_mode, M = e.M;
    if (e.meta_pad > 0) {
        if (r < e.meta_pad) {
            mode = ROWS_META;
            M = e.meta_M;
        } else {
            r -= e.meta_pad;
        }
    }
    if (r >= M || c0 >= e.N) return;
    const int n = min(64, e.N - c0);
    if (e.kind == EPI_DELTA) {
        float* dst = e.delta + (long long)r * e.N + c0;
        const float* bias = e.b_dt + c0;
        if (n == 64 && (e.N & 3) == 0) {
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 bb = *reinterpret_cast<const float4*>(bias + j);
                *reinterpret_cast<float4*>(dst + j) =
                    make_float4(softplus_fast(v[j] + bb.x), softplus_fast(v[j + 1] + bb.y), softplus_fast(v[j + 2] + bb.z),
                                softplus_fast(v[j + 3] + bb.w));
            }
        } else {
            for (int j = 0; j < n; ++j) dst[j] = softplus_fast(v[j] + bias[j]);
        }
        return;
    }
    if (e.kind == EPI_OUT) {
        if (e.res_mode == 1) {
            const T* src = e.res_x + (long long)r * e.N + c0;
            for (int j = 0; j < n; ++j) v[j] += to_f(src[j]);
        } else if (e.res_mode == 2) {
            int b = r / e.Tp, t = r % e.Tp;
            if (t < e.n_meta) {
                if (e.res_meta_bf16) {
                    const bf16* src = static_cast<const bf16*>(e.res_meta) + (long long)t * e.N + c0;
                    for (int j = 0; j < n; ++j) v[j] += to_f(src[j]);
                } else {
                    const T* src = static_cast<const T*>(e.res_meta) + (long long)t * e.N + c0;
                    for (int j = 0; j < n; ++j) v[j] += to_f(src[j]);
                }
            } else {
                const T* src = e.res_x + ((long long)b * e.Tu + (t - e.n_meta)) * e.N + c0;
                for (int j = 0; j < n; ++j) v[j] += to_f(src[j]);
            }
        }
        store_run<T>(e.y + (long long)r * e.N + c0, v, n);
        return;
    }
    // EPI_INPROJ
    int b0, b1, t;
    if (mode == ROWS_DIRECT) { b0 = r / e.Tp; b1 = b0 + 1; t = r % e.Tp; }
    else if (mode == ROWS_META) { b0 = 0; b1 = e.B; t = r; }
    else if (mode == ROWS_USER) { b0 = r / e.Tu; b1 = b0 + 1; t = e.n_meta + r % e.Tu; }
    else {
        b0 = r; b1 = r + 1; t = e.pos[r] + e.pos_offset;
        if (t < 0) return;  // no position to write; the decode attention reports the range error
    }
    const int qw = e.H * e.dh;
    const int kw = e.k_out ? e.G * e.dh : 0;
    const int vw = e.k_out ? e.G * e.dv : 0;
    if (c0 < qw + kw) {
        if (mode == ROWS_DECODE) {
            float2 cs[32];
#pragma unroll 4
            for (int i = 0; i < 32; ++i) cs[i] = rope_cs_at(t, i, 64, e.rope_base);
            rope_run64(v, cs);
        } else {
            rope_run64(v, e.rope + (long long)t * 32);
        }
    }
    for (int b = b0; b < b1; ++b) {
        if (c0 >= qw && c0 < qw + kw) {
            int g = (c0 - qw) / e.dh;
            int slot = t;
            if (mode == ROWS_DECODE && t >= e.n_meta) slot = e.n_meta + (t - e.n_meta) % e.n_meta_ring;
            store_run<T>(e.k_out + (((long long)b * e.G + g) * e.kcap + slot) * e.dh, v, 64);
        } else if (c0 >= qw + kw && c0 < qw + kw + vw) {
            int cv = c0 - qw - kw;
            int g = cv / e.dv, off = cv % e.dv;
            int slot = t;
            if (mode == ROWS_DECODE && t >= e.n_meta) slot = e.n_meta + (t - e.n_meta) % e.n_meta_ring;
            store_run<T>(e.v_out + (((long long)b * e.G + g) * e.kcap + slot) * e.dv + off, v, 64);
        } else {
            long long row = mode == ROWS_DECODE ? b : (long long)b * e.Tp + t;
            store_run<T>(e.P + row * e.ldP + c0, v, n);
        }
    }
}

}  // namespace hymba
