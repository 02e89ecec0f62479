// Epilogues of the three projections of a mixer layer. Every GEMM of the library
// (SIMT or tcgen05) hands its fp32 accumulators to epi_run64 in runs of 64
// consecutive output columns of one output row, so that RoPE (pairs i, i+32 of a
// 64-wide head) and the per-head scatter of K and V happen before rounding.
#pragma once
#include "common.cuh"

namespace hymba {

enum EpiKind { EPI_INPROJ = 0, EPI_DELTA = 1, EPI_OUT = 2, EPI_GLU = 3 };

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
    const float2* rope;    // prefill: [T', dh/2] (cos, sin) of position * theta_i; decode: [B, dh/2] for
                           // each sequence's new position (computed on the fly when null)
    const int* pos;        // decode: [B] positions held (len); the new token sits at pos[b] + pos_offset
    int pos_offset;        // decode: 0 for a producer (appends), -1 for a consumer
    int n_meta_ring;       // decode: ring length (cache_cap - n_meta)
    float rope_base;       // decode: angles computed on the fly
    const float* q_scale;  // consumer with an adapted shared K: [G, dh] scales applied to the
                           // queries of each KV head's group after RoPE (NULL: none)
    // EPI_DELTA
    float* delta;          // [M, N] fp32
    const float* b_dt;
    // EPI_OUT
    T* y;                  // [M, N]
    int res_mode;          // 0: none; 1: residual = res_x row r; 2: residual = X^ row (meta or user)
    const T* res_x;
    const void* res_meta;  // [n_meta, N] of the layer's weight type
    int res_meta_bf16;     // 1: res_meta is bf16; 0: it has type T
    // EPI_GLU: y = SiLU(gate) * (this GEMM's result), gate [M, N] of type T
    const T* glu_gate;
    // EPI_OUT into fp32 with accumulate = 1: the run is added to y (red.global.add) instead
    // of stored, no residual (split-K partial sums; y holds the residual beforehand)
    int accumulate;
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

// v[0..n) += the residual run at src (16-byte loads when the run is full and aligned);
// every index into v is a compile-time constant, so v stays in registers
template <typename S>
__device__ __forceinline__ void add_residual64(float* v, const S* src, int n) {
    constexpr int PER = 16 / (int)sizeof(S);
    if (n == 64 && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
#pragma unroll
        for (int j = 0; j < 64; j += PER) {
            const uint4 u = *reinterpret_cast<const uint4*>(src + j);
            const S* q = reinterpret_cast<const S*>(&u);
#pragma unroll
            for (int k = 0; k < PER; ++k) v[j + k] += to_f(q[k]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 64; ++j)
            if (j < n) v[j] += to_f(src[j]);
    }
}

// Where one row's run of (up to) 64 output columns goes: `count` copies `stride` bytes
// apart (a meta row of the in-projection is written once per sequence), `nbytes` valid
// bytes of elements of `esz` bytes (fp32 Delta, otherwise the output type).
struct RunDst {
    char* p;
    long long stride;
    int count;
    int nbytes;
    int esz;
    int add;   // fp32 runs only: accumulate into the destination
};

// Everything the epilogue does to one run except the store: bias + softplus (Delta),
// residual (output projection), RoPE (Q and K of the in-projection), and the run's
// destination. count = 0 when the row has nothing to write. KIND >= 0 fixes the
// epilogue kind at compile time (the kernel then holds that kind's code only);
// KIND < 0 reads it from e.kind. DEC fixes the decode form as well: decode rows and no
// meta rows (in-projection), split-K partial sums (output projection).
template <typename T, int KIND = -1, bool DEC = false>
__device__ __forceinline__ RunDst epi_prepare64(const EpiArgs<T>& e, int r, int c0, float* v) {
    const int kind = KIND >= 0 ? KIND : e.kind;
    // the element size depends on the launch only (the staged store relies on it being
    // the same in every lane, rows without output included)
    RunDst d{nullptr, 0, 0, 0, kind == EPI_DELTA ? 4 : (int)sizeof(T), 0};
    int mode = DEC ? (int)ROWS_DECODE : e.row_mode, M = e.M;
    if (!DEC && e.meta_pad > 0) {
        if (r < e.meta_pad) {
            mode = ROWS_META;
            M = e.meta_M;
        } else {
            r -= e.meta_pad;
        }
    }
    if (r >= M || c0 >= e.N) return d;
    const int n = min(64, e.N - c0);
    if (kind == EPI_DELTA) {
        const float* bias = e.b_dt + c0;
        if (n == 64 && (e.N & 3) == 0) {
            float4 bb[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) bb[j] = reinterpret_cast<const float4*>(bias)[j];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                v[4 * j] = softplus_fast(v[4 * j] + bb[j].x);
                v[4 * j + 1] = softplus_fast(v[4 * j + 1] + bb[j].y);
                v[4 * j + 2] = softplus_fast(v[4 * j + 2] + bb[j].z);
                v[4 * j + 3] = softplus_fast(v[4 * j + 3] + bb[j].w);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j)
                if (j < n) v[j] = softplus_fast(v[j] + bias[j]);
        }
        d.p = reinterpret_cast<char*>(e.delta + (long long)r * e.N + c0);
        d.count = 1;
        d.nbytes = n * 4;
        return d;
    }
    if (kind == EPI_GLU) {
        // the gated MLP: SiLU of the gate projection (same row and columns) times this one
        float gv[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) gv[j] = 0.f;
        add_residual64(gv, e.glu_gate + (long long)r * e.N + c0, n);
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] *= silu_f(gv[j]);
        d.p = reinterpret_cast<char*>(e.y + (long long)r * e.N + c0);
        d.count = 1;
        d.nbytes = n * (int)sizeof(T);
        return d;
    }
    if (kind == EPI_OUT) {
        if (DEC || e.accumulate) {
            d.p = reinterpret_cast<char*>(e.y + (long long)r * e.N + c0);
            d.count = 1;
            d.nbytes = n * (int)sizeof(T);
            d.add = 1;
            return d;
        }
        if (e.res_mode == 1) {
            add_residual64(v, e.res_x + (long long)r * e.N + c0, n);
        } else if (e.res_mode == 2) {
            int b = r / e.Tp, t = r % e.Tp;
            if (t < e.n_meta) {
                if (e.res_meta_bf16)
                    add_residual64(v, static_cast<const bf16*>(e.res_meta) + (long long)t * e.N + c0, n);
                else
                    add_residual64(v, static_cast<const T*>(e.res_meta) + (long long)t * e.N + c0, n);
            } else {
                add_residual64(v, e.res_x + ((long long)b * e.Tu + (t - e.n_meta)) * e.N + c0, n);
            }
        }
        d.p = reinterpret_cast<char*>(e.y + (long long)r * e.N + c0);
        d.count = 1;
        d.nbytes = n * (int)sizeof(T);
        return d;
    }
    // EPI_INPROJ
    int b0, b1, t;
    if (mode == ROWS_DIRECT) { b0 = r / e.Tp; b1 = b0 + 1; t = r % e.Tp; }
    else if (mode == ROWS_META) { b0 = 0; b1 = e.B; t = r; }
    else if (mode == ROWS_USER) { b0 = r / e.Tu; b1 = b0 + 1; t = e.n_meta + r % e.Tu; }
    else {
        b0 = r; b1 = r + 1; t = e.pos[r] + e.pos_offset;
        if (t < 0) return d;  // no position to write; the decode attention reports the range error
    }
    const int qw = e.H * e.dh;
    const int kw = e.k_out ? e.G * e.dh : 0;
    const int vw = e.k_out ? e.G * e.dv : 0;
    if (c0 < qw + kw) {
        if (mode == ROWS_DECODE) {
            if (e.rope) {
                rope_run64(v, e.rope + (long long)r * 32);  // the step's table, one row per sequence
            } else {
                float2 cs[32];
#pragma unroll 4
                for (int i = 0; i < 32; ++i) cs[i] = rope_cs_at(t, i, 64, e.rope_base);
                rope_run64(v, cs);
            }
        } else {
            rope_run64(v, e.rope + (long long)t * 32);
        }
        if (e.q_scale && c0 < qw) {
            // q . (k * s) = (q * s) . k: the K scale of the query's KV head moves onto q
            const float4* s4 = reinterpret_cast<const float4*>(e.q_scale + (c0 / e.dh) / (e.H / e.G) * e.dh);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float4 f = s4[j];
                v[4 * j] *= f.x;
                v[4 * j + 1] *= f.y;
                v[4 * j + 2] *= f.z;
                v[4 * j + 3] *= f.w;
            }
        }
    }
    d.count = b1 - b0;
    if (c0 >= qw && c0 < qw + kw) {
        const int g = (c0 - qw) / e.dh;
        int slot = t;
        if (mode == ROWS_DECODE && t >= e.n_meta) slot = e.n_meta + (t - e.n_meta) % e.n_meta_ring;
        d.p = reinterpret_cast<char*>(e.k_out + (((long long)b0 * e.G + g) * e.kcap + slot) * e.dh);
        d.stride = (long long)e.G * e.kcap * e.dh * (long long)sizeof(T);
        d.nbytes = 64 * (int)sizeof(T);
    } else if (c0 >= qw + kw && c0 < qw + kw + vw) {
        const int cv = c0 - qw - kw;
        const int g = cv / e.dv, off = cv % e.dv;
        int slot = t;
        if (mode == ROWS_DECODE && t >= e.n_meta) slot = e.n_meta + (t - e.n_meta) % e.n_meta_ring;
        d.p = reinterpret_cast<char*>(e.v_out + (((long long)b0 * e.G + g) * e.kcap + slot) * e.dv + off);
        d.stride = (long long)e.G * e.kcap * e.dv * (long long)sizeof(T);
        d.nbytes = 64 * (int)sizeof(T);
    } else {
        const long long row = mode == ROWS_DECODE ? b0 : (long long)b0 * e.Tp + t;
        d.p = reinterpret_cast<char*>(e.P + row * e.ldP + c0);
        d.stride = (long long)e.Tp * e.ldP * (long long)sizeof(T);
        d.nbytes = n * (int)sizeof(T);
    }
    return d;
}

// One thread stores its own row's run (CUDA-core GEMM).
template <typename T>
__device__ void epi_run64(const EpiArgs<T>& e, int r, int c0, float* v) {
    const RunDst d = epi_prepare64<T>(e, r, c0, v);
    for (int b = 0; b < d.count; ++b) {
        char* p = d.p + b * d.stride;
        if (d.add) {
            for (int j = 0; j < d.nbytes / 4; ++j) atomicAdd(reinterpret_cast<float*>(p) + j, v[j]);
            continue;
        }
        if (d.esz == 4) store_run<float>(reinterpret_cast<float*>(p), v, d.nbytes / 4);
        else store_run<T>(reinterpret_cast<T*>(p), v, d.nbytes / (int)sizeof(T));
    }
}

// Shared-memory staging of one warp's 32 rows: 128 bytes per row and unit, rows padded
// to 144 bytes so that both the per-row writes and the per-segment reads are free of
// bank conflicts.
constexpr int kStageRow = 144;
constexpr int kStageWarpBytes = 32 * kStageRow;

// Warp-collective store of the 32 rows' runs (lane l holds row l's values and RunDst):
// each 128-byte unit (32 fp32 or 64 16-bit values) goes through shared memory so that
// eight lanes write one row's 128 contiguous bytes with 16-byte stores, instead of each
// lane writing its own row (32 rows, 32 cache lines per store instruction).
template <typename T>
__device__ __forceinline__ void epi_store_staged(const RunDst& d, const float* v, uint8_t* stage, RunDst* info, int lane) {
    const int units = d.esz == 4 ? 2 : 1;  // esz is the same in every lane (one kind per launch)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (h >= units) break;
        uint4* srow = reinterpret_cast<uint4*>(stage + lane * kStageRow);
        if (d.esz == 4) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                srow[i] = make_uint4(__float_as_uint(v[h * 32 + 4 * i]), __float_as_uint(v[h * 32 + 4 * i + 1]),
                                     __float_as_uint(v[h * 32 + 4 * i + 2]), __float_as_uint(v[h * 32 + 4 * i + 3]));
        } else if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                srow[i] = make_uint4(pack2<T>(v[8 * i], v[8 * i + 1]), pack2<T>(v[8 * i + 2], v[8 * i + 3]),
                                     pack2<T>(v[8 * i + 4], v[8 * i + 5]), pack2<T>(v[8 * i + 6], v[8 * i + 7]));
        }
        RunDst di = d;
        di.p += h * 128;
        di.nbytes = min(max(d.nbytes - h * 128, 0), 128);
        if (di.nbytes == 0) di.count = 0;
        info[lane] = di;
        __syncwarp();
#pragma unroll 1
        for (int it = 0; it < 8; ++it) {
            const int row = it * 4 + (lane >> 3), off = (lane & 7) * 16;
            const RunDst ri = info[row];
            if (ri.count > 0 && off < ri.nbytes) {
                const uint4 val = *reinterpret_cast<const uint4*>(stage + row * kStageRow + off);
                const bool vec = off + 16 <= ri.nbytes && ((reinterpret_cast<uintptr_t>(ri.p) | (uintptr_t)ri.stride) & 15) == 0;
                for (int b = 0; b < ri.count; ++b) {
                    char* dst = ri.p + b * ri.stride + off;
                    if (ri.add) {
                        // split-K partial sums of an fp32 output
                        if (vec) {
                            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst),
                                         "f"(__uint_as_float(val.x)), "f"(__uint_as_float(val.y)),
                                         "f"(__uint_as_float(val.z)), "f"(__uint_as_float(val.w))
                                         : "memory");
                        } else {
                            const float* src = reinterpret_cast<const float*>(&val);
                            for (int k = 0; 4 * k < min(16, ri.nbytes - off); ++k)
                                atomicAdd(reinterpret_cast<float*>(dst) + k, src[k]);
                        }
                        continue;
                    }
                    if (vec) {
                        *reinterpret_cast<uint4*>(dst) = val;
                    } else {
                        const uint8_t* src = reinterpret_cast<const uint8_t*>(&val);
                        const int nb = min(16, ri.nbytes - off);
                        if (ri.esz == 4)
                            for (int k = 0; k < nb; k += 4)
                                *reinterpret_cast<uint32_t*>(dst + k) = *reinterpret_cast<const uint32_t*>(src + k);
                        else
                            for (int k = 0; k < nb; k += 2)
                                *reinterpret_cast<uint16_t*>(dst + k) = *reinterpret_cast<const uint16_t*>(src + k);
                    }
                }
            }
        }
        __syncwarp();
    }
}

}  // namespace hymba
