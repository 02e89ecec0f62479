// Fusion epilogue of the two head families: SiLU(z) gate of the Mamba branch,
// RMSNorm of each branch over its full width, beta1 / beta2 scaling and average:
//     Y = y_pre * SiLU(z),  U = (beta1 * g_a * O / rms(O) + beta2 * g_s * Y / rms(Y)) / 2
// ("Hymba Guide", Parallel Hybrid-Head Layer Formulation: both families feed one
// output projection; normalise-scale-average is the reading used for how they are
// combined). HBM-bound: per (row, channel) it reads O, y_pre and z and writes U once.
//
// One row per 256-thread block; each thread keeps its (at most two) 8-element pieces
// of the row in registers between the two passes (sums of squares, then the output),
// moving 8 elements per 16-byte access. Few registers per thread keep many rows in
// flight per SM, which is what an HBM-bound row kernel needs.
//
// Decode variant (SPLIT): the attention output arrives as the split-KV partials of the
// decode attention (per head and key split: unnormalised sum of p v, the split's
// max logit and sum of p) and is merged here, piece by piece, with the usual
// rescaling by exp2(m_s - max_s m_s).
#include "kernels.h"

namespace hymba {

namespace {

constexpr int TPR = 256;                // threads per row
constexpr int RPB = 1;                  // rows per block
constexpr int VMAX = 2;                 // 8-element vectors per thread and array (d_inner <= 4096)

template <typename I>
__device__ __forceinline__ void load8(const I* p, float* v) {
    if constexpr (sizeof(I) == 2) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const I* h = reinterpret_cast<const I*>(&u);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = to_f(h[i]);
    } else {
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

template <typename T>
__device__ __forceinline__ void store8(T* p, const float* v) {
    if constexpr (sizeof(T) == 2) {
        uint4 u;
        u.x = pack2<T>(v[0], v[1]);
        u.y = pack2<T>(v[2], v[3]);
        u.z = pack2<T>(v[4], v[5]);
        u.w = pack2<T>(v[6], v[7]);
        *reinterpret_cast<uint4*>(p) = u;
    } else {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
}

__device__ __forceinline__ void load8f(const float* p, float* v) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Attention output piece c..c+7 of row `row` merged from its head's split partials
// (layout [row, head, split, dv + 2]: dv sums, then max logit and sum of weights).
__device__ __forceinline__ void merge8(const float* __restrict__ part, int n_split, int H, int dv,
                                       long long row, int c, float* o) {
    const int hd = c / dv, e = c - hd * dv;
    const float* base = part + ((long long)row * H + hd) * n_split * (dv + 2);
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, base[s * (dv + 2) + dv]);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = 0.f;
    float den = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < n_split; ++s) {
            const float* ps = base + s * (dv + 2);
            const float w = exp2f(ps[dv] - M);
            den = fmaf(w, ps[dv + 1], den);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 v = *reinterpret_cast<const float2*>(ps + e + 2 * i);
                o[2 * i] = fmaf(w, v.x, o[2 * i]);
                o[2 * i + 1] = fmaf(w, v.y, o[2 * i + 1]);
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] *= inv;
}

// (the decode variant runs one block per sequence, so it asks for no more than one
// block per SM and keeps its merge temporaries in registers)
// CONCAT: U = [beta2 * RMS(Y) | beta1 * RMS(O)] (d_inner + H * dv wide) instead of the
// average (O and Y of equal width d_inner).
template <typename I, typename T, bool SPLIT, bool CONCAT>
__global__ void __launch_bounds__(TPR * RPB, SPLIT ? 1 : 4)
fuse_kernel(const I* __restrict__ O, const float* __restrict__ part, int n_split, int H, int dv,
            const I* __restrict__ ypre, const I* __restrict__ P, long long ldP, int col_z,
            const float* __restrict__ g_attn, const float* __restrict__ g_ssm, const float* __restrict__ beta1,
            const float* __restrict__ beta2, const float* __restrict__ v_scale, const float* __restrict__ v_bias,
            int rep, T* __restrict__ U, int rows, int di, float eps, int* len_inc) {
    griddep_sync();
    __shared__ float red[RPB][TPR / 32][2];
    const int sub = threadIdx.x / TPR, t = threadIdx.x % TPR;
    const long long row = (long long)blockIdx.x * RPB + sub;
    const bool live = row < rows;
    const int hv = H * dv;                 // attention branch width
    const int nvo = hv / 8, nvy = di / 8;  // pieces of 8 per branch
    float o[VMAX][8], y[VMAX][8];
    float ss_o = 0.f, ss_y = 0.f;
#pragma unroll
    for (int k = 0; k < VMAX; ++k) {
        const int vi = t + k * TPR;
        if (live && vi < nvo) {
            const int c = vi * 8;
            if constexpr (SPLIT)
                merge8(part, n_split, H, dv, row, c, o[k]);
            else
                load8<I>(O + row * hv + c, o[k]);
            if (v_scale) {
                // a consumer's adapted shared V: attention over V * s + b is the attention
                // output * s + b (the softmax weights sum to 1)
                const int hd = c / dv;
                const int idx = (hd / rep) * dv + (c - hd * dv);
                float vs[8], vb[8];
                load8f(v_scale + idx, vs);
                load8f(v_bias + idx, vb);
#pragma unroll
                for (int i = 0; i < 8; ++i) o[k][i] = fmaf(o[k][i], vs[i], vb[i]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) ss_o = fmaf(o[k][i], o[k][i], ss_o);
        }
        if (live && vi < nvy) {
            const int c = vi * 8;
            float z[8];
            load8<I>(ypre + row * di + c, y[k]);
            load8<I>(P + row * ldP + col_z + c, z);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                y[k][i] *= z[i] / (1.0f + __expf(-z[i]));
                ss_y = fmaf(y[k][i], y[k][i], ss_y);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        ss_o += __shfl_xor_sync(0xffffffffu, ss_o, off);
        ss_y += __shfl_xor_sync(0xffffffffu, ss_y, off);
    }
    if ((t & 31) == 0) {
        red[sub][t >> 5][0] = ss_o;
        red[sub][t >> 5][1] = ss_y;
    }
    __syncthreads();
    ss_o = 0.f;
    ss_y = 0.f;
#pragma unroll
    for (int w = 0; w < TPR / 32; ++w) {
        ss_o += red[sub][w][0];
        ss_y += red[sub][w][1];
    }
    // the average halves both branches; the concatenation keeps them whole
    const float half = CONCAT ? 1.0f : 0.5f;
    const float ro = half / sqrtf(ss_o / hv + eps);
    const float ry = half / sqrtf(ss_y / di + eps);
#pragma unroll
    for (int k = 0; k < VMAX; ++k) {
        const int vi = t + k * TPR;
        if constexpr (CONCAT) {
            const long long ldu = di + hv;
            if (live && vi < nvy) {
                const int c = vi * 8;
                float gs[8], b2[8], u[8];
                load8f(g_ssm + c, gs);
                load8f(beta2 + c, b2);
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] = b2[i] * gs[i] * y[k][i] * ry;
                store8<T>(U + row * ldu + c, u);
            }
            if (live && vi < nvo) {
                const int c = vi * 8;
                float ga[8], b1[8], u[8];
                load8f(g_attn + c, ga);
                load8f(beta1 + c, b1);
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] = b1[i] * ga[i] * o[k][i] * ro;
                store8<T>(U + row * ldu + di + c, u);
            }
        } else {
            if (live && vi < nvy) {
                const int c = vi * 8;
                float ga[8], gs[8], b1[8], b2[8], u[8];
                load8f(g_attn + c, ga);
                load8f(g_ssm + c, gs);
                load8f(beta1 + c, b1);
                load8f(beta2 + c, b2);
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] = b1[i] * ga[i] * o[k][i] * ro + b2[i] * gs[i] * y[k][i] * ry;
                store8<T>(U + row * di + c, u);
            }
        }
    }
    if (len_inc && live && t == 0) len_inc[row] += 1;
}

// An 8-element piece of an input row as loaded (16-bit: one 16-byte word; fp32: two).
template <typename I>
struct Piece {
    uint4 v[sizeof(I) / 2];
};

template <typename I>
__device__ __forceinline__ void load_piece(Piece<I>& p, const I* src) {
#pragma unroll
    for (int i = 0; i < (int)(sizeof(I) / 2); ++i) p.v[i] = reinterpret_cast<const uint4*>(src)[i];
}

template <typename I>
__device__ __forceinline__ void unpack_piece(const Piece<I>& p, float* v) {
    if constexpr (sizeof(I) == 2) {
        const I* h = reinterpret_cast<const I*>(&p.v[0]);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = to_f(h[i]);
    } else {
        const float* f = reinterpret_cast<const float*>(&p.v[0]);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = f[i];
    }
}

template <typename I>
__device__ __forceinline__ void pack_piece(Piece<I>& p, const float* v) {
    if constexpr (sizeof(I) == 2) {
        p.v[0] = make_uint4(pack2<I>(v[0], v[1]), pack2<I>(v[2], v[3]), pack2<I>(v[4], v[5]), pack2<I>(v[6], v[7]));
    } else {
        p.v[0] = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
        p.v[1] = make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]), __float_as_uint(v[7]));
    }
}

// Prefill fusion, persistent over rows: block b takes rows b, b + grid, ... and loads the
// next row's pieces into registers before working on the current one, so every block
// keeps a row of loads in flight through its reductions and stores (a row kernel that
// loads, reduces and stores in turn leaves HBM idle while it reduces). The per-channel
// factors beta * gain (halved for the average) are formed once per block in shared
// memory. The gated Mamba branch is kept between the two passes in the intermediate
// type (fp16 for 16-bit layers: the normalised result is written as bf16 or fp16).
template <typename I, typename T, bool CONCAT>
__global__ void __launch_bounds__(TPR, 3)
fuse_rows_kernel(const I* __restrict__ O, int H, int dv, const I* __restrict__ ypre, const I* __restrict__ P,
                 long long ldP, int col_z, const float* __restrict__ g_attn, const float* __restrict__ g_ssm,
                 const float* __restrict__ beta1, const float* __restrict__ beta2, const float* __restrict__ v_scale,
                 const float* __restrict__ v_bias, int rep, T* __restrict__ U, long long rows, int di, float eps) {
    constexpr bool PF = sizeof(I) == 2;  // prefetch the next row (16-bit inputs: few registers per piece)
    extern __shared__ float fac[];        // [hv] attention factors, then [di] Mamba factors
    __shared__ float red[2][TPR / 32][2];
    griddep_sync();
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int hv = H * dv, nvo = hv / 8, nvy = di / 8;
    const float half = CONCAT ? 1.0f : 0.5f;  // the average halves both branches
    for (int c = t; c < hv; c += TPR) fac[c] = half * beta1[c] * g_attn[c];
    for (int c = t; c < di; c += TPR) fac[hv + c] = half * beta2[c] * g_ssm[c];
    __syncthreads();
    const long long ldu = CONCAT ? (long long)di + hv : di;

    Piece<I> po[VMAX], py[VMAX], pz[VMAX];
    auto load_row = [&](long long r, Piece<I>* a, Piece<I>* b, Piece<I>* z) {
#pragma unroll
        for (int k = 0; k < VMAX; ++k) {
            const int vi = t + k * TPR;
            if (vi < nvo) load_piece<I>(a[k], O + r * hv + vi * 8);
            if (vi < nvy) {
                load_piece<I>(b[k], ypre + r * di + vi * 8);
                load_piece<I>(z[k], P + r * ldP + col_z + vi * 8);
            }
        }
    };
    long long row = blockIdx.x;
    if (PF && row < rows) load_row(row, po, py, pz);
    for (int it = 0; row < rows; ++it, row += gridDim.x) {
        Piece<I> no[VMAX], ny[VMAX], nz[VMAX];
        const long long nrow = row + gridDim.x;
        if (PF) {
            if (nrow < rows) load_row(nrow, no, ny, nz);
        } else {
            load_row(row, po, py, pz);
        }
        // pass 1: the consumer's V transform, the gate, both sums of squares
        float ss_o = 0.f, ss_y = 0.f;
#pragma unroll
        for (int k = 0; k < VMAX; ++k) {
            const int vi = t + k * TPR;
            if (vi < nvo) {
                float o[8];
                unpack_piece<I>(po[k], o);
                if (v_scale) {
                    // attention over V * s + b is the attention output * s + b (weights sum to 1)
                    const int c = vi * 8, hd = c / dv;
                    const int idx = (hd / rep) * dv + (c - hd * dv);
                    float vs[8], vb[8];
                    load8f(v_scale + idx, vs);
                    load8f(v_bias + idx, vb);
#pragma unroll
                    for (int i = 0; i < 8; ++i) o[i] = fmaf(o[i], vs[i], vb[i]);
                    pack_piece<I>(po[k], o);
                    unpack_piece<I>(po[k], o);  // normalise what is kept
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) ss_o = fmaf(o[i], o[i], ss_o);
            }
            if (vi < nvy) {
                float y[8], z[8];
                unpack_piece<I>(py[k], y);
                unpack_piece<I>(pz[k], z);
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] *= z[i] / (1.0f + __expf(-z[i]));
                pack_piece<I>(py[k], y);
                unpack_piece<I>(py[k], y);
#pragma unroll
                for (int i = 0; i < 8; ++i) ss_y = fmaf(y[i], y[i], ss_y);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            ss_o += __shfl_xor_sync(0xffffffffu, ss_o, off);
            ss_y += __shfl_xor_sync(0xffffffffu, ss_y, off);
        }
        if (lane == 0) {
            red[it & 1][warp][0] = ss_o;
            red[it & 1][warp][1] = ss_y;
        }
        __syncthreads();  // (the other buffer was last read before the previous barrier)
        ss_o = 0.f;
        ss_y = 0.f;
#pragma unroll
        for (int w = 0; w < TPR / 32; ++w) {
            ss_o += red[it & 1][w][0];
            ss_y += red[it & 1][w][1];
        }
        const float ro = rsqrtf(ss_o / hv + eps);
        const float ry = rsqrtf(ss_y / di + eps);
        // pass 2: scale, combine, store
#pragma unroll
        for (int k = 0; k < VMAX; ++k) {
            const int vi = t + k * TPR;
            const int c = vi * 8;
            if constexpr (CONCAT) {
                if (vi < nvy) {
                    float y[8], u[8];
                    unpack_piece<I>(py[k], y);
#pragma unroll
                    for (int i = 0; i < 8; ++i) u[i] = fac[hv + c + i] * y[i] * ry;
                    store8<T>(U + row * ldu + c, u);
                }
                if (vi < nvo) {
                    float o[8], u[8];
                    unpack_piece<I>(po[k], o);
#pragma unroll
                    for (int i = 0; i < 8; ++i) u[i] = fac[c + i] * o[i] * ro;
                    store8<T>(U + row * ldu + di + c, u);
                }
            } else if (vi < nvy) {
                float o[8], y[8], u[8];
                unpack_piece<I>(po[k], o);
                unpack_piece<I>(py[k], y);
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] = fmaf(fac[c + i] * ro, o[i], fac[hv + c + i] * ry * y[i]);
                store8<T>(U + row * ldu + c, u);
            }
        }
        if (PF) {
#pragma unroll
            for (int k = 0; k < VMAX; ++k) {
                po[k] = no[k];
                py[k] = ny[k];
                pz[k] = nz[k];
            }
        }
    }
}

}  // namespace

template <typename I, typename T, bool CONCAT>
static int fuse_variant(const Ctx& ctx, const I* O, const float* part, int n_split, int H, int dv, int G,
                        const I* ypre, const I* P, long long ldP, int col_z, const float* g_attn, const float* g_ssm,
                        const float* beta1, const float* beta2, const float* v_scale, const float* v_bias, T* U,
                        int rows, int di, float eps, int* len_inc) {
    if (part) {
        auto kern = fuse_kernel<I, T, true, CONCAT>;
        HYMBA_LAUNCH(ctx, "fuse", kern, ceil_div(rows, RPB), TPR * RPB, 0, O, part, n_split, H, dv, ypre, P, ldP,
                     col_z, g_attn, g_ssm, beta1, beta2, v_scale, v_bias, H / G, U, rows, di, eps, len_inc);
    } else {
        auto kern = fuse_rows_kernel<I, T, CONCAT>;
        const size_t smem = (size_t)(H * dv + di) * sizeof(float);
        static std::atomic<unsigned long long> smem_set{0};
        if (smem > 48 * 1024 && !smem_opt_in_once(smem_set, kern, smem, ctx)) return HYMBA_ERR_CUDA;
        const int grid = (int)std::min<long long>(rows, 3LL * (ctx.sm_count > 0 ? ctx.sm_count : 148));
        HYMBA_LAUNCH(ctx, "fuse", kern, grid, TPR, smem, O, H, dv, ypre, P, ldP, col_z, g_attn, g_ssm, beta1, beta2,
                     v_scale, v_bias, H / G, U, (long long)rows, di, eps);
    }
    return HYMBA_OK;
}

template <typename I, typename T>
int launch_fuse(const Ctx& ctx, const I* O, const float* part, int n_split, int H, int G, int dv, bool concat,
                const I* ypre, const I* P, long long ldP, int col_z, const float* g_attn, const float* g_ssm,
                const float* beta1, const float* beta2, const float* v_scale, const float* v_bias, T* U, int rows,
                int di, float eps, int* len_inc) {
    if (rows <= 0) return HYMBA_OK;
    const int hv = H * dv;
    if (di % 8 || di > VMAX * 8 * TPR || hv > VMAX * 8 * TPR || col_z % 8 || ldP % 8) return HYMBA_ERR_UNSUPPORTED;
    // pieces of 8 never straddle a head
    if (H <= 0 || G <= 0 || H % G || dv % 8 || (!concat && hv != di)) return HYMBA_ERR_UNSUPPORTED;
    if ((v_scale == nullptr) != (v_bias == nullptr) ||
        ((reinterpret_cast<uintptr_t>(v_scale) | reinterpret_cast<uintptr_t>(v_bias)) & 15))
        return HYMBA_ERR_UNSUPPORTED;
    // 8-byte loads of the partial sums
    if (part && (n_split <= 0 || (reinterpret_cast<uintptr_t>(part) & 7))) return HYMBA_ERR_UNSUPPORTED;
    if (concat)
        return fuse_variant<I, T, true>(ctx, O, part, n_split, H, dv, G, ypre, P, ldP, col_z, g_attn, g_ssm, beta1,
                                        beta2, v_scale, v_bias, U, rows, di, eps, len_inc);
    return fuse_variant<I, T, false>(ctx, O, part, n_split, H, dv, G, ypre, P, ldP, col_z, g_attn, g_ssm, beta1,
                                     beta2, v_scale, v_bias, U, rows, di, eps, len_inc);
}

#define HYMBA_FUSE_INST(I, T)                                                                                  \
    template int launch_fuse<I, T>(const Ctx&, const I*, const float*, int, int, int, int, bool, const I*, const I*, \
                                   long long, int, const float*, const float*, const float*, const float*,          \
                                   const float*, const float*, T*, int, int, float, int*);
HYMBA_FUSE_INST(float, float)
HYMBA_FUSE_INST(f16, bf16)
HYMBA_FUSE_INST(f16, f16)

}  // namespace hymba
