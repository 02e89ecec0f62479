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

// Merge weights of a row's split partials (layout [row, head, split, dv + 4]: dv sums,
// then the split's max logit and sum of weights): w[head][s] = exp2(m_s - M) / den with
// M = max_s m_s and den = sum_s exp2(m_s - M) l_s, formed once per (row, head) by the
// block into shared memory (zero for a head that saw no key).
__device__ __forceinline__ void merge_weights(const float* __restrict__ part, int n_split, int H, int dv,
                                              long long row, float* wts, int t, int nthreads) {
    // one warp per head, one lane per split (in rounds of 32 splits)
    const int warp = t >> 5, lane = t & 31, nwarps = nthreads >> 5;
    for (int hd = warp; hd < H; hd += nwarps) {
        const float* base = part + ((long long)row * H + hd) * n_split * (dv + 4) + dv;
        float M = -INFINITY;
        for (int s = lane; s < n_split; s += 32) M = fmaxf(M, base[s * (dv + 4)]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float den = 0.f;
        for (int s = lane; s < n_split; s += 32) {
            const float w = M != -INFINITY ? exp2f(base[s * (dv + 4)] - M) : 0.f;
            wts[hd * n_split + s] = w;
            den = fmaf(w, base[s * (dv + 4) + 1], den);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        const float inv = den > 0.f ? 1.f / den : 0.f;
        for (int s = lane; s < n_split; s += 32) wts[hd * n_split + s] *= inv;
    }
}

// Attention output piece c..c+7 of row `row`: the weighted sum of its head's split
// partials (the loads of four splits in flight at a time).
__device__ __forceinline__ void merge8(const float* __restrict__ part, int n_split, int H, int dv,
                                       long long row, int c, const float* wts, float* o) {
    const int hd = c / dv, e = c - hd * dv;
    const float* base = part + ((long long)row * H + hd) * n_split * (dv + 4) + e;
    const float* w = wts + hd * n_split;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = 0.f;
    int s = 0;
    for (; s + 4 <= n_split; s += 4) {
        float4 v[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            // records of dv + 4 floats start on 16-byte boundaries
            const float4* ps = reinterpret_cast<const float4*>(base + (s + u) * (dv + 4));
            v[u][0] = ps[0];
            v[u][1] = ps[1];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float wu = w[s + u];
            o[0] = fmaf(wu, v[u][0].x, o[0]); o[1] = fmaf(wu, v[u][0].y, o[1]);
            o[2] = fmaf(wu, v[u][0].z, o[2]); o[3] = fmaf(wu, v[u][0].w, o[3]);
            o[4] = fmaf(wu, v[u][1].x, o[4]); o[5] = fmaf(wu, v[u][1].y, o[5]);
            o[6] = fmaf(wu, v[u][1].z, o[6]); o[7] = fmaf(wu, v[u][1].w, o[7]);
        }
    }
    for (; s < n_split; ++s) {
        const float* ps = base + s * (dv + 4);
        const float wu = w[s];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = fmaf(wu, ps[i], o[i]);
    }
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
            int rep, T* __restrict__ U, int rows, int di, float eps, int* len_inc, float* __restrict__ y_init,
            const float* __restrict__ y_res, int d_model) {
    griddep_sync();
    __shared__ float red[RPB][TPR / 32][2];
    extern __shared__ float merge_wts[];  // SPLIT: [H, n_split] merge weights of the row
    const int sub = threadIdx.x / TPR, t = threadIdx.x % TPR;
    const long long row = (long long)blockIdx.x * RPB + sub;
    const bool live = row < rows;
    if constexpr (SPLIT) {
        if (live) merge_weights(part, n_split, H, dv, row, merge_wts, t, TPR);
        __syncthreads();
    }
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
                merge8(part, n_split, H, dv, row, c, merge_wts, o[k]);
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
    // the output projection that follows adds its split-K partial sums to y: y starts as
    // the residual (or zero), unless y is the residual itself
    if (y_init && live && y_init != y_res)
        for (int c = t; c < d_model; c += TPR)
            y_init[row * d_model + c] = y_res ? y_res[row * d_model + c] : 0.f;
}

constexpr int RT = 512;                 // prefill fusion: threads per row (one 8-channel piece each)

__device__ __forceinline__ void cp_async16_own(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
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

// Prefill fusion, persistent over rows: block b takes rows b, b + grid, ... and each
// thread copies its own pieces of the next three rows (O, y_pre, z: 16-byte cp.async into
// a four-slot shared-memory ring that only it reads) before working on the current one, so
// every block keeps three rows of loads in flight through its reductions and stores (a row
// kernel that loads, reduces and stores in turn leaves HBM idle while it reduces). The
// per-channel factors beta * gain (halved for the average) of a thread's columns are
// formed once, in registers; the gated Mamba branch stays in fp32 between the passes.
// One piece of 8 channels per thread and branch (widths up to 8 * RT).
constexpr int RSLOT = 4;  // ring slots: the current row and three in flight

template <typename I, typename T, bool CONCAT>
__global__ void __launch_bounds__(RT, 1)
fuse_rows_kernel(const I* __restrict__ O, int H, int dv, const I* __restrict__ ypre, const I* __restrict__ P,
                 long long ldP, int col_z, const float* __restrict__ g_attn, const float* __restrict__ g_ssm,
                 const float* __restrict__ beta1, const float* __restrict__ beta2, const float* __restrict__ v_scale,
                 const float* __restrict__ v_bias, int rep, T* __restrict__ U, long long rows, int di, float eps) {
    constexpr int PW = sizeof(I) / 2;  // 16-byte words per piece
    extern __shared__ uint4 ring[];    // [RSLOT][3 arrays][PW][RT]
    __shared__ float red[2][RT / 32][2];
    griddep_sync();
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int hv = H * dv, nvo = hv / 8, nvy = di / 8;
    const int c = t * 8;
    const bool has_o = t < nvo, has_y = t < nvy;
    const float half = CONCAT ? 1.0f : 0.5f;  // the average halves both branches
    // this thread's columns are the same in every row: their factors stay in registers
    float fa[8], fs[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        fa[i] = has_o ? half * beta1[c + i] * g_attn[c + i] : 0.f;
        fs[i] = has_y ? half * beta2[c + i] * g_ssm[c + i] : 0.f;
    }
    const int vidx = has_o ? (c / dv / rep) * dv + (c % dv) : 0;  // a consumer's V transform entries
    const long long ldu = CONCAT ? (long long)di + hv : di;
    auto slot = [&](int sl, int arr, int w) -> uint4* { return ring + ((sl * 3 + arr) * PW + w) * RT + t; };
    auto issue = [&](long long r, int sl) {
        if (r < rows) {
#pragma unroll
            for (int w = 0; w < PW; ++w) {
                if (has_o) cp_async16_own(slot(sl, 0, w), O + r * hv + c + 8 / PW * w);
                if (has_y) {
                    cp_async16_own(slot(sl, 1, w), ypre + r * di + c + 8 / PW * w);
                    cp_async16_own(slot(sl, 2, w), P + r * ldP + col_z + c + 8 / PW * w);
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    auto fetch = [&](int sl, int arr, float* v) {
        Piece<I> pc;
#pragma unroll
        for (int w = 0; w < PW; ++w) pc.v[w] = *slot(sl, arr, w);
        unpack_piece<I>(pc, v);
    };
    long long row = blockIdx.x;
    for (int k = 0; k < RSLOT - 1; ++k) issue(row + (long long)k * gridDim.x, k);
    for (int it = 0; row < rows; ++it, row += gridDim.x) {
        const int sl = it % RSLOT;
        issue(row + (long long)(RSLOT - 1) * gridDim.x, (it + RSLOT - 1) % RSLOT);
        // this thread's copies of `row` have landed (the RSLOT - 1 later groups may still fly)
        asm volatile("cp.async.wait_group %0;" ::"n"(RSLOT - 1) : "memory");
        // pass 1: the consumer's V transform, the gate, both sums of squares
        float o[8], yg[8];
        float ss_o = 0.f, ss_y = 0.f;
        if (has_o) {
            fetch(sl, 0, o);
            if (v_scale) {
                // attention over V * s + b is the attention output * s + b (weights sum to 1)
                float vs[8], vb[8];
                load8f(v_scale + vidx, vs);
                load8f(v_bias + vidx, vb);
#pragma unroll
                for (int i = 0; i < 8; ++i) o[i] = fmaf(o[i], vs[i], vb[i]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) ss_o = fmaf(o[i], o[i], ss_o);
        }
        if (has_y) {
            float z[8];
            fetch(sl, 1, yg);
            fetch(sl, 2, z);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                yg[i] *= __fdividef(z[i], 1.0f + __expf(-z[i]));
                ss_y = fmaf(yg[i], yg[i], ss_y);
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
        for (int w = 0; w < RT / 32; ++w) {
            ss_o += red[it & 1][w][0];
            ss_y += red[it & 1][w][1];
        }
        const float ro = rsqrtf(ss_o / hv + eps);
        const float ry = rsqrtf(ss_y / di + eps);
        // pass 2: scale, combine, store
        if constexpr (CONCAT) {
            if (has_y) {
                float u[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] = fs[i] * yg[i] * ry;
                store8<T>(U + row * ldu + c, u);
            }
            if (has_o) {
                float u[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] = fa[i] * o[i] * ro;
                store8<T>(U + row * ldu + di + c, u);
            }
        } else if (has_y) {
            float u[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] = fmaf(fa[i] * ro, o[i], fs[i] * ry * yg[i]);
            store8<T>(U + row * ldu + c, u);
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

}  // namespace

template <typename I, typename T, bool CONCAT>
static int fuse_variant(const Ctx& ctx, const I* O, const float* part, int n_split, int H, int dv, int G,
                        const I* ypre, const I* P, long long ldP, int col_z, const float* g_attn, const float* g_ssm,
                        const float* beta1, const float* beta2, const float* v_scale, const float* v_bias, T* U,
                        int rows, int di, float eps, int* len_inc, float* y_init, const float* y_res, int d_model) {
    if (part) {
        auto kern = fuse_kernel<I, T, true, CONCAT>;
        const size_t smem = (size_t)H * n_split * sizeof(float);
        static std::atomic<unsigned long long> smem_set{0};
        if (smem > 48 * 1024 && !smem_opt_in_once(smem_set, kern, smem, ctx)) return HYMBA_ERR_CUDA;
        HYMBA_LAUNCH(ctx, "fuse", kern, ceil_div(rows, RPB), TPR * RPB, smem, O, part, n_split, H, dv, ypre, P, ldP,
                     col_z, g_attn, g_ssm, beta1, beta2, v_scale, v_bias, H / G, U, rows, di, eps, len_inc, y_init,
                     y_res, d_model);
    } else {
        auto kern = fuse_rows_kernel<I, T, CONCAT>;
        const size_t smem = (size_t)RSLOT * 3 * RT * sizeof(I) * 8;
        static std::atomic<unsigned long long> smem_set{0};
        if (!smem_opt_in_once(smem_set, kern, smem, ctx)) return HYMBA_ERR_CUDA;
        const int grid = (int)std::min<long long>(rows, ctx.sm_count > 0 ? ctx.sm_count : 148);
        HYMBA_LAUNCH(ctx, "fuse", kern, grid, RT, smem, O, H, dv, ypre, P, ldP, col_z, g_attn, g_ssm, beta1, beta2,
                     v_scale, v_bias, H / G, U, (long long)rows, di, eps);
    }
    return HYMBA_OK;
}

template <typename I, typename T>
int launch_fuse(const Ctx& ctx, const I* O, const float* part, int n_split, int H, int G, int dv, bool concat,
                const I* ypre, const I* P, long long ldP, int col_z, const float* g_attn, const float* g_ssm,
                const float* beta1, const float* beta2, const float* v_scale, const float* v_bias, T* U, int rows,
                int di, float eps, int* len_inc, float* y_init, const float* y_res, int d_model) {
    if (rows <= 0) return HYMBA_OK;
    if (y_init && (!part || d_model <= 0)) return HYMBA_ERR_UNSUPPORTED;
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
                                        beta2, v_scale, v_bias, U, rows, di, eps, len_inc, y_init, y_res, d_model);
    return fuse_variant<I, T, false>(ctx, O, part, n_split, H, dv, G, ypre, P, ldP, col_z, g_attn, g_ssm, beta1,
                                     beta2, v_scale, v_bias, U, rows, di, eps, len_inc, y_init, y_res, d_model);
}

#define HYMBA_FUSE_INST(I, T)                                                                                  \
    template int launch_fuse<I, T>(const Ctx&, const I*, const float*, int, int, int, int, bool, const I*, const I*, \
                                   long long, int, const float*, const float*, const float*, const float*,          \
                                   const float*, const float*, T*, int, int, float, int*, float*, const float*, \
                                   int);
HYMBA_FUSE_INST(float, float)
HYMBA_FUSE_INST(f16, bf16)
HYMBA_FUSE_INST(f16, f16)

}  // namespace hymba
