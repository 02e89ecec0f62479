// Fusion epilogue of the two head families: SiLU(z) gate of the Mamba branch,
// RMSNorm of each branch over its full width, beta1 / beta2 scaling and average:
//     Y = y_pre * SiLU(z),  U = (beta1 * g_a * O / rms(O) + beta2 * g_s * Y / rms(Y)) / 2
// ("Hymba Guide", Parallel Hybrid-Head Layer Formulation: both families feed one
// output projection; normalise-scale-average is the reading used for how they are
// combined). HBM-bound: per (row, channel) it reads O, y_pre and z and writes U once.
//
// Two kernels: the prefill one (persistent over rows, loads of the next rows in flight
// through each row's reductions) and the decode one (one thread-block cluster per row,
// merging the split partials of the decode attention); both keep a thread's pieces of a
// row in registers between the two passes (sums of squares, then the output) and move 8
// elements per 16-byte access.
#include "kernels.h"

namespace hymba {

namespace {

constexpr int kMaxWidth = 4096;         // widest branch (channels) either kernel takes

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

// Decode fusion: one thread-block cluster of FC CTAs per sequence row. CTA r of the
// cluster takes pieces [r * po, (r + 1) * po) of the attention branch (po = ceil(pieces /
// FC)) and likewise of the Mamba branch, one 8-channel piece per thread and branch. The
// attention pieces arrive as the split partials of the decode attention, layout [row,
// head, split, dv + 4] (dv sums of p v, then the split's max logit m_s and sum of p l_s),
// merged with the weights w_s = exp2(m_s - M) / sum_s exp2(m_s - M) l_s, M = max_s m_s.
// Every load of a thread (its first FSPL split records, y_pre and z, its heads' (m_s, l_s))
// is issued before the first barrier. The two sums of squares of the row meet across the
// cluster through distributed shared memory: each CTA publishes its partial sums, and
// after a cluster barrier reads the other CTAs' from their shared memory.
constexpr int FC = 8;    // CTAs per row (cluster size)
constexpr int FT = 64;   // threads per CTA
constexpr int FSPL = 16;  // split records per piece loaded ahead of the merge weights
constexpr int FYI = 4;    // residual values per thread loaded ahead (y_init)
static_assert(FC * FT * 8 >= kMaxWidth, "one piece per thread and branch");

template <typename I, typename T, bool CONCAT>
__global__ void __launch_bounds__(FT)
fuse_split_kernel(const float* __restrict__ part, int n_split, int H, int dv, const I* __restrict__ ypre,
                  const I* __restrict__ P, long long ldP, int col_z, const float* __restrict__ g_attn,
                  const float* __restrict__ g_ssm, const float* __restrict__ beta1, const float* __restrict__ beta2,
                  const float* __restrict__ v_scale, const float* __restrict__ v_bias, int rep, T* __restrict__ U,
                  int di, float eps, int* len_inc, float* __restrict__ y_init, const float* __restrict__ y_res,
                  int d_model) {
    griddep_sync();
    extern __shared__ float fsm[];  // [nh * n_split] m_s, [nh * n_split] l_s, [nh] M, [nh] 1 / den
    __shared__ float wsum[FT / 32][2];
    __shared__ float csum[2];  // this CTA's partial sums of squares, read by the whole cluster
    __shared__ float tot[2];
    const int cr = (int)cluster_rank();
    const long long row = blockIdx.x / FC;
    const int t = threadIdx.x;
    const int hv = H * dv, nvo = hv / 8, nvy = di / 8;
    const int po = (nvo + FC - 1) / FC, py = (nvy + FC - 1) / FC;
    const int a_lo = min(cr * po, nvo), a_hi = min(a_lo + po, nvo);
    const int vo = a_lo + t, vy = cr * py + t;
    const bool has_o = vo < a_hi, has_y = t < py && vy < nvy;
    // heads of this CTA's attention pieces (pieces never straddle a head)
    const int h_lo = a_lo * 8 / dv, nh = a_hi > a_lo ? (a_hi * 8 - 1) / dv + 1 - h_lo : 0;
    float* fm = fsm;
    float* fl = fsm + nh * n_split;
    float* hM = fl + nh * n_split;
    float* hinv = hM + nh;
    const float* rbase = part + (long long)row * H * n_split * (dv + 4);
    // issue every load: split records of this piece, y_pre and z, the heads' statistics
    const int hd = has_o ? vo * 8 / dv : 0, e = has_o ? vo * 8 - hd * dv : 0;
    const float* pp = rbase + (long long)hd * n_split * (dv + 4) + e;
    const int npre = min(n_split, FSPL);
    float4 pv[FSPL][2];
#pragma unroll
    for (int sp = 0; sp < FSPL; ++sp)
        if (has_o && sp < npre) {
            const float4* q = reinterpret_cast<const float4*>(pp + (long long)sp * (dv + 4));
            pv[sp][0] = q[0];
            pv[sp][1] = q[1];
        }
    float y[8], z[8];
    if (has_y) {
        load8<I>(ypre + row * di + vy * 8, y);
        load8<I>(P + row * ldP + col_z + vy * 8, z);
    }
    // the per-channel factors of this thread's pieces and its share of the residual
    float fa[8], fb[8], fc[8], fd[8];
    if constexpr (CONCAT) {
        if (has_y) { load8f(g_ssm + vy * 8, fa); load8f(beta2 + vy * 8, fb); }
        if (has_o) { load8f(g_attn + vo * 8, fc); load8f(beta1 + vo * 8, fd); }
    } else if (has_y) {
        load8f(g_attn + vy * 8, fa); load8f(beta1 + vy * 8, fb);
        load8f(g_ssm + vy * 8, fc); load8f(beta2 + vy * 8, fd);
    }
    const bool init = y_init && y_init != y_res;
    float yr[FYI];
#pragma unroll
    for (int k = 0; k < FYI; ++k) {
        const int c = cr * FT + t + k * FC * FT;
        yr[k] = init && y_res && c < d_model ? y_res[row * d_model + c] : 0.f;
    }
    for (int i = t; i < nh * n_split; i += FT) {
        const int hh = i / n_split, sp = i - hh * n_split;
        const float2 ml = *reinterpret_cast<const float2*>(rbase + ((long long)(h_lo + hh) * n_split + sp) * (dv + 4) + dv);
        fm[i] = ml.x;
        fl[i] = ml.y;
    }
    __syncthreads();
    for (int hh = t; hh < nh; hh += FT) {
        float M = -INFINITY;
        for (int sp = 0; sp < n_split; ++sp) M = fmaxf(M, fm[hh * n_split + sp]);
        float den = 0.f;
        if (M != -INFINITY)
            for (int sp = 0; sp < n_split; ++sp) den = fmaf(exp2f(fm[hh * n_split + sp] - M), fl[hh * n_split + sp], den);
        hM[hh] = M;
        hinv[hh] = den > 0.f ? 1.f / den : 0.f;
    }
    __syncthreads();
    float o[8];
    float ss_o = 0.f, ss_y = 0.f;
    if (has_o) {
        const int hh = hd - h_lo;
        const float M = hM[hh], inv = hinv[hh];
        const float* mrow = fm + hh * n_split;
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = 0.f;
#pragma unroll
        for (int sp = 0; sp < FSPL; ++sp)
            if (sp < npre) {
                const float w = M != -INFINITY ? exp2f(mrow[sp] - M) * inv : 0.f;
                o[0] = fmaf(w, pv[sp][0].x, o[0]); o[1] = fmaf(w, pv[sp][0].y, o[1]);
                o[2] = fmaf(w, pv[sp][0].z, o[2]); o[3] = fmaf(w, pv[sp][0].w, o[3]);
                o[4] = fmaf(w, pv[sp][1].x, o[4]); o[5] = fmaf(w, pv[sp][1].y, o[5]);
                o[6] = fmaf(w, pv[sp][1].z, o[6]); o[7] = fmaf(w, pv[sp][1].w, o[7]);
            }
        for (int sp = npre; sp < n_split; ++sp) {
            const float4* q = reinterpret_cast<const float4*>(pp + (long long)sp * (dv + 4));
            const float4 a = q[0], b = q[1];
            const float w = M != -INFINITY ? exp2f(mrow[sp] - M) * inv : 0.f;
            o[0] = fmaf(w, a.x, o[0]); o[1] = fmaf(w, a.y, o[1]); o[2] = fmaf(w, a.z, o[2]); o[3] = fmaf(w, a.w, o[3]);
            o[4] = fmaf(w, b.x, o[4]); o[5] = fmaf(w, b.y, o[5]); o[6] = fmaf(w, b.z, o[6]); o[7] = fmaf(w, b.w, o[7]);
        }
        if (v_scale) {
            // a consumer's adapted shared V: attention over V * s + b is the attention
            // output * s + b (the softmax weights sum to 1)
            const int idx = (hd / rep) * dv + e;
            float vs[8], vb[8];
            load8f(v_scale + idx, vs);
            load8f(v_bias + idx, vb);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = fmaf(o[i], vs[i], vb[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) ss_o = fmaf(o[i], o[i], ss_o);
    }
    if (has_y) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            y[i] *= z[i] / (1.0f + __expf(-z[i]));
            ss_y = fmaf(y[i], y[i], ss_y);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        ss_o += __shfl_xor_sync(0xffffffffu, ss_o, off);
        ss_y += __shfl_xor_sync(0xffffffffu, ss_y, off);
    }
    if ((t & 31) == 0) {
        wsum[t >> 5][0] = ss_o;
        wsum[t >> 5][1] = ss_y;
    }
    __syncthreads();
    if (t < 2) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < FT / 32; ++w) v += wsum[w][t];
        csum[t] = v;
    }
    cluster_arrive();
    cluster_wait();
    if (t < 2) {
        float v = 0.f;
#pragma unroll
        for (int r = 0; r < FC; ++r) v += ld_cluster_f32(&csum[t], (uint32_t)r);
        tot[t] = v;
    }
    __syncthreads();
    // the other CTAs may leave once every CTA has read their sums
    cluster_arrive();
    // the average halves both branches; the concatenation keeps them whole
    const float half = CONCAT ? 1.0f : 0.5f;
    const float ro = half / sqrtf(tot[0] / hv + eps);
    const float ry = half / sqrtf(tot[1] / di + eps);
    if constexpr (CONCAT) {
        const long long ldu = di + hv;
        if (has_y) {
            float u[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] = fb[i] * fa[i] * y[i] * ry;
            store8<T>(U + row * ldu + vy * 8, u);
        }
        if (has_o) {
            float u[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] = fd[i] * fc[i] * o[i] * ro;
            store8<T>(U + row * ldu + di + vo * 8, u);
        }
    } else if (has_o && has_y) {
        // equal widths: a thread holds the same channels of both branches
        float u[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) u[i] = fb[i] * fa[i] * o[i] * ro + fd[i] * fc[i] * y[i] * ry;
        store8<T>(U + row * di + vy * 8, u);
    }
    if (len_inc && cr == 0 && t == 0) len_inc[row] += 1;
    // the output projection that follows adds its split-K partial sums to y: y starts as
    // the residual (or zero), unless y is the residual itself
    if (init) {
#pragma unroll
        for (int k = 0; k < FYI; ++k) {
            const int c = cr * FT + t + k * FC * FT;
            if (c < d_model) y_init[row * d_model + c] = yr[k];
        }
        for (int c = cr * FT + t + FYI * FC * FT; c < d_model; c += FC * FT)
            y_init[row * d_model + c] = y_res ? y_res[row * d_model + c] : 0.f;
    }
    cluster_wait();
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
        auto kern = fuse_split_kernel<I, T, CONCAT>;
        // heads spanned by one CTA's attention pieces: at most ceil(po * 8 / dv) + 1
        const int po = ceil_div(H * dv / 8, FC);
        const int nh = std::min(H, ceil_div(po * 8, dv) + 1);
        const size_t smem = (2 * (size_t)nh * n_split + 2 * (size_t)nh) * sizeof(float);
        static std::atomic<unsigned long long> smem_set{0};
        if (smem > 48 * 1024 && !smem_opt_in_once(smem_set, kern, smem, ctx)) return HYMBA_ERR_CUDA;
        HYMBA_LAUNCH_CLUSTER(ctx, "fuse", kern, (long long)rows * FC, FT, smem, FC, part, n_split, H, dv, ypre, P,
                             ldP, col_z, g_attn, g_ssm, beta1, beta2, v_scale, v_bias, H / G, U, di, eps, len_inc,
                             y_init, y_res, d_model);
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
    if (di % 8 || di > kMaxWidth || hv > kMaxWidth || col_z % 8 || ldP % 8) return HYMBA_ERR_UNSUPPORTED;
    // pieces of 8 never straddle a head
    if (H <= 0 || G <= 0 || H % G || dv % 8 || (!concat && hv != di)) return HYMBA_ERR_UNSUPPORTED;
    if ((v_scale == nullptr) != (v_bias == nullptr) ||
        ((reinterpret_cast<uintptr_t>(v_scale) | reinterpret_cast<uintptr_t>(v_bias)) & 15))
        return HYMBA_ERR_UNSUPPORTED;
    // 16-byte loads of the partial sums; one cluster per row along x
    if (part && (n_split <= 0 || (reinterpret_cast<uintptr_t>(part) & 15) || (long long)rows * FC > INT32_MAX))
        return HYMBA_ERR_UNSUPPORTED;
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
