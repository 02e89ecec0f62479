// Small data-movement kernels around the mixer: the RoPE angle table with the padded
// W_dt copy of a prefill, zero-padded weight copies for TMA-aligned strides, and the
// decode-cache fill after a prefill; and the stalled wait that exercises the failure
// path of the bounded waits.
#include <algorithm>

#include "kernels.h"
#include "tc.cuh"

namespace hymba {

namespace {

template <typename TS, typename TD>
__global__ void pad_copy_kernel(const TS* src, int rows, int cols, TD* dst, int ld_dst) {
    griddep_sync();
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)rows * ld_dst) return;
    const int r = (int)(idx / ld_dst), c = (int)(idx % ld_dst);
    dst[idx] = from_f<TD>(c < cols ? to_f(src[(long long)r * cols + c]) : 0.f);
}

// Eight elements of a row as fp32 (one or two 16-byte loads).
template <typename TS>
__device__ __forceinline__ void load8_any(const TS* p, float* v) {
    if constexpr (sizeof(TS) == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p));
        const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const TS* h = reinterpret_cast<const TS*>(&u);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = to_f(h[i]);
    }
}

// The same copy, eight elements per thread and iteration with 16-byte accesses (cols and
// ld_dst multiples of 8, both rows 16-byte aligned), grid-stride over the 8-element
// pieces of the destination. HBM-bound: it moves (sizeof(TS) + 2) bytes per element.
template <typename TS, typename TD>
__global__ void __launch_bounds__(256) pad_copy8_kernel(const TS* __restrict__ src, int rows, int cols,
                                                        TD* __restrict__ dst, int ld_dst) {
    griddep_sync();
    const int per_row = ld_dst / 8;
    const long long n = (long long)rows * per_row;
    for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < n; v += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(v / per_row), c = (int)(v - (long long)r * per_row) * 8;
        float x[8];
        if (c < cols) {
            load8_any<TS>(src + (long long)r * cols + c, x);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = 0.f;
        }
        uint4 o;
        o.x = pack2<TD>(x[0], x[1]);
        o.y = pack2<TD>(x[2], x[3]);
        o.z = pack2<TD>(x[4], x[5]);
        o.w = pack2<TD>(x[6], x[7]);
        *reinterpret_cast<uint4*>(dst + (long long)r * ld_dst + c) = o;
    }
}

// The two small inputs of a prefill in one launch: blocks [0, nb_rope) fill the RoPE
// table, the rest copy W_dt into its zero-padded 16-bit form.
template <typename TS, typename TD>
__global__ void prefill_prep_kernel(float2* tab, int Tp, int half, int dh, float base, int nb_rope, const TS* w,
                                    int rows, int cols, TD* wdst, int ld_dst) {
    griddep_sync();
    if ((int)blockIdx.x < nb_rope) {
        const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
        if (idx >= (long long)Tp * half) return;
        const int p = (int)(idx / half), i = (int)(idx % half);
        tab[idx] = rope_cs_at(p, i, dh, base);
    } else {
        const long long idx = (long long)(blockIdx.x - nb_rope) * blockDim.x + threadIdx.x;
        if (idx >= (long long)rows * ld_dst) return;
        const int r = (int)(idx / ld_dst), c = (int)(idx % ld_dst);
        wdst[idx] = from_f<TD>(c < cols ? to_f(w[(long long)r * cols + c]) : 0.f);
    }
}

// The small inputs of a decode step in one launch: blocks [0, nb_rope) fill the RoPE
// table of each sequence's new position (len[b] + pos_offset; rows without a valid
// position get the identity rotation, their outputs are never written), the rest copy
// the step's input rows into the layer's compute type when they arrive in another.
template <typename TS, typename TD>
__global__ void decode_prep_kernel(float2* tab, const int* len, int pos_offset, int B, int half, int dh, float base,
                                   int nb_rope, const TS* w, int rows, int cols, TD* wdst, int ld_dst) {
    griddep_sync();
    if ((int)blockIdx.x < nb_rope) {
        const int idx = blockIdx.x * blockDim.x + threadIdx.x;
        if (idx >= B * half) return;
        const int b = idx / half, i = idx % half;
        const int p = len[b] + pos_offset;
        tab[idx] = p >= 0 ? rope_cs_at(p, i, dh, base) : make_float2(1.f, 0.f);
    } else {
        const long long idx = (long long)(blockIdx.x - nb_rope) * blockDim.x + threadIdx.x;
        if (idx >= (long long)rows * ld_dst) return;
        const int r = (int)(idx / ld_dst), c = (int)(idx % ld_dst);
        wdst[idx] = from_f<TD>(c < cols ? to_f(w[(long long)r * cols + c]) : 0.f);
    }
}

// Slot of position p: meta positions keep their slot, the others wrap in a ring of
// cache_cap - n_meta slots. Rows copied: meta positions and the newest ring-full.
template <typename T>
__global__ void cache_fill_kernel(const T* k_seq, const T* v_seq, int seq_cap, T* k_cache,
                                  T* v_cache, int cache_cap, int* len, int G, int dh, int dv,
                                  int n_meta, int Tp) {
    griddep_sync();
    const int ring = cache_cap - n_meta;
    const int first_kept = max(n_meta, Tp - ring);
    const int n_rows = min(n_meta, Tp) + max(0, Tp - first_kept);
    const int b = blockIdx.z, g = blockIdx.y;
    for (int ri = blockIdx.x; ri < n_rows; ri += gridDim.x) {
        const int meta_rows = min(n_meta, Tp);
        const int p = ri < meta_rows ? ri : first_kept + (ri - meta_rows);
        const int slot = p < n_meta ? p : n_meta + (p - n_meta) % ring;
        const long long src = ((long long)b * G + g) * seq_cap + p;
        const long long dst = ((long long)b * G + g) * cache_cap + slot;
        for (int e = threadIdx.x; e < dh; e += blockDim.x) k_cache[dst * dh + e] = k_seq[src * dh + e];
        for (int e = threadIdx.x; e < dv; e += blockDim.x) v_cache[dst * dv + e] = v_seq[src * dv + e];
    }
    if (blockIdx.x == 0 && g == 0 && threadIdx.x == 0) len[b] = Tp;
}

}  // namespace

template <typename TS, typename TD>
int launch_pad_copy(const Ctx& ctx, const TS* src, int rows, int cols, TD* dst, int ld_dst) {
    const long long n = (long long)rows * ld_dst;
    if constexpr (sizeof(TD) == 2) {
        if (cols % 8 == 0 && ld_dst % 8 == 0 && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0) {
            auto kern = pad_copy8_kernel<TS, TD>;
            const long long pieces = n / 8;
            const int grid = (int)std::min<long long>(ceil_div(pieces, 256), (long long)ctx.sm_count * 8);
            HYMBA_LAUNCH(ctx, "pad_copy", kern, grid, 256, 0, src, rows, cols, dst, ld_dst);
            return HYMBA_OK;
        }
    }
    auto kern = pad_copy_kernel<TS, TD>;
    HYMBA_LAUNCH(ctx, "pad_copy", kern, ceil_div(n, 256), 256, 0, src, rows, cols, dst, ld_dst);
    return HYMBA_OK;
}

template <typename TS, typename TD>
int launch_prefill_prep(const Ctx& ctx, float2* tab, int Tp, int dh, float base, const TS* w, int rows, int cols,
                        TD* wdst, int ld_dst) {
    const int nb_rope = ceil_div((long long)Tp * (dh / 2), 256);
    const int nb_pad = ceil_div((long long)rows * ld_dst, 256);
    auto kern = prefill_prep_kernel<TS, TD>;
    HYMBA_LAUNCH(ctx, "prefill_prep", kern, nb_rope + nb_pad, 256, 0, tab, Tp, dh / 2, dh, base, nb_rope, w, rows,
                 cols, wdst, ld_dst);
    return HYMBA_OK;
}

template <typename TS, typename TD>
int launch_decode_prep(const Ctx& ctx, float2* tab, const int* len, int pos_offset, int B, int dh, float base,
                       const TS* w, int rows, int cols, TD* wdst, int ld_dst) {
    const int nb_rope = ceil_div((long long)B * (dh / 2), 256);
    const int nb_pad = ceil_div((long long)rows * ld_dst, 256);
    auto kern = decode_prep_kernel<TS, TD>;
    HYMBA_LAUNCH(ctx, "decode_prep", kern, nb_rope + nb_pad, 256, 0, tab, len, pos_offset, B, dh / 2, dh, base,
                 nb_rope, w, rows, cols, wdst, ld_dst);
    return HYMBA_OK;
}

template <typename T>
int launch_cache_fill(const Ctx& ctx, const T* k_seq, const T* v_seq, int seq_cap, T* k_cache,
                      T* v_cache, int cache_cap, int* len, int B, int G, int dh, int dv, int n_meta,
                      int Tp) {
    dim3 grid(256, G, B);
    HYMBA_LAUNCH(ctx, "cache_fill", cache_fill_kernel<T>, grid, 128, 0, k_seq, v_seq, seq_cap,
                 k_cache, v_cache, cache_cap, len, G, dh, dv, n_meta, Tp);
    return HYMBA_OK;
}

template int launch_pad_copy<float, float>(const Ctx&, const float*, int, int, float*, int);
template int launch_pad_copy<float, bf16>(const Ctx&, const float*, int, int, bf16*, int);
template int launch_pad_copy<float, f16>(const Ctx&, const float*, int, int, f16*, int);
template int launch_pad_copy<bf16, f16>(const Ctx&, const bf16*, int, int, f16*, int);
template int launch_prefill_prep<float, float>(const Ctx&, float2*, int, int, float, const float*, int, int, float*,
                                               int);
template int launch_prefill_prep<bf16, f16>(const Ctx&, float2*, int, int, float, const bf16*, int, int, f16*, int);
template int launch_decode_prep<float, float>(const Ctx&, float2*, const int*, int, int, int, float, const float*,
                                              int, int, float*, int);
template int launch_decode_prep<bf16, bf16>(const Ctx&, float2*, const int*, int, int, int, float, const bf16*, int,
                                            int, bf16*, int);
template int launch_decode_prep<float, bf16>(const Ctx&, float2*, const int*, int, int, int, float, const float*, int,
                                             int, bf16*, int);
template int launch_cache_fill<float>(const Ctx&, const float*, const float*, int, float*, float*,
                                      int, int*, int, int, int, int, int, int);
template int launch_cache_fill<f16>(const Ctx&, const f16*, const f16*, int, f16*, f16*, int,
                                    int*, int, int, int, int, int, int);

}  // namespace hymba

namespace hymba {
namespace {

// One thread waits on an mbarrier that nothing arrives on, with the progress-wait limit
// the tensor-core kernels use: the wait runs out and records HYMBA_ERR_DEVICE_TIMEOUT
// (role 4) the way theirs do, and the block returns with nothing in flight.
__global__ void stalled_wait_kernel(int* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int zero = 0;
        if (!tc::mbar_wait(&bar, 0, &zero, tc::wait_limit(status))) tc::record_timeout(status, 4, 0, 0);
    }
}

}  // namespace
}  // namespace hymba

extern "C" int hymba_debug_stalled_wait(void* stream) {
    hymba::Ctx ctx;
    int rc = hymba::launch_context(static_cast<cudaStream_t>(stream), &ctx);
    if (rc) return rc;
    HYMBA_LAUNCH(ctx, "stalled_wait", hymba::stalled_wait_kernel, 1, 32, 0, ctx.status);
    return HYMBA_OK;
}

namespace hymba {
namespace {

// Row RMSNorm with gain into another type: dst[r, c] = g[c] * src[r, c] / sqrt(mean_c
// src[r, c]^2 + eps). One row per 256-thread block, pieces of 8 elements (16-byte
// accesses when the element type allows), the row held in registers between the sum of
// squares and the output (cols <= 4096).
template <typename TS, typename TD>
__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(const TS* __restrict__ src, const float* __restrict__ g,
                                                           TD* __restrict__ dst, int rows, int cols, float eps) {
    griddep_sync();
    __shared__ float red[8];
    const long long r = blockIdx.x;
    const int t = threadIdx.x;
    const int npc = cols / 8;
    float v[2][8];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int pc = t + k * 256;
        if (pc < npc) {
            const TS* p = src + r * cols + 8 * pc;
            if constexpr (sizeof(TS) == 4) {
                const float4 a = *reinterpret_cast<const float4*>(p);
                const float4 b = *reinterpret_cast<const float4*>(p + 4);
                v[k][0] = a.x; v[k][1] = a.y; v[k][2] = a.z; v[k][3] = a.w;
                v[k][4] = b.x; v[k][5] = b.y; v[k][6] = b.z; v[k][7] = b.w;
            } else {
                const uint4 u = *reinterpret_cast<const uint4*>(p);
                const TS* h = reinterpret_cast<const TS*>(&u);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[k][i] = to_f(h[i]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) ss = fmaf(v[k][i], v[k][i], ss);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((t & 31) == 0) red[t >> 5] = ss;
    __syncthreads();
    ss = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) ss += red[w];
    const float inv = 1.0f / sqrtf(ss / cols + eps);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int pc = t + k * 256;
        if (pc < npc) {
            const float4 ga = *reinterpret_cast<const float4*>(g + 8 * pc);
            const float4 gb = *reinterpret_cast<const float4*>(g + 8 * pc + 4);
            const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            TD* q = dst + r * cols + 8 * pc;
            if constexpr (sizeof(TD) == 4) {
                *reinterpret_cast<float4*>(q) = make_float4(gg[0] * v[k][0] * inv, gg[1] * v[k][1] * inv,
                                                            gg[2] * v[k][2] * inv, gg[3] * v[k][3] * inv);
                *reinterpret_cast<float4*>(q + 4) = make_float4(gg[4] * v[k][4] * inv, gg[5] * v[k][5] * inv,
                                                                gg[6] * v[k][6] * inv, gg[7] * v[k][7] * inv);
            } else {
                uint4 o;
                o.x = pack2<TD>(gg[0] * v[k][0] * inv, gg[1] * v[k][1] * inv);
                o.y = pack2<TD>(gg[2] * v[k][2] * inv, gg[3] * v[k][3] * inv);
                o.z = pack2<TD>(gg[4] * v[k][4] * inv, gg[5] * v[k][5] * inv);
                o.w = pack2<TD>(gg[6] * v[k][6] * inv, gg[7] * v[k][7] * inv);
                *reinterpret_cast<uint4*>(q) = o;
            }
        }
    }
}

}  // namespace

template <typename TS, typename TD>
int launch_rmsnorm_rows(const Ctx& ctx, const TS* src, const float* g, TD* dst, long long rows, int cols, float eps) {
    if (rows <= 0) return HYMBA_OK;
    if (cols % 8 || cols > 4096 || rows > 0x7fffffffLL ||
        ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(g)) & 15))
        return HYMBA_ERR_UNSUPPORTED;
    auto kern = rmsnorm_rows_kernel<TS, TD>;
    HYMBA_LAUNCH(ctx, "rmsnorm", kern, (unsigned)rows, 256, 0, src, g, dst, (int)rows, cols, eps);
    return HYMBA_OK;
}

template int launch_rmsnorm_rows<float, float>(const Ctx&, const float*, const float*, float*, long long, int, float);
template int launch_rmsnorm_rows<float, f16>(const Ctx&, const float*, const float*, f16*, long long, int, float);
template int launch_rmsnorm_rows<bf16, bf16>(const Ctx&, const bf16*, const float*, bf16*, long long, int, float);
template int launch_rmsnorm_rows<float, bf16>(const Ctx&, const float*, const float*, bf16*, long long, int, float);

}  // namespace hymba
