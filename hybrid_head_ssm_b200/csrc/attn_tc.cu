// Attention heads of the mixer, prefill, on the tcgen05 tensor cores: causal GQA
// softmax(Q K^T / sqrt(d_k)) V ("Jamba: Hybrid SSM-Transformer", section 1) over the
// meta-token prefix, which every query sees ("Hymba Guide", Learnable Meta-Tokens),
// plus a sliding window or the whole causal history (51cto Hymba-1.5B article,
// section 2). Key j is visible to query i iff j <= i and (j < n_meta or i - j < W).
//
// One CTA per (128-query tile, query head, sequence), 6 warps:
//   warp 0      TMA: the Q tile once, then K (128 keys x 64) and V (128 keys x 128, two
//               64-wide panels) of each visible key block into a 2-stage ring;
//   warp 1      MMA issuer: S_j = Q K_j^T (128 x 128 x 64) into one of two TMEM S buffers,
//               then O += P_j V_j (128 x 128 x 128) into the TMEM O accumulator;
//   warps 2..5  softmax, one query row per thread: S_j from TMEM, scale and mask, running
//               max; P_j = 2^(s - m) in fp16 into a 128-byte-swizzled shared-memory tile
//               (the A operand of the PV MMA); O is rescaled in TMEM only when the
//               running max grows by more than 2^8, so most blocks need no rescale.
//               At the end O / l is written in fp16.
// Only key blocks that hold visible keys are visited: the meta blocks and the blocks of
// [max(n_meta, i0 - W + 1), i_last]. Operands are fp16 (the layer's intermediate type).
#include "kernels.h"
#include "tc.cuh"

namespace hymba {

namespace {

constexpr int QT = 128, KBLK = 128, DH = 64, DV = 128, NTHREADS = 192;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_LOG2 = 8.0f;

struct AttnSmem {
    alignas(1024) uint8_t q[QT * DH * 2];
    alignas(1024) uint8_t k[2][KBLK * DH * 2];
    alignas(1024) uint8_t v[2][2][KBLK * 64 * 2];
    alignas(1024) uint8_t p[2][2][QT * 64 * 2];
    uint64_t q_full;
    uint64_t kv_full[2], kv_empty[2];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], pv_done[2];
    uint64_t o_done, drain;
    uint32_t tmem_base;
    int abort;
};

struct Blocks {
    int n_meta_blk, meta_end, lo, hi, n;
    __device__ void init(int i0, int Tp, int n_meta, int window) {
        const int i_last = min(i0 + QT, Tp) - 1;
        meta_end = min(n_meta, i_last + 1);
        n_meta_blk = (meta_end + KBLK - 1) / KBLK;
        lo = window > 0 ? max(n_meta, i0 - window + 1) : n_meta;
        hi = i_last + 1;
        n = n_meta_blk + (hi > lo ? (hi - lo + KBLK - 1) / KBLK : 0);
    }
    // first key, and the key range [rs, re) the block belongs to
    __device__ void get(int j, int* j0, int* rs, int* re) const {
        if (j < n_meta_blk) { *j0 = j * KBLK; *rs = 0; *re = meta_end; }
        else { *j0 = lo + (j - n_meta_blk) * KBLK; *rs = lo; *re = hi; }
    }
};

__device__ __forceinline__ void fail(volatile int* abort, int* status, int role, int step, int bar) {
    *abort = 1;
    tc::record_timeout(status, role, step, bar);
}

__global__ void __launch_bounds__(NTHREADS, 1)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, f16* __restrict__ O, int Tp, int H, int G,
                       int n_meta, int window, int* status) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem& s = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    constexpr uint32_t IDESC_S = tc::idesc_f16(false, QT, KBLK);
    constexpr uint32_t IDESC_PV = tc::idesc_f16(false, QT, DV, true);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * QT, h = blockIdx.y, b = blockIdx.z;
    const int bg = b * G + h / (H / G);
    Blocks blk;
    blk.init(i0, Tp, n_meta, window);
    const int nblk = blk.n;

    if (threadIdx.x == 0) {
        tc::mbar_init(&s.q_full, 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&s.kv_full[i], 1);
            tc::mbar_init(&s.kv_empty[i], 1);
            tc::mbar_init(&s.s_full[i], 1);
            tc::mbar_init(&s.s_free[i], 128);
            tc::mbar_init(&s.p_full[i], 128);
            tc::mbar_init(&s.pv_done[i], 1);
        }
        tc::mbar_init(&s.o_done, 1);
        tc::mbar_init(&s.drain, 1);
        s.abort = 0;
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tmQ);
        tc::prefetch_tmap(&tmK);
        tc::prefetch_tmap(&tmV);
    }
    if (warp == 1) {
        tc::tmem_alloc(&s.tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = s.tmem_base;  // O: columns 0..127, S buffers: 128..255, 256..383
    volatile int* abort = &s.abort;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (tc::elect_one()) {
            int zero = 0;
            int last_phase[2] = {-1, -1};
            tc::mbar_arrive_expect_tx(&s.q_full, QT * DH * 2);
            tc::tma_load_3d(s.q, &tmQ, &s.q_full, h * DH, i0, b);
            for (int j = 0; j < nblk; ++j) {
                const int st = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                if (!tc::mbar_wait(&s.kv_empty[st], ph ^ 1, abort)) { fail(abort, status, 0, j, 1); break; }
                int j0, rs, re;
                blk.get(j, &j0, &rs, &re);
                tc::mbar_arrive_expect_tx(&s.kv_full[st], KBLK * (DH + DV) * 2);
                tc::tma_load_3d(s.k[st], &tmK, &s.kv_full[st], 0, j0, bg);
                tc::tma_load_3d(s.v[st][0], &tmV, &s.kv_full[st], 0, j0, bg);
                tc::tma_load_3d(s.v[st][1], &tmV, &s.kv_full[st], 64, j0, bg);
                last_phase[st] = (int)ph;
            }
            tc::mbar_wait(&s.q_full, 0, &zero);
            if (*abort)
                for (int i = 0; i < 2; ++i)
                    if (last_phase[i] >= 0) tc::mbar_wait(&s.kv_full[i], (uint32_t)last_phase[i], &zero);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (tc::elect_one()) {
            bool ok = tc::mbar_wait(&s.q_full, 0, abort);
            if (!ok) fail(abort, status, 1, 0, 0);
            const uint32_t qa = tc::smem_u32(s.q);
            for (int j = 0; ok && j <= nblk; ++j) {
                if (j < nblk) {
                    const int st = j & 1;
                    const uint32_t ph = (j >> 1) & 1;
                    if (!tc::mbar_wait(&s.kv_full[st], ph, abort)) { fail(abort, status, 1, j, 2); break; }
                    if (!tc::mbar_wait(&s.s_free[st], ph ^ 1, abort)) { fail(abort, status, 1, j, 3); break; }
                    tc::tc_fence_after();
                    const uint32_t ka = tc::smem_u32(s.k[st]);
                    const uint32_t sd = tmem + 128 + st * 128;
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk)
                        tc::mma_f16_ss(sd, tc::sdesc_k_sw128(qa + kk * 32), tc::sdesc_k_sw128(ka + kk * 32), IDESC_S,
                                       kk > 0);
                    tc::mma_commit(&s.s_full[st]);
                }
                if (j >= 1) {
                    const int jj = j - 1, pb = jj & 1;
                    if (!tc::mbar_wait(&s.p_full[pb], (jj >> 1) & 1, abort)) { fail(abort, status, 1, jj, 4); break; }
                    tc::tc_fence_after();
                    const uint32_t pa = tc::smem_u32(s.p[pb][0]);
                    const uint32_t va = tc::smem_u32(s.v[pb][0]);
#pragma unroll
                    for (int kk = 0; kk < KBLK / 16; ++kk) {
                        const uint64_t ad = tc::sdesc_k_sw128(pa + (kk >> 2) * (QT * 128) + (kk & 3) * 32);
                        const uint64_t bd = tc::sdesc_mn_sw128(va + kk * 2048, KBLK * 128);
                        tc::mma_f16_ss(tmem, ad, bd, IDESC_PV, (jj > 0 || kk > 0));
                    }
                    tc::mma_commit(&s.pv_done[pb]);
                    tc::mma_commit(&s.kv_empty[pb]);
                }
            }
            tc::mma_commit(&s.o_done);
            tc::mma_commit(&s.drain);
            int zero = 0;
            tc::mbar_wait(&s.drain, 0, &zero);
        }
    } else {
        // ---------------- softmax + output (warps 2..5 -> TMEM lane quadrants 2, 3, 0, 1) ----------------
        const int q = warp & 3;
        const int r = q * 32 + lane;  // row within the tile
        const int i = i0 + r;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float scale = LOG2E * 0.125f;  // log2(e) / sqrt(64)
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nblk; ++j) {
            const int sb = j & 1;
            int j0, rs, re;
            blk.get(j, &j0, &rs, &re);
            // tcgen05.ld/st are warp-collective: every decision that guards them is
            // taken by the whole warp (__all_sync / __any_sync)
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&s.s_full[sb], (j >> 1) & 1, abort))) {
                fail(abort, status, 2, j, 5);
                ok = false;
                break;
            }
            tc::tc_fence_after();
            float sv[KBLK];
#pragma unroll
            for (int c = 0; c < KBLK / 32; ++c) {
                uint32_t rr[32];
                tc::tmem_ld32(tmem + lane_base + 128 + sb * 128 + c * 32, rr);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(rr[e]);
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&s.s_free[sb]);
            // scale, mask, block max
            const bool row_full = j0 >= rs && j0 + KBLK <= re && j0 + KBLK - 1 <= i &&
                                  (j0 + KBLK <= n_meta || window <= 0 || i - j0 < window);
            float mx = -INFINITY;
            if (row_full) {
#pragma unroll
                for (int c = 0; c < KBLK; ++c) {
                    sv[c] *= scale;
                    mx = fmaxf(mx, sv[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < KBLK; ++c) {
                    const int jk = j0 + c;
                    const bool vis = jk >= rs && jk < re && jk <= i && (jk < n_meta || window <= 0 || i - jk < window);
                    sv[c] = vis ? sv[c] * scale : -INFINITY;
                    mx = fmaxf(mx, sv[c]);
                }
            }
            const float m_new = fmaxf(m_used, mx);
            // the P buffer of this block is free once PV[j-2] has completed
            if (j >= 2 && !__all_sync(0xffffffffu, tc::mbar_wait(&s.pv_done[sb], ((j - 2) >> 1) & 1, abort))) {
                fail(abort, status, 2, j, 6);
                ok = false;
                break;
            }
            // rows whose running max grew by more than 2^8 move to the new max; their O row
            // (PV[0..j-1]) is scaled by f in TMEM, the other rows of the warp by 1
            float f = 1.f;
            bool scale_o = false;
            if (m_new > m_used + RESCALE_LOG2) {
                if (m_used != -INFINITY) {
                    f = exp2f(m_used - m_new);
                    l *= f;
                    scale_o = j >= 1;
                }
                m_used = m_new;
            }
            if (__any_sync(0xffffffffu, scale_o)) {
                if (!__all_sync(0xffffffffu, tc::mbar_wait(&s.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort))) {
                    fail(abort, status, 2, j, 7);
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < DV / 32; ++c) {
                    uint32_t rr[32];
                    tc::tmem_ld32(tmem + lane_base + c * 32, rr);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * f);
                    tc::tmem_st32(tmem + lane_base + c * 32, rr);
                }
                tc::tmem_wait_st();
            }
            const float mu = m_used == -INFINITY ? 0.f : m_used;
            uint8_t* prow = s.p[sb][0];
#pragma unroll
            for (int c8 = 0; c8 < KBLK / 8; ++c8) {
                float pv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pv[e] = fast_exp2(sv[c8 * 8 + e] - mu);
                    l += pv[e];
                }
                uint4 pk;
                pk.x = pack_f16x2(pv[0], pv[1]);
                pk.y = pack_f16x2(pv[2], pv[3]);
                pk.z = pack_f16x2(pv[4], pv[5]);
                pk.w = pack_f16x2(pv[6], pv[7]);
                const int panel = c8 >> 3, ch = c8 & 7;
                *reinterpret_cast<uint4*>(prow + panel * (QT * 128) + r * 128 + ((ch ^ (r & 7)) << 4)) = pk;
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(&s.p_full[sb]);
        }
        if (ok && __all_sync(0xffffffffu, tc::mbar_wait(&s.o_done, 0, abort))) {
            tc::tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            f16* orow = O + ((long long)b * Tp + i) * ((long long)H * DV) + h * DV;
#pragma unroll 1
            for (int c = 0; c < DV / 32; ++c) {
                uint32_t rr[32];
                tc::tmem_ld32(tmem + lane_base + c * 32, rr);
                tc::tmem_wait_ld();
                if (i < Tp) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 pk;
                        pk.x = pack_f16x2(__uint_as_float(rr[e]) * inv, __uint_as_float(rr[e + 1]) * inv);
                        pk.y = pack_f16x2(__uint_as_float(rr[e + 2]) * inv, __uint_as_float(rr[e + 3]) * inv);
                        pk.z = pack_f16x2(__uint_as_float(rr[e + 4]) * inv, __uint_as_float(rr[e + 5]) * inv);
                        pk.w = pack_f16x2(__uint_as_float(rr[e + 6]) * inv, __uint_as_float(rr[e + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + e) = pk;
                    }
                }
            }
        } else if (ok) {
            fail(abort, status, 2, nblk, 8);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

int launch_attn_prefill_tc(const Ctx& ctx, const f16* P, long long ldP, const f16* k_seq, const f16* v_seq,
                           int kcap, f16* O, int B, int Tp, int H, int G, int dv, int n_meta, int window) {
    if (dv != DV) return HYMBA_ERR_UNSUPPORTED;
    CUtensorMap tq, tk, tv;
    // Q: P viewed as [B][Tp][ldP]; K: [B*G][Tp][64]; V: [B*G][Tp][128] (rows >= Tp read as 0)
    if (!tc::make_tmap_3d(&tq, P, false, B, Tp, (uint64_t)H * DH, ldP, (uint64_t)Tp * ldP, QT) ||
        !tc::make_tmap_3d(&tk, k_seq, false, (uint64_t)B * G, Tp, DH, DH, (uint64_t)kcap * DH, KBLK) ||
        !tc::make_tmap_3d(&tv, v_seq, false, (uint64_t)B * G, Tp, DV, DV, (uint64_t)kcap * DV, KBLK))
        return HYMBA_ERR_UNSUPPORTED;
    const size_t smem = sizeof(AttnSmem) + 1024;
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(attn_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return HYMBA_ERR_CUDA;
        attr_set = true;
    }
    dim3 grid(ceil_div(Tp, QT), H, B);
    HYMBA_LAUNCH(ctx, "attn_prefill", attn_prefill_tc_kernel, grid, NTHREADS, smem, tq, tk, tv, O, Tp, H, G,
                 n_meta, window, ctx.status);
    return HYMBA_OK;
}

}  // namespace hymba
