// Attention heads of the mixer, prefill, on the tcgen05 tensor cores: causal GQA
// softmax(Q K^T / sqrt(d_k)) V ("Jamba: Hybrid SSM-Transformer", section 1) over the
// meta-token prefix, which every query sees ("Hymba Guide", Learnable Meta-Tokens),
// plus a sliding window or the whole causal history (51cto Hymba-1.5B article,
// section 2). Key j is visible to query i iff j <= i and (j < n_meta or i - j < W).
//
// One CTA per pair of consecutive 128-query tiles (A: rows i0..i0+127, B: the next 128)
// of one query head and sequence. The two tiles share every K and V block the CTA
// loads and run as two independent pipelines, so that the tensor cores work on one
// tile while the other tile's softmax runs. 12 warps:
//   warp 0      TMA: lane 0 the two Q tiles, then K (128 keys x 64) of every key block
//               of the pair into a 3-stage ring; lane 1 V (128 keys x 128, two 64-wide
//               panels) into a 3-stage ring;
//   warp 1      TMEM allocation and the MMA issuer. Per tile t and block u:
//               S_t = Q_t K^T (128 x 128 x 64, operands in shared memory) into the tile's
//               S columns of TMEM, then, once the softmax has written P_t (fp16) over
//               those columns, O_t += P_t V (128 x 128 x 128, A operand P_t read from
//               TMEM, B = V from shared memory). P lives in TMEM, so the PV operand
//               traffic stays off shared memory. The next S_t overwrites P_t, so it is
//               issued once that PV has completed; the order A, B, A, B ... lets each
//               tile's MMAs run under the other tile's softmax;
//   warps 2-3   idle after setup;
//   warps 4-7   softmax of tile A, warps 8-11 of tile B: one thread per query row
//               (TMEM lane), 128 scores in registers (four TMEM loads in flight, one wait):
//               scale and mask, row max, P = 2^(s - m) in fp32 (MUFU ex2; with the MMAs
//               of the other tile running meanwhile the exponentials are not the limit:
//               moving a quarter of them to an FMA-pipe polynomial measured no faster),
//               row sum in fp32, P packed to fp16 pairs
//               and stored to TMEM with tcgen05.st. O is rescaled in TMEM only when the
//               running max grows by more than 2^8 (P then stays below 2^8, far inside
//               fp16). At the end O / l is written in fp16.
// Warpgroup 0 (warps 0-3) gives registers to the softmax warpgroups (setmaxnreg:
// 4 x 32 x 64 + 8 x 32 x 216 <= 384 x 168, the launch's allocation).
// Key blocks: the meta blocks [0, meta_end) and the window blocks from the pair's
// first visible window key; a tile skips the blocks that hold none of its keys.
// Operands are fp16 (the layer's intermediate type).
#include "kernels.h"
#include "tc.cuh"

namespace hymba {

namespace {

constexpr int QT = 128, KBLK = 128, DH = 64;
constexpr int NTHREADS = 384;
constexpr int KST = 3;      // K ring stages
constexpr int VST = 3;      // V ring stages
constexpr int REG_SOFT = 216, REG_OTHER = 64;
// the launch allocates 168 registers per thread (65536 / 384, rounded down to 8): the
// split must fit that pool (the launcher also checks the compiled count)
static_assert(4 * 32 * REG_OTHER + 8 * 32 * REG_SOFT <= NTHREADS * 168, "register split exceeds the launch's pool");
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_LOG2 = 8.0f;
// TMEM columns: O_A [0,128), O_B [128,256), S_A [256,384), S_B [384,512); P_t in the
// first 64 columns of S_t (128 fp16 keys per row, two per column)
constexpr uint32_t TM_O = 0, TM_S = 256;

// DV: the V head dim (64 or 128), one or two 64-wide V panels per key block
template <int DV>
struct AttnSmem {
    alignas(1024) uint8_t q[2][QT * DH * 2];
    alignas(1024) uint8_t k[KST][KBLK * DH * 2];
    alignas(1024) uint8_t v[VST][DV / 64][KBLK * 64 * 2];
    uint64_t q_full;
    uint64_t k_full[KST], k_empty[KST];
    uint64_t v_full[VST], v_empty[VST];
    uint64_t s_full[2], p_full[2], pv_done[2], o_done[2], drain;
    uint32_t tmem_base;
    int abort;
};

// Visible keys of a 128-row query tile: [0, meta_end) and [lo, hi).
struct Span {
    int meta_end, lo, hi, valid;
    __device__ void init(int i0, int Tp, int n_meta, int window) {
        valid = i0 < Tp;
        const int i_last = min(i0 + QT, Tp) - 1;
        meta_end = valid ? min(n_meta, i_last + 1) : 0;
        lo = window > 0 ? max(n_meta, i0 - window + 1) : n_meta;
        hi = valid ? i_last + 1 : lo;
        if (hi < lo) hi = lo;
    }
};

// Key blocks of the tile pair: nmb meta blocks of 128 keys from 0, then window blocks of
// 128 keys from the pair's lowest window key.
struct Blocks {
    Span t[2];
    int nmb, lo, n;
    __device__ void init(int i0, int Tp, int n_meta, int window) {
        t[0].init(i0, Tp, n_meta, window);
        t[1].init(i0 + QT, Tp, n_meta, window);
        const int meta_end = max(t[0].meta_end, t[1].meta_end);
        nmb = (meta_end + KBLK - 1) / KBLK;
        lo = t[0].lo;
        const int hi = max(t[0].hi, t[1].hi);
        n = nmb + (hi > lo ? (hi - lo + KBLK - 1) / KBLK : 0);
    }
    __device__ int key0(int j) const { return j < nmb ? j * KBLK : lo + (j - nmb) * KBLK; }
    // does block j hold keys visible to some row of tile s?
    __device__ bool uses(int s, int j) const {
        const Span& p = t[s];
        if (!p.valid) return false;
        const int k0 = key0(j);
        if (j < nmb) return k0 < p.meta_end;
        return p.lo < p.hi && k0 < p.hi && k0 + KBLK > p.lo;
    }
    __device__ int users(int j) const { return (int)uses(0, j) + (int)uses(1, j); }
    // the u-th block tile s uses (blocks are used in increasing order), or -1
    __device__ int nth(int s, int u) const {
        for (int j = 0; j < n; ++j)
            if (uses(s, j) && u-- == 0) return j;
        return -1;
    }
    __device__ int count(int s) const {
        int c = 0;
        for (int j = 0; j < n; ++j) c += uses(s, j);
        return c;
    }
};

__device__ __forceinline__ void fail(volatile int* abort, int* status, int role, int step, int bar) {
    *abort = 1;
    tc::record_timeout(status, role, step, bar);
}

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// D[tmem] (+)= A[tmem] * B[smem]: the A operand (M x K, 16-bit, two K elements per
// 32-bit column) read from tensor memory.
__device__ __forceinline__ void mma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// 32 lanes x 64 consecutive 32-bit columns from registers (thread t writes lane base + t).
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,"
        "%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
        "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]),
          "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]),
          "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]),
          "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]),
          "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
        : "memory");
}

template <int DV>
__global__ void __launch_bounds__(NTHREADS, 1)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, f16* __restrict__ O, int Tp, int H, int G,
                       int n_meta, int window, int n_pairs, int* status) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<DV>& s = *reinterpret_cast<AttnSmem<DV>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    constexpr uint32_t IDESC_S = tc::idesc_f16(false, QT, KBLK);
    constexpr uint32_t IDESC_PV = tc::idesc_f16(false, QT, DV, true);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the heaviest pairs (latest query rows) first: the grid's slowest dimension walks
    // the pairs from the last one down
    const int pair = n_pairs - 1 - (int)blockIdx.z;
    const int i0 = pair * 2 * QT, h = blockIdx.x, b = blockIdx.y;
    const int bg = b * G + h / (H / G);
    Blocks blk;
    blk.init(i0, Tp, n_meta, window);
    const int nblk = blk.n;

    if (threadIdx.x == 0) {
        tc::mbar_init(&s.q_full, 1);
        for (int i = 0; i < KST; ++i) {
            tc::mbar_init(&s.k_full[i], 1);
            tc::mbar_init(&s.k_empty[i], 2);  // one commit per tile (two for a block one tile skips)
        }
        for (int i = 0; i < VST; ++i) {
            tc::mbar_init(&s.v_full[i], 1);
            tc::mbar_init(&s.v_empty[i], 2);
        }
        for (int t = 0; t < 2; ++t) {
            tc::mbar_init(&s.s_full[t], 1);
            tc::mbar_init(&s.p_full[t], QT);
            tc::mbar_init(&s.pv_done[t], 1);
            tc::mbar_init(&s.o_done[t], 1);
        }
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
    // setup above touches no global memory; everything below may read the previous
    // kernel's output
    griddep_sync();
    const uint32_t tmem = s.tmem_base;
    volatile int* abort = &s.abort;
    const long long wlim = tc::wait_limit(status);

    if (warp < 4) {
        setmaxnreg_dec<REG_OTHER>();
        if (warp == 0) {
            // ---------------- TMA producers ----------------
            int zero = 0;
            if (lane == 0) {
                int last_phase[KST];
                for (int i = 0; i < KST; ++i) last_phase[i] = -1;
                tc::mbar_arrive_expect_tx(&s.q_full, 2 * QT * DH * 2);
                tc::tma_load_3d(s.q[0], &tmQ, &s.q_full, h * DH, i0, b);
                tc::tma_load_3d(s.q[1], &tmQ, &s.q_full, h * DH, i0 + QT, b);
                for (int j = 0; j < nblk; ++j) {
                    const int st = j % KST;
                    const uint32_t ph = (j / KST) & 1;
                    if (!tc::mbar_wait(&s.k_empty[st], ph ^ 1, abort, wlim)) { fail(abort, status, 0, j, 1); break; }
                    tc::mbar_arrive_expect_tx(&s.k_full[st], KBLK * DH * 2);
                    tc::tma_load_3d(s.k[st], &tmK, &s.k_full[st], 0, blk.key0(j), bg);
                    last_phase[st] = (int)ph;
                }
                tc::mbar_wait(&s.q_full, 0, &zero);
                if (*abort)
                    for (int i = 0; i < KST; ++i)
                        if (last_phase[i] >= 0) tc::mbar_wait(&s.k_full[i], (uint32_t)last_phase[i], &zero);
            } else if (lane == 1) {
                int last_phase[VST];
                for (int i = 0; i < VST; ++i) last_phase[i] = -1;
                for (int j = 0; j < nblk; ++j) {
                    const int st = j % VST;
                    const uint32_t ph = (j / VST) & 1;
                    if (!tc::mbar_wait(&s.v_empty[st], ph ^ 1, abort, wlim)) { fail(abort, status, 0, j, 9); break; }
                    const int k0 = blk.key0(j);
                    tc::mbar_arrive_expect_tx(&s.v_full[st], KBLK * DV * 2);
#pragma unroll
                    for (int pnl = 0; pnl < DV / 64; ++pnl)
                        tc::tma_load_3d(s.v[st][pnl], &tmV, &s.v_full[st], pnl * 64, k0, bg);
                    last_phase[st] = (int)ph;
                }
                if (*abort)
                    for (int i = 0; i < VST; ++i)
                        if (last_phase[i] >= 0) tc::mbar_wait(&s.v_full[i], (uint32_t)last_phase[i], &zero);
            }
        } else if (warp == 1) {
            // ---------------- MMA issuer ----------------
            if (tc::elect_one()) {
                bool ok = tc::mbar_wait(&s.q_full, 0, abort, wlim);
                if (!ok) fail(abort, status, 1, 0, 0);
                const int n_t[2] = {blk.count(0), blk.count(1)};
                int jS[2] = {blk.nth(0, 0), blk.nth(1, 0)};  // union block of each tile's next S
                int jP[2] = {jS[0], jS[1]};                  // ... and of its next PV
                int uS[2] = {0, 0}, uP[2] = {0, 0};
                // S_t(u) = Q_t K_j^T; frees the K stage (two commits when the other tile
                // skips block j)
                auto issue_s = [&](int t) -> bool {
                    const int j = jS[t];
                    const int kst = j % KST;
                    if (!tc::mbar_wait(&s.k_full[kst], (j / KST) & 1, abort, wlim)) { fail(abort, status, 1, j, 2); return false; }
                    tc::tc_fence_after();
                    const uint32_t qa = tc::smem_u32(s.q[t]);
                    const uint32_t ka = tc::smem_u32(s.k[kst]);
                    const uint32_t sd = tmem + TM_S + t * 128;
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk)
                        tc::mma_f16_ss(sd, tc::sdesc_k_sw128(qa + kk * 32), tc::sdesc_k_sw128(ka + kk * 32), IDESC_S,
                                       kk > 0);
                    tc::mma_commit(&s.s_full[t]);
                    tc::mma_commit(&s.k_empty[kst]);
                    if (blk.users(j) == 1) tc::mma_commit(&s.k_empty[kst]);
                    ++uS[t];
                    int nj = jS[t] + 1;
                    while (nj < nblk && !blk.uses(t, nj)) ++nj;
                    jS[t] = uS[t] < n_t[t] ? nj : -1;
                    return true;
                };
                // O_t += P_t V_j, P_t read from TMEM (the tile's S columns)
                auto issue_pv = [&](int t) -> bool {
                    const int j = jP[t], u = uP[t];
                    const int vst = j % VST;
                    if (!tc::mbar_wait(&s.p_full[t], u & 1, abort, wlim)) { fail(abort, status, 1, j, 4 + t); return false; }
                    if (!tc::mbar_wait(&s.v_full[vst], (j / VST) & 1, abort, wlim)) { fail(abort, status, 1, j, 10); return false; }
                    tc::tc_fence_after();
                    const uint32_t va = tc::smem_u32(s.v[vst][0]);
                    const uint32_t pa = tmem + TM_S + t * 128;
#pragma unroll
                    for (int kk = 0; kk < KBLK / 16; ++kk)
                        mma_f16_ts(tmem + TM_O + t * 128, pa + kk * 8, tc::sdesc_mn_sw128(va + kk * 2048, KBLK * 128),
                                   IDESC_PV, (u > 0 || kk > 0));
                    tc::mma_commit(&s.pv_done[t]);
                    tc::mma_commit(&s.v_empty[vst]);
                    if (blk.users(j) == 1) tc::mma_commit(&s.v_empty[vst]);
                    ++uP[t];
                    int nj = jP[t] + 1;
                    while (nj < nblk && !blk.uses(t, nj)) ++nj;
                    jP[t] = uP[t] < n_t[t] ? nj : -1;
                    if (uP[t] == n_t[t]) tc::mma_commit(&s.o_done[t]);
                    return true;
                };
                for (int t = 0; ok && t < 2; ++t)
                    if (n_t[t] > 0) ok = issue_s(t);
                // then whatever is ready, tiles in turn: the PV of a tile once its softmax
                // wrote P, and its next S once that PV completed (S overwrites P)
                long long t_idle = 0;
                uint32_t spins = 0;
                while (ok && (uP[0] < n_t[0] || uP[1] < n_t[1])) {
                    bool progressed = false;
                    for (int t = 0; ok && t < 2; ++t) {
                        if (uP[t] < uS[t] && tc::mbar_test_wait(&s.p_full[t], uP[t] & 1) &&
                            tc::mbar_test_wait(&s.v_full[jP[t] % VST], (jP[t] / VST) & 1)) {
                            ok = issue_pv(t);
                            progressed = true;
                        }
                        if (ok && uS[t] < n_t[t] && uS[t] == uP[t] &&
                            tc::mbar_test_wait(&s.pv_done[t], (uP[t] - 1) & 1) &&
                            tc::mbar_test_wait(&s.k_full[jS[t] % KST], (jS[t] / KST) & 1)) {
                            ok = issue_s(t);
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        t_idle = 0;
                    } else if ((++spins & 255) == 0) {
                        const long long now = clock64();
                        if (*abort) ok = false;
                        else if (t_idle == 0) t_idle = now;
                        else if (now - t_idle > wlim) {
                            fail(abort, status, 1, uP[0] + uP[1], 11);
                            ok = false;
                        }
                    }
                }
                // drain: every MMA issued has completed before the block exits
                tc::mma_commit(&s.drain);
                int zero = 0;
                tc::mbar_wait(&s.drain, 0, &zero);
            }
        }
    } else {
        setmaxnreg_inc<REG_SOFT>();
        // ---------------- softmax + output: tile t, TMEM lane quadrant q ----------------
        const int t = (warp - 4) >> 2, q = warp & 3;
        const int r = q * 32 + lane;
        const int it0 = i0 + t * QT;
        const int i = it0 + r;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const uint32_t s_cols = tmem + lane_base + TM_S + t * 128;
        const uint32_t o_cols = tmem + lane_base + TM_O + t * 128;
        const float scale = LOG2E * 0.125f;  // log2(e) / sqrt(64)
        const int nt = blk.count(t);
        // the row's visible keys: meta [0, min(n_meta, i+1)), window [wa, i+1)
        const int meta_e = min(n_meta, i + 1);
        const int wa = window > 0 ? max(n_meta, i - window + 1) : n_meta;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        int j = -1;
        for (int u = 0; u < nt; ++u) {
            do { ++j; } while (!blk.uses(t, j));
            // tcgen05.ld/st are warp-collective: every decision that guards them is taken
            // by the whole warp (__all_sync / __any_sync)
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&s.s_full[t], u & 1, abort, wlim))) {
                if (lane == 0) fail(abort, status, 2, u, 5);
                ok = false;
                break;
            }
            tc::tc_fence_after();
            // the four 32-column loads in flight together, one wait
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld32(s_cols + c * 32, sr[c]);
            tc::tmem_wait_ld();
            float* sv = reinterpret_cast<float*>(&sr[0][0]);
            // mask: the keys row i sees in this block form one interval [a, e)
            const int k0 = blk.key0(j);
            const bool meta_blk = j < blk.nmb;
            const int a = meta_blk ? 0 : wa;
            const int e = meta_blk ? meta_e : i + 1;
            if (a > k0 || e < k0 + KBLK) {
                const unsigned span = e > a ? (unsigned)(e - a) : 0u;
#pragma unroll
                for (int c = 0; c < 128; ++c) sv[c] = (unsigned)(k0 + c - a) < span ? sv[c] : -INFINITY;
            }
            // row max with three-input max: 8 independent chains over the 128 scores
            float mx8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx8[c] = fmax3(sv[c], sv[c + 8], sv[c + 16]);
#pragma unroll
            for (int c = 24; c + 16 < 128; c += 16)
#pragma unroll
                for (int x = 0; x < 8; ++x) mx8[x] = fmax3(mx8[x], sv[c + x], sv[c + 8 + x]);
#pragma unroll
            for (int x = 0; x < 8; ++x) mx8[x] = fmaxf(mx8[x], sv[120 + x]);
            const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                   fmaxf(mx8[6], mx8[7])) * scale;
            // a row whose running max grows by more than 2^8 moves to the new max; its O
            // (PV of the earlier blocks, all completed: this S was issued after the last
            // PV of the tile completed) is scaled in TMEM once P is stored (before the PV
            // of this block is released)
            float f = 1.f;
            bool scale_o = false;
            if (mx > m_used + RESCALE_LOG2) {
                if (m_used != -INFINITY) {
                    f = exp2f(m_used - mx);
                    l *= f;
                    scale_o = true;
                }
                m_used = mx;
            }
            // P = 2^(s * scale - m) in fp32, summed in fp32, stored as fp16 pairs
            const float mu = m_used == -INFINITY ? 0.f : m_used;
            const float2 sc2 = make_float2(scale, scale), nmu2 = make_float2(-mu, -mu);
            uint32_t pk[64];
            float2 l4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float2 x = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nmu2);
                const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                l4[c & 3] = __fadd2_rn(l4[c & 3], p);
                pk[c] = pack_f16x2(p.x, p.y);
            }
            const float2 l2 = __fadd2_rn(__fadd2_rn(l4[0], l4[1]), __fadd2_rn(l4[2], l4[3]));
            l += l2.x + l2.y;
            tmem_st64(s_cols, pk);
            tc::tmem_wait_st();
            if (__any_sync(0xffffffffu, scale_o)) {
                uint32_t rr[DV / 32][32];
#pragma unroll
                for (int c = 0; c < DV / 32; ++c) tc::tmem_ld32(o_cols + c * 32, rr[c]);
                tc::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < DV / 32; ++c) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) rr[c][x] = __float_as_uint(__uint_as_float(rr[c][x]) * f);
                    tc::tmem_st32(o_cols + c * 32, rr[c]);
                }
                tc::tmem_wait_st();
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&s.p_full[t]);
        }
        if (ok && nt > 0 && __all_sync(0xffffffffu, tc::mbar_wait(&s.o_done[t], 0, abort, wlim))) {
            tc::tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            f16* orow = O + ((long long)b * Tp + i) * ((long long)H * DV) + h * DV;
#pragma unroll 1
            for (int c = 0; c < DV / 32; ++c) {
                uint32_t rr[32];
                tc::tmem_ld32(o_cols + c * 32, rr);
                tc::tmem_wait_ld();
                if (i < Tp) {
#pragma unroll
                    for (int x = 0; x < 32; x += 8) {
                        uint4 pk;
                        pk.x = pack_f16x2(__uint_as_float(rr[x]) * inv, __uint_as_float(rr[x + 1]) * inv);
                        pk.y = pack_f16x2(__uint_as_float(rr[x + 2]) * inv, __uint_as_float(rr[x + 3]) * inv);
                        pk.z = pack_f16x2(__uint_as_float(rr[x + 4]) * inv, __uint_as_float(rr[x + 5]) * inv);
                        pk.w = pack_f16x2(__uint_as_float(rr[x + 6]) * inv, __uint_as_float(rr[x + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + x) = pk;
                    }
                }
            }
        } else if (ok && nt > 0) {
            if (lane == 0) fail(abort, status, 2, nt, 8);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

template <int DV>
int launch_dv(const Ctx& ctx, const f16* P, long long ldP, const f16* k_seq, const f16* v_seq, int kcap, f16* O,
              int B, int Tp, int H, int G, int n_meta, int window) {
    CUtensorMap tq, tk, tv;
    // Q: P viewed as [B][Tp][ldP]; K: [B*G][Tp][64]; V: [B*G][Tp][DV] (rows >= Tp read as 0)
    if (!tc::make_tmap_3d(&tq, P, false, B, Tp, (uint64_t)H * DH, ldP, (uint64_t)Tp * ldP, QT) ||
        !tc::make_tmap_3d(&tk, k_seq, false, (uint64_t)B * G, Tp, DH, DH, (uint64_t)kcap * DH, KBLK) ||
        !tc::make_tmap_3d(&tv, v_seq, false, (uint64_t)B * G, Tp, DV, DV, (uint64_t)kcap * DV, KBLK))
        return HYMBA_ERR_UNSUPPORTED;
    auto kern = attn_prefill_tc_kernel<DV>;
    const size_t smem = sizeof(AttnSmem<DV>) + 1024;
    static std::atomic<unsigned long long> smem_set{0};
    if (!smem_opt_in_once(smem_set, kern, smem, ctx)) return HYMBA_ERR_CUDA;
    // the warpgroups' register split (setmaxnreg) must fit the registers the block is
    // launched with, or the increase would wait forever: check the compiled count
    static std::atomic<int> regs{0};
    if (regs.load(std::memory_order_relaxed) == 0) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return HYMBA_ERR_CUDA;
        regs.store(fa.numRegs, std::memory_order_relaxed);
    }
    if (4 * 32 * REG_OTHER + 8 * 32 * REG_SOFT > NTHREADS * regs.load(std::memory_order_relaxed))
        return HYMBA_ERR_UNSUPPORTED;
    const int n_pairs = ceil_div(Tp, 2 * QT);
    dim3 grid(H, B, n_pairs);
    HYMBA_LAUNCH(ctx, "attn_prefill", kern, grid, NTHREADS, smem, tq, tk, tv, O, Tp, H, G, n_meta, window,
                 n_pairs, ctx.status);
    return HYMBA_OK;
}

}  // namespace

int launch_attn_prefill_tc(const Ctx& ctx, const f16* P, long long ldP, const f16* k_seq, const f16* v_seq,
                           int kcap, f16* O, int B, int Tp, int H, int G, int dv, int n_meta, int window) {
    if (dv == 128) return launch_dv<128>(ctx, P, ldP, k_seq, v_seq, kcap, O, B, Tp, H, G, n_meta, window);
    if (dv == 64) return launch_dv<64>(ctx, P, ldP, k_seq, v_seq, kcap, O, B, Tp, H, G, n_meta, window);
    return HYMBA_ERR_UNSUPPORTED;
}

}  // namespace hymba
