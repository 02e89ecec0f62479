// Projection GEMM C = A B^T on the 5th-generation tensor cores (tcgen05), used for
// the fused input projection, the Delta projection and the output projection of the
// mixer ("Hymba Guide", Parallel Hybrid-Head Layer Formulation: one projection
// feeds both head families, one output projection mixes them).
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0      TMA producer: 128 x 64 A box and BN x 64 B box per k-block into a
//               4-stage ring of 128-byte-swizzled shared-memory tiles;
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 x tcgen05.mma
//               (128 x BN x 16) per k-block into a TMEM accumulator;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (32 rows per warp) in runs of
//               64 columns, then the layer's epilogue (RoPE, K/V scatter, softplus,
//               residual) and the stores.
// The accumulator is double-buffered in TMEM so the epilogue of one tile overlaps the
// MMAs of the next. Every mbarrier wait is bounded; on timeout the CTA records
// HYMBA_ERR_DEVICE_TIMEOUT, drains what it issued and exits.
#include <algorithm>

#include "kernels.h"
#include "tc.cuh"

namespace hymba {

namespace tc {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, bool is_bf16, uint64_t rows, uint64_t cols, uint64_t ld,
                  uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || ((uintptr_t)base & 15) || (ld * 2) % 16) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, is_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, const void* base, bool is_bf16, uint64_t planes, uint64_t rows,
                  uint64_t cols, uint64_t ld, uint64_t plane_ld, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || ((uintptr_t)base & 15) || (ld * 2) % 16 || (plane_ld * 2) % 16) return false;
    cuuint64_t dims[3] = {cols, rows, planes};
    cuuint64_t strides[2] = {ld * 2, plane_ld * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, is_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc

namespace {

constexpr int BM = 128, BK = 64, NUM_THREADS = 192;

// STAGES-deep operand ring; GEMMs of at most two k-blocks use two stages, which leaves
// room for two CTAs per SM (their epilogues, the bulk of such a GEMM, then overlap)
template <int BN, int STAGES>
struct GemmSmem {
    alignas(1024) uint8_t a[STAGES][BM * BK * 2];
    alignas(1024) uint8_t b[STAGES][BN * BK * 2];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    alignas(16) uint8_t stage[4][kStageWarpBytes];  // epilogue warps' store staging
    RunDst info[4][32];
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void fail(volatile int* abort, int* status, int role, int step, int bar) {
    *abort = 1;
    tc::record_timeout(status, role, step, bar);
}

// Tile order: groups of GM row blocks, each walked column block by column block (row
// blocks fastest), so the CTAs in flight share a few A row panels and a run of B
// column panels, and both stay in L2 while they are reused (a plain row-fastest order
// streams the whole A once per column block, which no longer fits in L2 for long
// batches).
constexpr int GM = 8;
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int* m_blk, int* n_blk) {
    const int group = tile / (GM * num_n);
    const int first_m = group * GM;
    const int gsize = min(GM, num_m - first_m);
    const int local = tile - group * GM * num_n;
    *m_blk = first_m + local % gsize;
    *n_blk = local / gsize;
}

// KIND >= 0: the epilogue kind fixed at compile time, and DEC its decode form (the decode
// projections, whose launches follow kernels that stream far more than L2 holds: a
// smaller kernel refetches less code); KIND < 0: the kind from the arguments.
template <typename TA, typename TO, int BN, int STAGES, int KIND = -1, bool DEC = false>
__global__ void __launch_bounds__(NUM_THREADS, STAGES == 2 ? 2 : 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmA0, int M0, int M, int N, int K, int ksplit, EpiArgs<TO> e,
               int* status) {
    extern __shared__ uint8_t smem_raw[];
    GemmSmem<BN, STAGES>& s = *reinterpret_cast<GemmSmem<BN, STAGES>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                        ~static_cast<uintptr_t>(1023));
    constexpr bool kBF16 = sizeof(TA) == 2 && std::is_same<TA, bf16>::value;
    constexpr uint32_t IDESC = tc::idesc_f16(kBF16, BM, BN);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // M-blocks [0, num_m0) come from the optional second operand A0 (M0 rows), the
    // rest from A (M rows); the epilogue tells them apart by row index (EpiArgs::meta_pad)
    const int num_m0 = (M0 + BM - 1) / BM;
    const int num_m = num_m0 + (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
    // split-K: tile index = output tile * ksplit + split; split s covers k-blocks
    // [s nk / ksplit, (s + 1) nk / ksplit) and adds its partial sum to the output
    const int num_tiles = num_m * num_n * ksplit, nk = (K + BK - 1) / BK;
    auto krange = [&](int tile, int* kb0, int* kb1) {
        const int sp = tile % ksplit;
        *kb0 = sp * nk / ksplit;
        *kb1 = (sp + 1) * nk / ksplit;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            tc::mbar_init(&s.full[i], 1);
            tc::mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&s.tfull[i], 1);
            tc::mbar_init(&s.tempty[i], 128);
        }
        tc::mbar_init(&s.drain, 1);
        s.abort = 0;
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tmA);
        tc::prefetch_tmap(&tmB);
        if (M0 > 0) tc::prefetch_tmap(&tmA0);
    }
    if (warp == 1) {
        tc::tmem_alloc(&s.tmem_base, 2 * BN);
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

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (tc::elect_one()) {
            int it = 0;
            int issued_phase[STAGES];
            for (int i = 0; i < STAGES; ++i) issued_phase[i] = -1;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort; tile += gridDim.x) {
                int m_blk, n_blk, kb0, kb1;
                tile_coords(tile / ksplit, num_m, num_n, &m_blk, &n_blk);
                krange(tile, &kb0, &kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int st = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!tc::mbar_wait(&s.empty[st], ph ^ 1, abort, wlim)) { fail(abort, status, 0, kb, 1); break; }
                    tc::mbar_arrive_expect_tx(&s.full[st], (BM + BN) * BK * 2);
                    if (m_blk < num_m0) tc::tma_load_2d(s.a[st], &tmA0, &s.full[st], kb * BK, m_blk * BM);
                    else tc::tma_load_2d(s.a[st], &tmA, &s.full[st], kb * BK, (m_blk - num_m0) * BM);
                    tc::tma_load_2d(s.b[st], &tmB, &s.full[st], kb * BK, n_blk * BN);
                    issued_phase[st] = (int)ph;
                }
            }
            if (*abort) {
                // let the copies this thread issued land before the CTA exits
                int zero = 0;
                for (int i = 0; i < STAGES; ++i)
                    if (issued_phase[i] >= 0) tc::mbar_wait(&s.full[i], (uint32_t)issued_phase[i], &zero);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (tc::elect_one()) {
            int it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort; tile += gridDim.x, ++tcount) {
                const int buf = tcount & 1;
                const uint32_t tph = (tcount >> 1) & 1;
                if (!tc::mbar_wait(&s.tempty[buf], tph ^ 1, abort, wlim)) { fail(abort, status, 1, tcount, 4); break; }
                tc::tc_fence_after();
                const uint32_t d = tmem + buf * BN;
                bool ok = true;
                int kb0, kb1;
                krange(tile, &kb0, &kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int st = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!tc::mbar_wait(&s.full[st], ph, abort, wlim)) { fail(abort, status, 1, kb, 2); ok = false; break; }
                    tc::tc_fence_after();
                    const uint32_t a0 = tc::smem_u32(s.a[st]), b0 = tc::smem_u32(s.b[st]);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc::mma_f16_ss(d, tc::sdesc_k_sw128(a0 + kk * 32), tc::sdesc_k_sw128(b0 + kk * 32), IDESC,
                                       (kb != kb0 || kk != 0));
                    tc::mma_commit(&s.empty[st]);
                }
                if (!ok) break;
                tc::mma_commit(&s.tfull[buf]);
            }
            // all MMAs issued by this thread have completed once `drain` flips
            tc::mma_commit(&s.drain);
            int zero = 0;
            tc::mbar_wait(&s.drain, 0, &zero);
        }
    } else {
        // ---------------- epilogue (warps 2..5 -> TMEM lane quadrants 2, 3, 0, 1) ----------------
        const int q = warp & 3;
        int tcount = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
            const int buf = tcount & 1;
            const uint32_t tph = (tcount >> 1) & 1;
            // tcgen05.ld is warp-collective: the whole warp decides together
            if (!__all_sync(0xffffffffu, tc::mbar_wait(&s.tfull[buf], tph, abort, wlim))) { fail(abort, status, 2, tcount, 3); break; }
            tc::tc_fence_after();
            int m_blk, n_blk;
            tile_coords(tile / ksplit, num_m, num_n, &m_blk, &n_blk);
            const int row = m_blk * BM + q * 32 + lane;
#pragma unroll 1
            for (int j = 0; j < BN / 64; ++j) {
                uint32_t r0[32], r1[32];
                const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + buf * BN + j * 64;
                tc::tmem_ld32(taddr, r0);
                tc::tmem_ld32(taddr + 32, r1);
                tc::tmem_wait_ld();
                float v[64];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    v[i] = __uint_as_float(r0[i]);
                    v[32 + i] = __uint_as_float(r1[i]);
                }
                const RunDst d = epi_prepare64<TO, KIND, DEC>(e, row, n_blk * BN + j * 64, v);
                epi_store_staged<TO>(d, v, s.stage[q], s.info[q], lane);
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&s.tempty[buf]);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 2 * BN);
    }
}

template <typename TA, typename TO, int BN, int STAGES, int KIND = -1, bool DEC = false>
int launch_bn(const Ctx& ctx, const char* name, const TA* A, long long lda, const TA* Bw, long long ldb, int M,
              int N, int K, const EpiArgs<TO>& e, const TA* A0, int M0, int ksplit) {
    constexpr bool kBF16 = std::is_same<TA, bf16>::value;
    CUtensorMap ta, tb, ta0;
    if (!tc::make_tmap_2d(&ta, A, kBF16, M, K, lda, BM)) return HYMBA_ERR_UNSUPPORTED;
    if (!tc::make_tmap_2d(&tb, Bw, kBF16, N, K, ldb, BN)) return HYMBA_ERR_UNSUPPORTED;
    if (M0 > 0) {
        if (!tc::make_tmap_2d(&ta0, A0, kBF16, M0, K, lda, BM)) return HYMBA_ERR_UNSUPPORTED;
    } else {
        ta0 = ta;
    }
    const size_t smem = sizeof(GemmSmem<BN, STAGES>) + 1024;
    auto kern = gemm_tc_kernel<TA, TO, BN, STAGES, KIND, DEC>;
    static std::atomic<unsigned long long> smem_set{0};
    if (!smem_opt_in_once(smem_set, kern, smem, ctx)) return HYMBA_ERR_CUDA;
    const int tiles = ((M0 + BM - 1) / BM + (M + BM - 1) / BM) * ((N + BN - 1) / BN) * ksplit;
    const int slots = ctx.sm_count * (STAGES == 2 ? 2 : 1);
    const int grid = tiles < slots ? tiles : slots;
    EpiArgs<TO> e2 = e;
    e2.meta_pad = ((M0 + BM - 1) / BM) * BM;
    e2.meta_M = M0;
    HYMBA_LAUNCH(ctx, name, kern, grid, NUM_THREADS, smem, ta, tb, ta0, M0, M, N, K, ksplit, e2, ctx.status);
    return HYMBA_OK;
}

}  // namespace

// Tile width: the BN in {256, 128, 64} with the least estimated time, counting whole
// waves of persistent CTAs and the lower operand reuse of narrow tiles.
static int pick_bn(int M, int N, int sms) {
    int best = 256;
    double best_cost = 1e30;
    for (int bn : {256, 128, 64}) {
        const long long tiles = (long long)((M + BM - 1) / BM) * ((N + bn - 1) / bn);
        const long long waves = (tiles + sms - 1) / sms;
        // narrower tiles re-read the operands more often from L2: per unit of work a
        // 128-wide tile runs about 1.25x and a 64-wide one 1.9x slower than a 256-wide one
        // (the in-projection measured at 958 and 1105 TFLOP/s for 128 and 256)
        const double cost = (double)waves * bn * (bn == 256 ? 1.0 : bn == 128 ? 1.25 : 1.9);
        if (cost < best_cost - 1e-9) { best_cost = cost; best = bn; }
    }
    return best;
}

template <typename TA, typename TO>
int launch_gemm_tc(const Ctx& ctx, const char* name, const TA* A, long long lda, const TA* Bw, long long ldb,
                   int M, int N, int K, const EpiArgs<TO>& e, const TA* A0, int M0) {
    if (M <= 0 || N <= 0) return HYMBA_OK;
    if (M0 > 0 && (!A0 || ((uintptr_t)A0 & 15))) return HYMBA_ERR_INVALID_ARG;
    const int sms = ctx.sm_count > 0 ? ctx.sm_count : 148;
    if (e.accumulate) {
        // split-K into an fp32 output that holds the rest of the sum: 64-wide tiles, and
        // as many splits as fill the SMs (a few rows x a long K, the decode projections)
        if (sizeof(TO) != 4 || e.kind != EPI_OUT || M0 > 0) return HYMBA_ERR_INVALID_ARG;
        const int tiles = ((M + BM - 1) / BM) * ((N + 63) / 64), nk = (K + BK - 1) / BK;
        const int ksplit = std::max(1, std::min(nk, sms / std::max(1, tiles)));
        return launch_bn<TA, TO, 64, 4, EPI_OUT, true>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, ksplit);
    }
    switch (pick_bn(M + M0, N, sms)) {
        case 256: return launch_bn<TA, TO, 256, 4>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, 1);
        case 128:
            if (K <= 2 * BK) return launch_bn<TA, TO, 128, 2>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, 1);
            return launch_bn<TA, TO, 128, 4>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, 1);
        default:
            if (K <= 2 * BK) return launch_bn<TA, TO, 64, 2>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, 1);
            // one row block streaming a long K (decode): a deeper ring keeps more weight
            // tiles in flight per CTA
            if (M + M0 <= BM && K > 4 * BK) {
                if (e.kind == EPI_INPROJ && e.row_mode == ROWS_DECODE && M0 == 0)
                    return launch_bn<TA, TO, 64, 8, EPI_INPROJ, true>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, 1);
                return launch_bn<TA, TO, 64, 8>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, 1);
            }
            return launch_bn<TA, TO, 64, 4>(ctx, name, A, lda, Bw, ldb, M, N, K, e, A0, M0, 1);
    }
}

#define INST(TA, TO)                                                                                        \
    template int launch_gemm_tc<TA, TO>(const Ctx&, const char*, const TA*, long long, const TA*, long long, \
                                        int, int, int, const EpiArgs<TO>&, const TA*, int);
INST(bf16, f16)
INST(f16, f16)
INST(bf16, bf16)
INST(bf16, float)
INST(f16, float)
INST(f16, bf16)
#undef INST

}  // namespace hymba
