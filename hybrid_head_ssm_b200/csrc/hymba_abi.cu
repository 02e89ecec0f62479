// The C ABI of libhymba.so: argument checks, workspace planning, and the order of
// kernel launches of one mixer layer (prefill and decode). Every step of the layer
// runs in the kernels of this library; this file only queues them on the caller's
// stream.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <type_traits>
#include <mutex>
#include <vector>

#include "kernels.h"

namespace hymba {

// ---------------------------------------------------------------------------
// device status word (one per device that loads the library)
// ---------------------------------------------------------------------------
// [0]: status code; [1..7]: where the first timed-out wait gave up (flag, block
// x, y, z, role, step, barrier), for diagnosis; [8..9]: the limit in cycles of the
// kernels' progress waits (0: the default), set by hymba_debug_set_wait_limit.
__device__ __align__(8) int g_status_word[10];

static std::mutex g_mu;
// Per device: the status word's device address and the SM count, published together.
// A reader that sees the pointer (acquire) also sees the SM count written before it
// (release), so no caller can launch with a zero grid.
static std::atomic<int*> g_status_ptr[64];
static int g_sm_count[64];

static int current_ctx(cudaStream_t stream, Ctx* ctx) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HYMBA_ERR_CUDA;
    int* status = g_status_ptr[dev].load(std::memory_order_acquire);
    if (!status) {
        std::lock_guard<std::mutex> lk(g_mu);
        status = g_status_ptr[dev].load(std::memory_order_relaxed);
        if (!status) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return HYMBA_ERR_CUDA;
            int sms = 0;
            if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
                return HYMBA_ERR_CUDA;
            g_sm_count[dev] = sms;
            status = static_cast<int*>(p);
            g_status_ptr[dev].store(status, std::memory_order_release);
        }
    }
    ctx->stream = stream;
    ctx->status = status;
    ctx->sm_count = g_sm_count[dev];
    ctx->device = dev;
    return HYMBA_OK;
}

int launch_context(cudaStream_t stream, Ctx* ctx) { return current_ctx(stream, ctx); }

// ---------------------------------------------------------------------------
// tracing and launch counting
// ---------------------------------------------------------------------------
struct TraceRec {
    cudaEvent_t a, b;
    const char* name;
};
static constexpr int kTracePool = 8192;
static std::atomic<int> g_trace_on{0};
static std::atomic<unsigned long long> g_launches{0};
static std::vector<TraceRec> g_trace;
static std::atomic<int> g_trace_used{0};
static thread_local int t_trace_slot = -1;

static char g_trace_only[64] = {0};  // non-empty: trace only launches of this name

void trace_before(const Ctx& ctx, const char* name) {
    t_trace_slot = -1;
    if (!g_trace_on.load(std::memory_order_relaxed)) return;
    if (g_trace_only[0] && strcmp(g_trace_only, name) != 0) return;
    const int slot = g_trace_used.fetch_add(1);
    if (slot >= (int)g_trace.size()) return;
    t_trace_slot = slot;
    cudaEventRecord(g_trace[slot].a, ctx.stream);
}

// HYMBA_SYNC_DEBUG=1: synchronise after every launch and log it to stderr (a
// debugging aid: it serialises the host with the device).
static int sync_debug() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("HYMBA_SYNC_DEBUG");
        v = (e && e[0] == '1') ? 1 : 0;
    }
    return v;
}

bool trace_after(const Ctx& ctx, const char* name) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (sync_debug()) {
        fprintf(stderr, "[hymba] launched %s\n", name);
        fflush(stderr);
        const cudaError_t e2 = cudaStreamSynchronize(ctx.stream);
        int st = 0;
        cudaMemcpy(&st, ctx.status, sizeof(int), cudaMemcpyDeviceToHost);
        fprintf(stderr, "[hymba] finished %s: %s, status %d\n", name, cudaGetErrorString(e2), st);
        fflush(stderr);
    }
    const cudaError_t err = cudaGetLastError();
    if (t_trace_slot >= 0) {
        g_trace[t_trace_slot].name = name;
        cudaEventRecord(g_trace[t_trace_slot].b, ctx.stream);
        t_trace_slot = -1;
    }
    return err != cudaSuccess;
}

// ---------------------------------------------------------------------------
// configuration checks and workspace plan
// ---------------------------------------------------------------------------
static int check_cfg(const hymba_layer_cfg* c) {
    if (!c) return HYMBA_ERR_INVALID_ARG;
    if (c->d_model <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->d_inner <= 0 ||
        c->dt_rank <= 0 || c->n_meta < 0 || (c->dtype != HYMBA_F32 && c->dtype != HYMBA_BF16) ||
        !(c->rms_eps >= 0.f) || !(c->rope_base > 0.f))
        return HYMBA_ERR_INVALID_ARG;
    if (c->head_dim != 64 || c->d_state != 16 || c->d_conv != 4) return HYMBA_ERR_UNSUPPORTED;
    if (c->n_q_heads % c->n_kv_heads) return HYMBA_ERR_UNSUPPORTED;
    if (c->n_q_heads / c->n_kv_heads > 8) return HYMBA_ERR_UNSUPPORTED;
    if (c->fusion != HYMBA_FUSION_AVERAGE && c->fusion != HYMBA_FUSION_CONCAT) return HYMBA_ERR_INVALID_ARG;
    if (c->v_head_dim != 128 && c->v_head_dim != 64) return HYMBA_ERR_UNSUPPORTED;
    const int hv = c->v_head_dim * c->n_q_heads;
    if (c->fusion == HYMBA_FUSION_AVERAGE && hv != c->d_inner) return HYMBA_ERR_UNSUPPORTED;
    if (c->d_model % 64 || c->d_inner % 64 || hv % 64) return HYMBA_ERR_UNSUPPORTED;
    if (c->d_inner > 4096 || hv > 4096) return HYMBA_ERR_UNSUPPORTED;
    if (c->ssm_heads < 0 || (c->ssm_heads > 0 && c->d_inner % c->ssm_heads)) return HYMBA_ERR_INVALID_ARG;
    if (c->ssm_heads > 0) {
        const int hp = c->d_inner / c->ssm_heads;
        if (hp % 8) return HYMBA_ERR_UNSUPPORTED;
        if (c->dtype == HYMBA_BF16 && !ssd_scan_applies(c->d_inner, c->ssm_heads)) return HYMBA_ERR_UNSUPPORTED;
    }
    return HYMBA_OK;
}

// Rows of W_dt: one per channel, or one per SSM head in the SSD form.
static int n_dt(const hymba_layer_cfg* c) { return c->ssm_heads > 0 ? c->ssm_heads : c->d_inner; }
// Channels per SSM head (0: the selective form).
static int ssm_hp(const hymba_layer_cfg* c) { return c->ssm_heads > 0 ? c->d_inner / c->ssm_heads : 0; }

// Width of the fused branches, the input of W_o.
static int u_width(const hymba_layer_cfg* c) {
    return c->fusion == HYMBA_FUSION_CONCAT ? c->d_inner + c->n_q_heads * c->v_head_dim : c->d_inner;
}

struct Cols {
    int n_in, x, z, dtl, Bc, Cc;
};

static Cols columns(const hymba_layer_cfg* c) {
    Cols k;
    const int q = c->n_q_heads * c->head_dim;
    const int kv = c->is_kv_producer ? c->n_kv_heads * (c->head_dim + c->v_head_dim) : 0;
    k.x = q + kv;
    k.z = k.x + c->d_inner;
    k.Bc = k.z + c->d_inner;
    k.Cc = k.Bc + c->d_state;
    k.dtl = k.Cc + c->d_state;
    k.n_in = k.dtl + c->dt_rank;
    return k;
}

struct Plan {
    size_t total = 0;
    size_t rope = 0, P = 0, delta = 0, O = 0, ypre = 0, U = 0, wdt = 0, part = 0, xcv = 0;
    size_t win16 = 0, meta16 = 0, wout16 = 0;
    long long ldP = 0;
    int rpad = 0, n_split = 1;
};

static size_t take(size_t* cur, size_t bytes) {
    const size_t off = *cur;
    *cur += (bytes + 255) / 256 * 256;
    return off;
}

// 128-key splits: the 16-bit decode attention streams each split through its shared
// memory ring in one K tile and two V tiles, and more, shorter blocks fill the waves
static int decode_splits(int cache_cap) { return ceil_div(cache_cap > 0 ? cache_cap : 1, 128); }

static Plan plan(const hymba_layer_cfg* c, int B, int T, int mode) {
    Plan p;
    const size_t esz = c->dtype == HYMBA_BF16 ? 2 : 4;
    const Cols k = columns(c);
    const long long rows = mode == HYMBA_MODE_PREFILL ? (long long)B * (c->n_meta + T) : B;
    const int di = c->d_inner;
    p.ldP = round_up(k.n_in, 64);
    p.rpad = (int)round_up(c->dt_rank, 64);
    size_t cur = 0;
    // RoPE table: prefill, one row per position; decode, one row per sequence
    p.rope = take(&cur, (size_t)(mode == HYMBA_MODE_PREFILL ? c->n_meta + T : B) * 32 * sizeof(float2));
    p.P = take(&cur, rows * p.ldP * esz);
    p.delta = take(&cur, rows * di * sizeof(float));
    p.O = take(&cur, rows * (size_t)c->n_q_heads * c->v_head_dim * esz);
    p.ypre = take(&cur, rows * di * esz);
    p.U = take(&cur, rows * u_width(c) * esz);
    p.wdt = take(&cur, (size_t)di * p.rpad * esz);
    // the projection's copy of the input rows: converted to 16 bits (fp32 stream of a
    // bf16 layer) or RMS-normalised (HYMBA_PRE_NORM)
    p.xcv = take(&cur, rows * c->d_model * esz);
    if (c->dtype == HYMBA_BF16) {
        if (mode == HYMBA_MODE_PREFILL) {
            // fp16 copies of the projection weights for fp32-stream calls (and of W_out
            // for the concat fusion)
            p.win16 = take(&cur, (size_t)k.n_in * c->d_model * 2);
            p.meta16 = take(&cur, (size_t)c->n_meta * c->d_model * 2);
            p.wout16 = take(&cur, (size_t)c->d_model * u_width(c) * 2);
        } else if (c->fusion == HYMBA_FUSION_CONCAT) {
            p.wout16 = take(&cur, (size_t)c->d_model * u_width(c) * 2);
        }
    }
    if (mode == HYMBA_MODE_DECODE) {
        p.n_split = decode_splits(T);
        p.part = take(&cur, (size_t)B * c->n_q_heads * p.n_split * (c->v_head_dim + 4) * sizeof(float));
    }
    p.total = cur;
    return p;
}

// ---------------------------------------------------------------------------
// dispatch: tcgen05 for 16-bit operands, CUDA cores for fp32
// ---------------------------------------------------------------------------
// Whether gemm() takes the tensor-core path for these operands.
template <typename TA>
static bool tc_gemm_ok(const TA* A, long long lda, const TA* W, long long ldw) {
#ifdef HYMBA_WITH_TCGEN05
    return sizeof(TA) == 2 && ((uintptr_t)A & 15) == 0 && ((uintptr_t)W & 15) == 0 && lda % 8 == 0 && ldw % 8 == 0;
#else
    (void)A; (void)lda; (void)W; (void)ldw;
    return false;
#endif
}

template <typename TA, typename TO>
static int gemm(const Ctx& ctx, const char* name, const TA* A, long long lda, const TA* W, long long ldw,
                int M, int N, int K, const EpiArgs<TO>& e) {
#ifdef HYMBA_WITH_TCGEN05
    if constexpr (sizeof(TA) == 2) {
        if (tc_gemm_ok(A, lda, W, ldw)) return launch_gemm_tc<TA, TO>(ctx, name, A, lda, W, ldw, M, N, K, e);
    }
#endif
    return launch_gemm_simt<TA, TO>(ctx, name, A, lda, W, ldw, M, N, K, e);
}

template <typename I>
static int attn_prefill(const Ctx& ctx, const I* P, long long ldP, const I* k, const I* v, int kcap,
                        I* O, int B, int Tp, int H, int G, int dv, int n_meta, int window) {
#ifdef HYMBA_WITH_TCGEN05_ATTN
    if constexpr (sizeof(I) == 2) {
        if (ldP % 8 == 0 && kcap % 8 == 0)
            return launch_attn_prefill_tc(ctx, P, ldP, k, v, kcap, O, B, Tp, H, G, dv, n_meta, window);
    }
#endif
    return launch_attn_prefill_simt<I>(ctx, P, ldP, k, v, kcap, O, B, Tp, H, G, dv, n_meta, window);
}

template <typename T>
static EpiArgs<T> epi_base(int kind, int M, int N) {
    EpiArgs<T> e;
    memset(&e, 0, sizeof(e));
    e.kind = kind;
    e.M = M;
    e.N = N;
    return e;
}

// The V half of a consumer's affine adaptation of the shared K/V (NULL: plain sharing).
static const float* vscale(const hymba_layer_cfg* c, const hymba_layer_weights* w) {
    return (!c->is_kv_producer && w->kv_scale) ? w->kv_scale + c->n_kv_heads * c->head_dim : nullptr;
}
static const float* vbias(const hymba_layer_cfg* c, const hymba_layer_weights* w) {
    return (!c->is_kv_producer && w->kv_bias) ? w->kv_bias + c->n_kv_heads * c->head_dim : nullptr;
}

// T: the layer's I/O and weight type (fp32 or bf16). I: its intermediate type
// (fp32, or fp16 for bf16 layers: the projection, K/V, attention output and y_pre are
// held in fp16, which has the same width as bf16 and a finer mantissa).
// TIO: type of x and y (T, or fp32 for a bf16 layer in a fp32 residual stream).
// A bf16 layer in an fp32 residual stream takes the operands of its in- and
// output projections in fp16: the stream and U are rounded to fp16 (8x finer than
// bf16) and W_in, meta and W_out are converted per call (exact for all but the
// tiniest weights). The stream's values at depth are several times larger than the
// first layer's, and the attention scores they feed are correspondingly sharper.
template <typename T, typename I, typename TIO>
static int prefill_impl(const Ctx& ctx, const hymba_layer_cfg* c, const hymba_layer_weights* w,
                        const TIO* x_io, int B, int T_, int flags, TIO* y, hymba_kv* kv,
                        hymba_ssm_state* st, char* ws) {
    constexpr bool kF16Ops = std::is_same<T, bf16>::value && std::is_same<TIO, float>::value;
    using TA = typename std::conditional<kF16Ops, f16, T>::type;
    const Plan pl = plan(c, B, T_, HYMBA_MODE_PREFILL);
    const Cols k = columns(c);
    const int m = c->n_meta, Tp = m + T_, d = c->d_model, di = c->d_inner, uw = u_width(c);
    const int H = c->n_q_heads, G = c->n_kv_heads, dh = c->head_dim, dv = c->v_head_dim;
    const long long rows = (long long)B * Tp;
    const bool has_meta = flags & HYMBA_X_HAS_META;
    float2* rope = reinterpret_cast<float2*>(ws + pl.rope);
    I* P = reinterpret_cast<I*>(ws + pl.P);
    float* delta = reinterpret_cast<float*>(ws + pl.delta);
    I* O = reinterpret_cast<I*>(ws + pl.O);
    I* ypre = reinterpret_cast<I*>(ws + pl.ypre);
    TA* U = reinterpret_cast<TA*>(ws + pl.U);
    I* wdt = reinterpret_cast<I*>(ws + pl.wdt);
    I* k_seq = static_cast<I*>(kv->k_seq);
    I* v_seq = static_cast<I*>(kv->v_seq);
    int rc;

    const TA *x, *W_in, *meta, *W_out;
    const bool pre_norm = flags & HYMBA_PRE_NORM;
    TA* xn = reinterpret_cast<TA*>(ws + pl.xcv);
    if constexpr (kF16Ops) {
        TA* wi = reinterpret_cast<TA*>(ws + pl.win16);
        TA* mt = reinterpret_cast<TA*>(ws + pl.meta16);
        TA* wo = reinterpret_cast<TA*>(ws + pl.wout16);
        const int xrows = B * (has_meta ? Tp : T_);
        if (pre_norm) {
            if ((rc = launch_rmsnorm_rows<TIO, TA>(ctx, x_io, w->pre_norm_w, xn, xrows, d, c->rms_eps))) return rc;
        } else if ((rc = launch_pad_copy<TIO, TA>(ctx, x_io, xrows, d, xn, d))) {
            return rc;
        }
        if ((rc = launch_pad_copy<T, TA>(ctx, static_cast<const T*>(w->w_in), k.n_in, d, wi, d))) return rc;
        if (m > 0 && !has_meta && (rc = launch_pad_copy<T, TA>(ctx, static_cast<const T*>(w->meta), m, d, mt, d)))
            return rc;
        if ((rc = launch_pad_copy<T, TA>(ctx, static_cast<const T*>(w->w_out), d, uw, wo, uw))) return rc;
        x = xn; W_in = wi; meta = mt; W_out = wo;
    } else {
        x = x_io;
        if (pre_norm) {
            if ((rc = launch_rmsnorm_rows<TIO, TA>(ctx, x_io, w->pre_norm_w, xn, (long long)B * Tp, d, c->rms_eps)))
                return rc;
            x = xn;
        }
        W_in = static_cast<const T*>(w->w_in);
        meta = static_cast<const T*>(w->meta);
        W_out = static_cast<const T*>(w->w_out);
    }
    // RoPE table and the padded 16-bit W_dt of step 2, one launch
    if ((rc = launch_prefill_prep<T, I>(ctx, rope, Tp, dh, c->rope_base, static_cast<const T*>(w->w_dt), n_dt(c),
                                        c->dt_rank, wdt, pl.rpad)))
        return rc;
    // 1. fused input projection (+ RoPE, K/V scatter) ------------------------------
    EpiArgs<I> ep = epi_base<I>(EPI_INPROJ, 0, k.n_in);
    ep.B = B; ep.Tu = T_; ep.Tp = Tp; ep.n_meta = m;
    ep.P = P; ep.ldP = pl.ldP;
    ep.k_out = c->is_kv_producer ? k_seq : nullptr;
    ep.v_out = c->is_kv_producer ? v_seq : nullptr;
    ep.kcap = kv->seq_cap;
    ep.H = H; ep.G = G; ep.dh = dh; ep.dv = dv;
    ep.rope = rope;
    ep.q_scale = c->is_kv_producer ? nullptr : w->kv_scale;
    if (has_meta) {
        ep.row_mode = ROWS_DIRECT; ep.M = (int)rows;
        if ((rc = gemm<TA, I>(ctx, "gemm_in_proj", x, d, W_in, d, (int)rows, k.n_in, d, ep))) return rc;
    } else {
        bool fused = false;
#ifdef HYMBA_WITH_TCGEN05
        if constexpr (sizeof(TA) == 2) {
            if (((uintptr_t)x & 15) == 0 && ((uintptr_t)W_in & 15) == 0 && ((uintptr_t)meta & 15) == 0 &&
                d % 8 == 0) {
                // one launch: meta rows (projected once, written for every sequence) + user rows
                ep.row_mode = ROWS_USER; ep.M = B * T_;
                if ((rc = launch_gemm_tc<TA, I>(ctx, "gemm_in_proj", x, d, W_in, d, B * T_, k.n_in, d, ep, meta, m)))
                    return rc;
                fused = true;
            }
        }
#endif
        if (!fused) {
            if (m > 0) {
                ep.row_mode = ROWS_META; ep.M = m;
                if ((rc = gemm<TA, I>(ctx, "gemm_in_proj_meta", meta, d, W_in, d, m, k.n_in, d, ep))) return rc;
            }
            ep.row_mode = ROWS_USER; ep.M = B * T_;
            if ((rc = gemm<TA, I>(ctx, "gemm_in_proj", x, d, W_in, d, B * T_, k.n_in, d, ep))) return rc;
        }
    }
    // 2. Delta = softplus(dt_low W_dt^T + b_dt), or inside the scan (step 4) when the
    // batch is wide enough for the one-thread-per-channel scan ------------------------
    const bool fold = std::is_same<I, f16>::value && c->ssm_heads == 0 &&
                      scan_wide_applies(B, di, c->dt_rank, ctx.sm_count);
    if (!fold) {
        // [rows, n_dt]: per channel, or per SSM head in the SSD form
        EpiArgs<I> ed = epi_base<I>(EPI_DELTA, (int)rows, n_dt(c));
        ed.delta = delta; ed.b_dt = w->b_dt;
        if ((rc = gemm<I, I>(ctx, "gemm_dt_proj", P + k.dtl, pl.ldP, wdt, pl.rpad, (int)rows, n_dt(c), c->dt_rank,
                             ed)))
            return rc;
    }
    // 3. attention heads ---------------------------------------------------------
    if ((rc = attn_prefill<I>(ctx, P, pl.ldP, k_seq, v_seq, kv->seq_cap, O, B, Tp, H, G, dv, m, c->window)))
        return rc;
    // 4. Mamba heads ---------------------------------------------------------------
    bool scanned = false;
    if constexpr (std::is_same<I, f16>::value) {
        if (c->ssm_heads > 0) {
            // SSD form: chunked matmuls on the tensor cores
            if ((rc = launch_ssd_scan(ctx, P, pl.ldP, k.x, k.Bc, delta, n_dt(c), w->conv_w, w->conv_b, w->A_log,
                                      w->D, ypre, st ? st->h : nullptr, st ? st->conv : nullptr, B, Tp, di,
                                      c->ssm_heads)))
                return rc;
            scanned = true;
        } else if (fold) {
            if ((rc = launch_conv_scan_wide(ctx, P, pl.ldP, k.x, k.Bc, k.dtl, c->dt_rank, wdt, pl.rpad, w->b_dt,
                                            w->conv_w, w->conv_b, w->A_log, w->D, ypre, st ? st->h : nullptr,
                                            st ? st->conv : nullptr, B, Tp, di)))
                return rc;
            scanned = true;
        }
    }
    if (!scanned && (rc = launch_conv_scan_prefill<I>(ctx, P, pl.ldP, k.x, k.Bc, k.Cc, delta, w->conv_w, w->conv_b,
                                                      w->A_log, w->D, ypre, st ? st->h : nullptr,
                                                      st ? st->conv : nullptr, B, Tp, di, ssm_hp(c))))
        return rc;
    // 5. gate, norms, beta, average (or concatenation) ----------------------------------
    // 6. output projection (+ residual) -------------------------------------------------
    const bool concat = c->fusion == HYMBA_FUSION_CONCAT;
    EpiArgs<TIO> eo = epi_base<TIO>(EPI_OUT, (int)rows, d);
    eo.y = y; eo.B = B; eo.Tu = T_; eo.Tp = Tp; eo.n_meta = m;
    if (flags & HYMBA_ADD_RESIDUAL) {
        eo.res_mode = has_meta ? 1 : 2;
        eo.res_x = x_io;
        eo.res_meta = w->meta;
        eo.res_meta_bf16 = std::is_same<T, bf16>::value;
    }
    bool projected = false;
    if constexpr (std::is_same<TA, bf16>::value) {
        if (concat) {
            // the concatenated branches are not halved, so U is twice as large as the
            // average's: U and W_out go to the tensor cores in fp16 (8x finer than bf16)
            f16* U16 = reinterpret_cast<f16*>(ws + pl.U);
            f16* wo16 = reinterpret_cast<f16*>(ws + pl.wout16);
            if ((rc = launch_pad_copy<T, f16>(ctx, static_cast<const T*>(w->w_out), d, uw, wo16, uw))) return rc;
            if ((rc = launch_fuse<I, f16>(ctx, O, nullptr, 0, H, G, dv, true, ypre, P, pl.ldP, k.z, w->norm_attn_w,
                                          w->norm_ssm_w, w->beta1, w->beta2, vscale(c, w), vbias(c, w), U16,
                                          (int)rows, di, c->rms_eps, nullptr)))
                return rc;
            if ((rc = gemm<f16, TIO>(ctx, "gemm_out_proj", U16, uw, wo16, uw, (int)rows, d, uw, eo))) return rc;
            projected = true;
        }
    }
    if (!projected) {
        if ((rc = launch_fuse<I, TA>(ctx, O, nullptr, 0, H, G, dv, concat, ypre, P, pl.ldP, k.z, w->norm_attn_w,
                                     w->norm_ssm_w, w->beta1, w->beta2, vscale(c, w), vbias(c, w), U, (int)rows, di,
                                     c->rms_eps, nullptr)))
            return rc;
        if ((rc = gemm<TA, TIO>(ctx, "gemm_out_proj", U, uw, W_out, uw, (int)rows, d, uw, eo))) return rc;
    }
    // 7. decode cache of a producer ------------------------------------------------------
    if (c->is_kv_producer && kv->k_cache) {
        if ((rc = launch_cache_fill<I>(ctx, k_seq, v_seq, kv->seq_cap, static_cast<I*>(kv->k_cache),
                                       static_cast<I*>(kv->v_cache), kv->cache_cap, kv->len, B, G, dh, dv, m, Tp)))
            return rc;
    }
    return HYMBA_OK;
}

template <typename T, typename I, typename TIO>
static int decode_impl(const Ctx& ctx, const hymba_layer_cfg* c, const hymba_layer_weights* w,
                       const TIO* x_io, int B, int flags, TIO* y, hymba_kv* kv, hymba_ssm_state* st,
                       char* ws) {
    const Plan pl = plan(c, B, kv->cache_cap, HYMBA_MODE_DECODE);
    const Cols k = columns(c);
    const int m = c->n_meta, d = c->d_model, di = c->d_inner, uw = u_width(c);
    const int H = c->n_q_heads, G = c->n_kv_heads, dh = c->head_dim, dv = c->v_head_dim;
    const int pos_offset = c->is_kv_producer ? 0 : -1;
    I* P = reinterpret_cast<I*>(ws + pl.P);
    I* ypre = reinterpret_cast<I*>(ws + pl.ypre);
    T* U = reinterpret_cast<T*>(ws + pl.U);
    float* part = reinterpret_cast<float*>(ws + pl.part);
    I* k_cache = static_cast<I*>(kv->k_cache);
    I* v_cache = static_cast<I*>(kv->v_cache);
    int rc;
    EpiArgs<I> ep = epi_base<I>(EPI_INPROJ, B, k.n_in);
    ep.row_mode = ROWS_DECODE;
    ep.B = B; ep.Tu = 1; ep.Tp = 1; ep.n_meta = m;
    ep.P = P; ep.ldP = pl.ldP;
    ep.k_out = c->is_kv_producer ? k_cache : nullptr;
    ep.v_out = c->is_kv_producer ? v_cache : nullptr;
    ep.kcap = kv->cache_cap;
    ep.H = H; ep.G = G; ep.dh = dh; ep.dv = dv;
    ep.pos = kv->len; ep.pos_offset = pos_offset;
    ep.n_meta_ring = kv->cache_cap - m;
    ep.rope_base = c->rope_base;
    ep.q_scale = c->is_kv_producer ? nullptr : w->kv_scale;
    // RoPE table of the new positions and, for a fp32 residual stream, the new rows in
    // the layer's type: one launch
    float2* rope = reinterpret_cast<float2*>(ws + pl.rope);
    const T* x;
    T* xc = reinterpret_cast<T*>(ws + pl.xcv);
    if (flags & HYMBA_PRE_NORM) {
        // the block's pre-norm: the projection reads RMSNorm(x) * g, the residual is x
        if ((rc = launch_rmsnorm_rows<TIO, T>(ctx, x_io, w->pre_norm_w, xc, B, d, c->rms_eps))) return rc;
        rc = launch_decode_prep<T, T>(ctx, rope, kv->len, pos_offset, B, dh, c->rope_base, nullptr, 0, 0,
                                      nullptr, 0);
        x = xc;
    } else if constexpr (std::is_same<TIO, T>::value) {
        x = x_io;
        rc = launch_decode_prep<T, T>(ctx, rope, kv->len, pos_offset, B, dh, c->rope_base, nullptr, 0, 0,
                                      nullptr, 0);
    } else {
        rc = launch_decode_prep<TIO, T>(ctx, rope, kv->len, pos_offset, B, dh, c->rope_base, x_io, B, d, xc, d);
        x = xc;
    }
    if (rc) return rc;
    ep.rope = rope;
    if ((rc = gemm<T, I>(ctx, "gemm_in_proj_decode", x, d, static_cast<const T*>(w->w_in), d, B, k.n_in, d, ep))) return rc;
    // split-KV attention, left as partials that the fusion kernel merges, and the SSM step
    // with the Delta projection of the new rows folded in: one launch for 16-bit layers
    bool both = false;
    if constexpr (std::is_same<I, f16>::value && std::is_same<T, bf16>::value) {
        rc = launch_decode_attn_ssm<bf16>(ctx, P, pl.ldP, k_cache, v_cache, kv->cache_cap, kv->len, pos_offset, part,
                                          pl.n_split, B, H, G, dv, m, c->window, k.x, k.Bc, k.Cc, k.dtl,
                                          static_cast<const bf16*>(w->w_dt), w->b_dt, c->dt_rank, w->conv_w,
                                          w->conv_b, w->A_log, w->D, st->h, st->conv, ypre, di, ssm_hp(c));
        if (rc != HYMBA_OK && rc != HYMBA_ERR_UNSUPPORTED) return rc;
        both = rc == HYMBA_OK;
    }
    if (!both) {
        if ((rc = launch_attn_decode<I>(ctx, P, pl.ldP, k_cache, v_cache, kv->cache_cap, kv->len, pos_offset,
                                        part, pl.n_split, nullptr, B, H, G, dv, m, c->window)))
            return rc;
        if ((rc = launch_ssm_decode<I, T>(ctx, P, pl.ldP, k.x, k.Bc, k.Cc, k.dtl, static_cast<const T*>(w->w_dt),
                                          w->b_dt, c->dt_rank, w->conv_w, w->conv_b, w->A_log, w->D, st->h,
                                          st->conv, ypre, B, di, ssm_hp(c))))
            return rc;
    }
    const bool concat = c->fusion == HYMBA_FUSION_CONCAT;
    EpiArgs<TIO> eo = epi_base<TIO>(EPI_OUT, B, d);
    eo.y = y;
    if (flags & HYMBA_ADD_RESIDUAL) { eo.res_mode = 1; eo.res_x = x_io; }
    // The out-projection of a decode step is a few rows against a long K: with an fp32
    // output it is split over K across the SMs, each split adding its partial sum to y,
    // which the fusion kernel first sets to the residual (or zero).
    float* y_init = nullptr;
    const float* y_res = nullptr;
    auto plan_split = [&](bool tc_path) {
        if constexpr (std::is_same<TIO, float>::value) {
            if (tc_path) {
                eo.accumulate = 1;
                y_init = y;
                y_res = eo.res_mode == 1 ? x_io : nullptr;
                eo.res_mode = 0;
            }
        } else {
            (void)tc_path;
        }
    };
    if constexpr (std::is_same<T, bf16>::value) {
        if (concat) {
            // as in the prefill: the concatenation's U and W_out in fp16
            f16* U16 = reinterpret_cast<f16*>(ws + pl.U);
            f16* wo16 = reinterpret_cast<f16*>(ws + pl.wout16);
            if ((rc = launch_pad_copy<T, f16>(ctx, static_cast<const T*>(w->w_out), d, uw, wo16, uw))) return rc;
            plan_split(tc_gemm_ok<f16>(U16, uw, wo16, uw));
            if ((rc = launch_fuse<I, f16>(ctx, nullptr, part, pl.n_split, H, G, dv, true, ypre, P, pl.ldP, k.z,
                                          w->norm_attn_w, w->norm_ssm_w, w->beta1, w->beta2, vscale(c, w),
                                          vbias(c, w), U16, B, di, c->rms_eps,
                                          c->is_kv_producer ? kv->len : nullptr, y_init, y_res, d)))
                return rc;
            return gemm<f16, TIO>(ctx, "gemm_out_proj_decode", U16, uw, wo16, uw, B, d, uw, eo);
        }
    }
    plan_split(tc_gemm_ok<T>(U, uw, static_cast<const T*>(w->w_out), uw));
    if ((rc = launch_fuse<I, T>(ctx, nullptr, part, pl.n_split, H, G, dv, concat, ypre, P, pl.ldP, k.z,
                                w->norm_attn_w, w->norm_ssm_w, w->beta1, w->beta2, vscale(c, w), vbias(c, w), U, B,
                                di, c->rms_eps, c->is_kv_producer ? kv->len : nullptr, y_init, y_res, d)))
        return rc;
    if ((rc = gemm<T, TIO>(ctx, "gemm_out_proj_decode", U, uw, static_cast<const T*>(w->w_out), uw, B, d, uw, eo)))
        return rc;
    return HYMBA_OK;
}

static int check_weights(const hymba_layer_cfg* c, const hymba_layer_weights* w) {
    if (!w || !w->w_in || !w->w_dt || !w->b_dt || !w->conv_w || !w->conv_b || !w->A_log || !w->D ||
        !w->norm_attn_w || !w->norm_ssm_w || !w->beta1 || !w->beta2 || !w->w_out)
        return HYMBA_ERR_INVALID_ARG;
    if (c->n_meta > 0 && !w->meta) return HYMBA_ERR_INVALID_ARG;
    // the affine adaptation of shared K/V: consumers only, both vectors or neither,
    // 16-byte aligned (read as float4)
    if ((w->kv_scale == nullptr) != (w->kv_bias == nullptr)) return HYMBA_ERR_INVALID_ARG;
    if (w->kv_scale && c->is_kv_producer) return HYMBA_ERR_INVALID_ARG;
    if (((uintptr_t)w->kv_scale | (uintptr_t)w->kv_bias) & 15) return HYMBA_ERR_INVALID_ARG;
    return HYMBA_OK;
}

static int kv_dtype(const hymba_layer_cfg* c) { return c->dtype == HYMBA_BF16 ? HYMBA_F16 : HYMBA_F32; }

static int check_kv_shape(const hymba_layer_cfg* c, const hymba_kv* kv, int B) {
    if (kv->batch != B || kv->n_meta != c->n_meta || kv->n_kv_heads != c->n_kv_heads ||
        kv->head_dim != c->head_dim || kv->v_head_dim != c->v_head_dim || kv->dtype != kv_dtype(c))
        return HYMBA_ERR_KV_INCOMPATIBLE;
    return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// the block's MLP: h += W_down (SiLU(W_gate n) * (W_up n)), n = RMSNorm(h) * g
// ---------------------------------------------------------------------------
struct MlpPlan {
    size_t total = 0, n = 0, gate = 0, act = 0, wg = 0, wu = 0, wd = 0;
};

static MlpPlan mlp_plan(const hymba_layer_cfg* c, int d_ff, long long rows) {
    MlpPlan p;
    const size_t esz = c->dtype == HYMBA_BF16 ? 2 : 4;  // fp16 operands for bf16 layers
    size_t cur = 0;
    p.n = take(&cur, rows * c->d_model * esz);
    p.gate = take(&cur, rows * (size_t)d_ff * esz);
    p.act = take(&cur, rows * (size_t)d_ff * esz);
    if (c->dtype == HYMBA_BF16) {
        p.wg = take(&cur, (size_t)d_ff * c->d_model * 2);
        p.wu = take(&cur, (size_t)d_ff * c->d_model * 2);
        p.wd = take(&cur, (size_t)c->d_model * d_ff * 2);
    }
    p.total = cur;
    return p;
}

// T: the layer's weight type; TA: the operand type (fp16 for bf16 weights, converted per
// call; fp32 for fp32 layers, CUDA-core GEMMs)
template <typename T, typename TA>
static int mlp_impl(const Ctx& ctx, const hymba_layer_cfg* c, int d_ff, const hymba_mlp_weights* w, float* h,
                    long long rows, char* ws) {
    const MlpPlan pl = mlp_plan(c, d_ff, rows);
    const int d = c->d_model;
    TA* n = reinterpret_cast<TA*>(ws + pl.n);
    TA* gate = reinterpret_cast<TA*>(ws + pl.gate);
    TA* act = reinterpret_cast<TA*>(ws + pl.act);
    const TA *Wg, *Wu, *Wd;
    int rc;
    if constexpr (std::is_same<T, TA>::value) {
        Wg = static_cast<const TA*>(w->w_gate);
        Wu = static_cast<const TA*>(w->w_up);
        Wd = static_cast<const TA*>(w->w_down);
    } else {
        TA* wg = reinterpret_cast<TA*>(ws + pl.wg);
        TA* wu = reinterpret_cast<TA*>(ws + pl.wu);
        TA* wd = reinterpret_cast<TA*>(ws + pl.wd);
        if ((rc = launch_pad_copy<T, TA>(ctx, static_cast<const T*>(w->w_gate), d_ff, d, wg, d))) return rc;
        if ((rc = launch_pad_copy<T, TA>(ctx, static_cast<const T*>(w->w_up), d_ff, d, wu, d))) return rc;
        if ((rc = launch_pad_copy<T, TA>(ctx, static_cast<const T*>(w->w_down), d, d_ff, wd, d_ff))) return rc;
        Wg = wg; Wu = wu; Wd = wd;
    }
    if ((rc = launch_rmsnorm_rows<float, TA>(ctx, h, w->norm_w, n, rows, d, c->rms_eps))) return rc;
    EpiArgs<TA> eg = epi_base<TA>(EPI_OUT, (int)rows, d_ff);
    eg.y = gate;
    if ((rc = gemm<TA, TA>(ctx, "gemm_mlp_gate", n, d, Wg, d, (int)rows, d_ff, d, eg))) return rc;
    EpiArgs<TA> eu = epi_base<TA>(EPI_GLU, (int)rows, d_ff);
    eu.y = act;
    eu.glu_gate = gate;
    if ((rc = gemm<TA, TA>(ctx, "gemm_mlp_up", n, d, Wu, d, (int)rows, d_ff, d, eu))) return rc;
    EpiArgs<float> ed = epi_base<float>(EPI_OUT, (int)rows, d);
    ed.y = h;
    ed.res_mode = 1;
    ed.res_x = h;  // in place: each output element is read, then written, by one thread
    return gemm<TA, float>(ctx, "gemm_mlp_down", act, d_ff, Wd, d_ff, (int)rows, d, d_ff, ed);
}

}  // namespace hymba

using namespace hymba;

extern "C" {

size_t hymba_workspace_bytes(const hymba_layer_cfg* cfg, int B, int T, int mode) {
    if (check_cfg(cfg) || B <= 0 || T <= 0 || (mode != HYMBA_MODE_PREFILL && mode != HYMBA_MODE_DECODE))
        return 0;
    return plan(cfg, B, T, mode).total;
}

int hymba_workspace_layout(const hymba_layer_cfg* cfg, int B, int T, int mode, int64_t* out, int n) {
    if (check_cfg(cfg) || B <= 0 || T <= 0 || !out || n < 10) return HYMBA_ERR_INVALID_ARG;
    const Plan p = plan(cfg, B, T, mode);
    const int64_t v[10] = {(int64_t)p.total, (int64_t)p.P,    (int64_t)p.ldP, (int64_t)p.delta,
                           (int64_t)p.O,     (int64_t)p.ypre, (int64_t)p.U,   (int64_t)p.rope,
                           (int64_t)p.part,  (int64_t)p.n_split};
    for (int i = 0; i < 10; ++i) out[i] = v[i];
    return HYMBA_OK;
}

int hymba_mixer_prefill(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const void* x,
                        int B, int T, int flags, void* y, hymba_kv* kv, hymba_ssm_state* st,
                        void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if ((rc = check_weights(cfg, w))) return rc;
    if (!x || !y || !kv || !workspace || B <= 0 || T <= 0 || (flags & ~15)) return HYMBA_ERR_INVALID_ARG;
    // the block's pre-norm acts on a stream that already holds the meta rows
    if ((flags & HYMBA_PRE_NORM) && (!(flags & HYMBA_X_HAS_META) || !w->pre_norm_w)) return HYMBA_ERR_INVALID_ARG;
    if ((flags & HYMBA_IO_F32) && cfg->dtype != HYMBA_BF16) return HYMBA_ERR_INVALID_ARG;
    if ((uintptr_t)workspace & 255) return HYMBA_ERR_INVALID_ARG;
    if (!kv->k_seq || !kv->v_seq) return HYMBA_ERR_INVALID_ARG;
    if ((rc = check_kv_shape(cfg, kv, B))) return rc;
    const int Tp = cfg->n_meta + T;
    if (kv->seq_cap < Tp) return HYMBA_ERR_KV_INCOMPATIBLE;
    if (cfg->is_kv_producer && kv->k_cache) {
        if (!kv->v_cache || !kv->len || kv->cache_cap <= cfg->n_meta) return HYMBA_ERR_INVALID_ARG;
    }
    if (st && (!st->h || !st->conv)) return HYMBA_ERR_INVALID_ARG;
    if (y != x) {
        const size_t xb = (size_t)B * ((flags & HYMBA_X_HAS_META) ? Tp : T) * cfg->d_model;
        const size_t yb = (size_t)B * Tp * cfg->d_model;
        const char* xs = static_cast<const char*>(x);
        const char* ys = static_cast<const char*>(y);
        const size_t es = (cfg->dtype == HYMBA_BF16 && !(flags & HYMBA_IO_F32)) ? 2 : 4;
        if (xs < ys + yb * es && ys < xs + xb * es) return HYMBA_ERR_INVALID_ARG;
    } else if (!(flags & HYMBA_X_HAS_META)) {
        return HYMBA_ERR_INVALID_ARG;
    }
    if (ws_bytes < plan(cfg, B, T, HYMBA_MODE_PREFILL).total) return HYMBA_ERR_WORKSPACE_TOO_SMALL;
    Ctx ctx;
    if ((rc = current_ctx(static_cast<cudaStream_t>(stream), &ctx))) return rc;
    char* ws = static_cast<char*>(workspace);
    if (cfg->dtype == HYMBA_BF16 && (flags & HYMBA_IO_F32))
        return prefill_impl<bf16, f16, float>(ctx, cfg, w, static_cast<const float*>(x), B, T, flags,
                                              static_cast<float*>(y), kv, st, ws);
    if (cfg->dtype == HYMBA_BF16)
        return prefill_impl<bf16, f16, bf16>(ctx, cfg, w, static_cast<const bf16*>(x), B, T, flags,
                                             static_cast<bf16*>(y), kv, st, ws);
    return prefill_impl<float, float, float>(ctx, cfg, w, static_cast<const float*>(x), B, T, flags,
                                             static_cast<float*>(y), kv, st, ws);
}

int hymba_mixer_decode(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const void* x_t,
                       int B, int flags, void* y_t, hymba_kv* kv, hymba_ssm_state* st,
                       void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if ((rc = check_weights(cfg, w))) return rc;
    if (!x_t || !y_t || !kv || !st || !st->h || !st->conv || !workspace || B <= 0 ||
        (flags & ~(HYMBA_ADD_RESIDUAL | HYMBA_IO_F32 | HYMBA_PRE_NORM)))
        return HYMBA_ERR_INVALID_ARG;
    if ((flags & HYMBA_PRE_NORM) && !w->pre_norm_w) return HYMBA_ERR_INVALID_ARG;
    if ((flags & HYMBA_IO_F32) && cfg->dtype != HYMBA_BF16) return HYMBA_ERR_INVALID_ARG;
    if ((uintptr_t)workspace & 255) return HYMBA_ERR_INVALID_ARG;
    if (!kv->k_cache || !kv->v_cache || !kv->len || kv->cache_cap <= cfg->n_meta) return HYMBA_ERR_INVALID_ARG;
    if ((rc = check_kv_shape(cfg, kv, B))) return rc;
    if (ws_bytes < plan(cfg, B, kv->cache_cap, HYMBA_MODE_DECODE).total) return HYMBA_ERR_WORKSPACE_TOO_SMALL;
    Ctx ctx;
    if ((rc = current_ctx(static_cast<cudaStream_t>(stream), &ctx))) return rc;
    char* ws = static_cast<char*>(workspace);
    if (cfg->dtype == HYMBA_BF16 && (flags & HYMBA_IO_F32))
        return decode_impl<bf16, f16, float>(ctx, cfg, w, static_cast<const float*>(x_t), B, flags,
                                             static_cast<float*>(y_t), kv, st, ws);
    if (cfg->dtype == HYMBA_BF16)
        return decode_impl<bf16, f16, bf16>(ctx, cfg, w, static_cast<const bf16*>(x_t), B, flags,
                                            static_cast<bf16*>(y_t), kv, st, ws);
    return decode_impl<float, float, float>(ctx, cfg, w, static_cast<const float*>(x_t), B, flags,
                                            static_cast<float*>(y_t), kv, st, ws);
}

int hymba_kv_share(const hymba_kv* producer, const hymba_layer_cfg* consumer_cfg, hymba_kv* out) {
    if (!producer || !consumer_cfg || !out) return HYMBA_ERR_INVALID_ARG;
    int rc = check_cfg(consumer_cfg);
    if (rc) return rc;
    if (consumer_cfg->is_kv_producer) return HYMBA_ERR_INVALID_ARG;
    if ((rc = check_kv_shape(consumer_cfg, producer, producer->batch))) return rc;
    if (producer->k_cache) {
        const int ring = producer->cache_cap - producer->n_meta;
        if (consumer_cfg->window > 0 && consumer_cfg->window > ring) return HYMBA_ERR_KV_INCOMPATIBLE;
        if (consumer_cfg->window <= 0 && producer->window > 0 && ring <= producer->window)
            return HYMBA_ERR_KV_INCOMPATIBLE;
    }
    *out = *producer;
    out->window = consumer_cfg->window;
    return HYMBA_OK;
}

uint64_t hymba_kv_bytes(int n_attn_layers, int n_kv_heads, int head_dim, int v_head_dim,
                        int64_t seq_len, int batch, int dtype_bytes) {
    if (n_attn_layers < 0 || n_kv_heads < 0 || head_dim < 0 || v_head_dim < 0 || seq_len < 0 ||
        batch < 0 || dtype_bytes < 0)
        return 0;
    return (uint64_t)batch * (uint64_t)seq_len * (uint64_t)n_attn_layers * (uint64_t)n_kv_heads *
           (uint64_t)(head_dim + v_head_dim) * (uint64_t)dtype_bytes;
}

uint64_t hymba_ssm_state_bytes(int n_layers, int channels, int d_state, int batch, int dtype_bytes) {
    if (n_layers < 0 || channels < 0 || d_state < 0 || batch < 0 || dtype_bytes < 0) return 0;
    return (uint64_t)n_layers * channels * d_state * batch * dtype_bytes;
}

size_t hymba_cache_bytes(const hymba_layer_cfg* cfg, int B, int max_T) {
    if (check_cfg(cfg) || B <= 0 || max_T <= 0) return 0;
    const int esz = cfg->dtype == HYMBA_BF16 ? 2 : 4;
    // slots: the meta block + a window-long ring, or one slot per position (meta
    // included in max_T) for a global layer
    const int slots = cfg->window > 0 ? cfg->n_meta + cfg->window : max_T;
    size_t kv = 0;
    if (cfg->is_kv_producer)
        kv = hymba_kv_bytes(1, cfg->n_kv_heads, cfg->head_dim, cfg->v_head_dim, slots, B, esz);
    return kv + hymba_ssm_state_bytes(1, cfg->d_inner, cfg->d_state, B, 4) +
           (size_t)B * cfg->d_inner * cfg->d_conv * 4 + (size_t)B * 4;
}

int hymba_get_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HYMBA_ERR_CUDA;
    Ctx ctx;
    if (current_ctx(static_cast<cudaStream_t>(stream), &ctx)) return HYMBA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, ctx.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return HYMBA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(ctx.status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return HYMBA_ERR_CUDA;
    return v;
}

int hymba_get_device_diag(int32_t* out, int n) {
    if (!out || n < 7) return HYMBA_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return HYMBA_ERR_CUDA;
    Ctx ctx;
    if (current_ctx(nullptr, &ctx)) return HYMBA_ERR_CUDA;
    int v[7] = {0};
    if (cudaMemcpy(v, ctx.status + 1, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return HYMBA_ERR_CUDA;
    const int zero[7] = {0};
    if (cudaMemcpy(ctx.status + 1, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return HYMBA_ERR_CUDA;
    for (int i = 0; i < 7; ++i) out[i] = v[i];
    return HYMBA_OK;
}

size_t hymba_mlp_workspace_bytes(const hymba_layer_cfg* cfg, int d_ff, long long rows) {
    if (check_cfg(cfg) || d_ff <= 0 || rows <= 0) return 0;
    return mlp_plan(cfg, d_ff, rows).total;
}

int hymba_mlp(const hymba_layer_cfg* cfg, int d_ff, const hymba_mlp_weights* w, float* h, long long rows,
              void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!w || !w->norm_w || !w->w_gate || !w->w_up || !w->w_down || !h || !workspace || rows <= 0 || d_ff <= 0 ||
        rows > 0x7fffffffLL)
        return HYMBA_ERR_INVALID_ARG;
    if (d_ff % 64) return HYMBA_ERR_UNSUPPORTED;
    if (((uintptr_t)workspace & 255) || ((uintptr_t)h & 15)) return HYMBA_ERR_INVALID_ARG;
    if (ws_bytes < mlp_plan(cfg, d_ff, rows).total) return HYMBA_ERR_WORKSPACE_TOO_SMALL;
    Ctx ctx;
    if ((rc = current_ctx(static_cast<cudaStream_t>(stream), &ctx))) return rc;
    char* ws = static_cast<char*>(workspace);
    if (cfg->dtype == HYMBA_BF16) return mlp_impl<bf16, f16>(ctx, cfg, d_ff, w, h, rows, ws);
    return mlp_impl<float, float>(ctx, cfg, d_ff, w, h, rows, ws);
}

int hymba_debug_set_wait_limit(long long cycles) {
    if (cycles < 0) return HYMBA_ERR_INVALID_ARG;
    Ctx ctx;
    if (current_ctx(nullptr, &ctx)) return HYMBA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return HYMBA_ERR_CUDA;
    if (cudaMemcpy(ctx.status + 8, &cycles, sizeof(cycles), cudaMemcpyHostToDevice) != cudaSuccess)
        return HYMBA_ERR_CUDA;
    return HYMBA_OK;
}

const char* hymba_strerror(int code) {
    switch (code) {
        case HYMBA_OK: return "ok";
        case HYMBA_ERR_INVALID_ARG: return "invalid argument";
        case HYMBA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case HYMBA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case HYMBA_ERR_KV_INCOMPATIBLE: return "KV descriptor incompatible with the layer";
        case HYMBA_ERR_CUDA: return "CUDA error";
        case HYMBA_ERR_DEVICE_TIMEOUT: return "bounded device wait timed out";
        case HYMBA_ERR_DEVICE_RANGE: return "device range check failed";
        case HYMBA_ERR_SCRATCH_LIMIT: return "request exceeds the fixed scratch of hymba_attn_decode_static";
        default: return "unknown status";
    }
}

int hymba_trace_enable(int on) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (on && g_trace.empty()) {
        g_trace.resize(kTracePool);
        for (auto& r : g_trace) {
            if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess)
                return HYMBA_ERR_CUDA;
            r.name = nullptr;
        }
    }
    g_trace_used.store(0);
    g_trace_on.store(on ? 1 : 0);
    return HYMBA_OK;
}

int hymba_trace_only(const char* name) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (name && strlen(name) >= sizeof(g_trace_only)) return HYMBA_ERR_INVALID_ARG;
    if (name) strcpy(g_trace_only, name);
    else g_trace_only[0] = 0;
    return HYMBA_OK;
}

int hymba_trace_collect(const char** names, float* ms, int max_records) {
    if (cudaDeviceSynchronize() != cudaSuccess) return HYMBA_ERR_CUDA;
    const int used = std::min(g_trace_used.load(), (int)g_trace.size());
    int n = 0;
    for (int i = 0; i < used && n < max_records; ++i) {
        float t = 0.f;
        if (!g_trace[i].name || cudaEventElapsedTime(&t, g_trace[i].a, g_trace[i].b) != cudaSuccess) continue;
        if (names) names[n] = g_trace[i].name;
        if (ms) ms[n] = t;
        ++n;
    }
    for (int i = 0; i < used; ++i) g_trace[i].name = nullptr;
    g_trace_used.store(0);
    return n;
}

uint64_t hymba_launch_count(void) { return g_launches.load(); }

}  // extern "C"
