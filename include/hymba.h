/*
 * hymba.h - C ABI of libhymba.so, the B200 (sm_100a) Hymba parallel hybrid-head mixer.
 *
 * What the library computes (one mixer layer; sources are cited by page title and
 * section):
 *   "Hymba Guide: NVIDIA Hybrid-Head Mamba & Attention SLM", section "Parallel
 *   Hybrid-Head Layer Formulation": attention heads and Mamba (SSM) heads run in
 *   parallel on the same input and one output projection W_o mixes them; section
 *   "Learnable Meta-Tokens": n_meta learned rows are prepended to every sequence;
 *   section "Cross-Layer KV Cache Sharing": a secondary layer reuses the K and V of
 *   the primary layer with no new buffer.
 *   "Jamba: Hybrid SSM-Transformer", How It Actually Works section 1: the selective
 *   scan h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) x_t, y_t = C_t h_t, and
 *   softmax(Q K^T / sqrt(d_k)) V attention with GQA.
 *   51cto "Hymba-1.5B" article, section 2: GQA + RoPE, sliding-window attention with
 *   a few global layers, KV shared by pairs of layers.
 *
 * Per layer and sequence, with X^ = [meta; x] (T' = n_meta + T rows):
 *   [Q K V x z B C dt_low] = X^ W_in^T                 one fused projection
 *   Q, K <- RoPE (rotate-half, base rope_base), position of row i is i
 *   O     = GQA softmax attention, key j visible to query i iff j <= i and
 *           (j < n_meta or i - j < window); window <= 0 means global
 *   xc    = SiLU(depthwise causal conv_{d_conv}(x) + conv_b)
 *   Delta = softplus(dt_low W_dt^T + b_dt),  A = -exp(A_log)
 *   h_t   = exp(Delta_t A) h_{t-1} + Delta_t B_t xc_t  (fp32 state)
 *   Y     = (C_t . h_t + D xc_t) * SiLU(z_t)
 *   U     = (beta1 * RMSNorm(O) + beta2 * RMSNorm(Y)) / 2
 *   y     = U W_out^T (+ X^ when HYMBA_ADD_RESIDUAL)
 *
 * Conventions for every entry point:
 *   - Every pointer marked "device" is device memory owned by the caller. The
 *     library never allocates, frees or synchronises on the compute entry points;
 *     all work is queued on `stream` (a cudaStream_t, NULL = legacy default stream).
 *   - Tensors are dense row-major with the shapes given; "dtype" is the layer's
 *     activation and weight type (HYMBA_F32 or HYMBA_BF16). Small per-channel
 *     parameters are always fp32. Inside a bf16 layer, the projection, K/V,
 *     attention output and pre-gate SSM output are held in fp16 (2 bytes like bf16,
 *     8x finer rounding); accumulation is fp32 everywhere.
 *   - Return value: HYMBA_OK (0) or a negative HYMBA_ERR_* code. Argument checks
 *     happen on the host before any launch; a failed check queues no work. Errors
 *     found on the device (bounded waits that time out, out-of-range positions)
 *     are recorded in a per-device status word read by hymba_get_device_status().
 *   - The functions keep no per-call global state and are safe to call from
 *     several host threads on different streams (except the opt-in tracing).
 */
#ifndef HYMBA_H
#define HYMBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define HYMBA_OK                       0
#define HYMBA_ERR_INVALID_ARG        (-1)  /* null pointer, non-positive size, bad flag */
#define HYMBA_ERR_UNSUPPORTED        (-2)  /* shape or dtype outside what the kernels handle */
#define HYMBA_ERR_WORKSPACE_TOO_SMALL (-3) /* ws_bytes < hymba_workspace_bytes(...) */
#define HYMBA_ERR_KV_INCOMPATIBLE    (-4)  /* KV descriptor does not fit the layer */
#define HYMBA_ERR_CUDA               (-5)  /* a CUDA call or launch failed */
#define HYMBA_ERR_DEVICE_TIMEOUT     (-6)  /* a bounded device wait ran out (status word) */
#define HYMBA_ERR_DEVICE_RANGE       (-7)  /* a device-side range check failed (status word) */
#define HYMBA_ERR_SCRATCH_LIMIT      (-8)  /* request larger than hymba_attn_decode_static's fixed scratch */

/* dtypes: a layer is HYMBA_F32 or HYMBA_BF16; the K/V buffers of a bf16 layer hold
 * HYMBA_F16 (same width as bf16, finer mantissa; see hymba_kv) */
#define HYMBA_F32  0
#define HYMBA_BF16 1
#define HYMBA_F16  2

/* flags of the mixer calls */
#define HYMBA_X_HAS_META    1  /* x already holds the n_meta rows (a later layer of a stack) */
#define HYMBA_ADD_RESIDUAL  2  /* y = X^ + mixer(X^) */
#define HYMBA_IO_F32        4  /* bf16 layer with fp32 x, y: a residual stream kept in fp32
                                  between stacked layers (the projection operand X^ is
                                  rounded to bf16 inside; the residual add is fp32) */
#define HYMBA_PRE_NORM      8  /* the block's pre-norm: the mixer reads RMSNorm(x) * pre_norm_w
                                  while the residual (HYMBA_ADD_RESIDUAL) stays x; prefill
                                  requires HYMBA_X_HAS_META (the stream holds the meta rows) */

/* fusion of the two head families (hymba_layer_cfg.fusion) */
#define HYMBA_FUSION_AVERAGE 0  /* U = (beta1 RMSNorm(O) + beta2 RMSNorm(Y)) / 2, d_inner wide */
#define HYMBA_FUSION_CONCAT  1  /* U = [beta2 RMSNorm(Y) | beta1 RMSNorm(O)], d_inner + H*dv wide */

/* workspace modes */
#define HYMBA_MODE_PREFILL 0
#define HYMBA_MODE_DECODE  1

/* Shape and numerics of one mixer layer. With HYMBA_FUSION_AVERAGE the V head dim
 * must equal d_inner / n_q_heads so that the two branches can be averaged; with
 * HYMBA_FUSION_CONCAT ("Hymba Guide", Parallel Hybrid-Head Layer Formulation:
 * y = W_o(Concat[MambaHeads(x), AttentionHeads(x)])) the branches are placed side by
 * side, Mamba first, and W_o takes d_inner + n_q_heads * v_head_dim inputs.
 * Supported: head_dim == 64; v_head_dim 64 or 128; n_q_heads % n_kv_heads == 0 with at
 * most 8 query heads per KV head; d_model, d_inner and n_q_heads * v_head_dim multiples
 * of 64, at most 4096; d_state == 16; d_conv == 4. */
typedef struct hymba_layer_cfg {
    int32_t d_model;
    int32_t n_q_heads;
    int32_t n_kv_heads;
    int32_t head_dim;        /* Q/K head dim (64) */
    int32_t v_head_dim;      /* = d_inner / n_q_heads */
    int32_t d_inner;
    int32_t d_state;
    int32_t d_conv;
    int32_t dt_rank;
    int32_t n_meta;
    int32_t window;          /* <= 0: global attention */
    int32_t is_kv_producer;  /* 1: projects its own K, V; 0: reads a producer's */
    int32_t dtype;           /* HYMBA_F32 or HYMBA_BF16 */
    float   rope_base;
    float   rms_eps;
    int32_t fusion;          /* HYMBA_FUSION_AVERAGE or HYMBA_FUSION_CONCAT */
    /* 0: the selective form, A per (channel, state) and Delta per channel. > 0: the SSD
     * form ("Lecture 04 - Beyond the Dense Transformer", section 3: Mamba-2 makes A a
     * scalar times the identity and gives the SSM a multi-head structure): the channels
     * split into ssm_heads heads of d_inner / ssm_heads consecutive channels, and
     * W_dt, b_dt and A_log hold one entry per head (Delta_t and A shared by the head's
     * channels and all states). The head width must be a multiple of 8, and exactly 64
     * for HYMBA_BF16 (whose prefill computes the chunked matmul form on the tensor
     * cores); otherwise HYMBA_ERR_UNSUPPORTED. */
    int32_t ssm_heads;
} hymba_layer_cfg;

/* Weights of one layer (device pointers, caller-owned, read only). Big matrices
 * use the [out, in] convention. n_in = H*dh + (producer ? G*(dh+dv) : 0)
 * + 2*d_inner + 2*d_state + dt_rank, rows in the order Q | K | V | x | z | B | C |
 * dt_low (B and C first so that their columns start on 16-byte boundaries). */
typedef struct hymba_layer_weights {
    const void*  w_in;        /* [n_in, d_model]        dtype */
    const void*  w_dt;        /* [n_dt, dt_rank]        dtype; n_dt = d_inner, or ssm_heads in the SSD form */
    const float* b_dt;        /* [n_dt] */
    const float* conv_w;      /* [d_inner, d_conv]      tap d_conv-1 meets the newest input */
    const float* conv_b;      /* [d_inner] */
    const float* A_log;       /* [d_inner, d_state]     A = -exp(A_log); [ssm_heads] in the SSD form */
    const float* D;           /* [d_inner] */
    const float* norm_attn_w; /* [n_q_heads*v_head_dim] RMSNorm gain of the attention branch */
    const float* norm_ssm_w;  /* [d_inner]              RMSNorm gain of the SSM branch */
    const float* beta1;       /* [n_q_heads*v_head_dim] */
    const float* beta2;       /* [d_inner] */
    const void*  w_out;       /* [d_model, u] dtype: u = d_inner (average) or d_inner + n_q_heads*v_head_dim (concat) */
    const void*  meta;        /* [n_meta, d_model]      dtype */
    /* Consumer layers only (NULL for a producer, and NULL for plain sharing): the
     * head-specific affine adaptation of the shared K and V ("Hymba Guide",
     * Cross-Layer KV Cache Sharing, section 1: K~ = K * w_scale + b_bias, and V~ the
     * same with its own scale and bias), elementwise per KV head on the K held in the
     * cache (after RoPE). Both [n_kv_heads*head_dim + n_kv_heads*v_head_dim] fp32: the
     * K vectors of the KV heads, then their V vectors. Both or neither. No K/V copy is
     * made: the K scale is applied to the queries instead (q . (k * s) = (q * s) . k),
     * the K bias adds the same q . b to every score of a query and so leaves the softmax
     * unchanged, and the V transform is applied to the attention output (its weights
     * sum to 1). */
    const float* kv_scale;
    const float* kv_bias;
    /* [d_model] fp32 gain of the block's pre-mixer RMSNorm (HYMBA_PRE_NORM; else unused) */
    const float* pre_norm_w;
} hymba_layer_weights;

/* K/V of one producer layer and of the consumers that share it ("Hymba Guide",
 * Cross-Layer KV Cache Sharing). Two parts, both caller-owned device memory:
 *   - prefill sequence K/V: k_seq [batch, n_kv_heads, seq_cap, head_dim] and
 *     v_seq [batch, n_kv_heads, seq_cap, v_head_dim]; position i of a sequence in
 *     row i. A producer's prefill writes them (K after RoPE), a consumer's reads.
 *     Required by prefill (seq_cap >= T'); unused by decode.
 *   - decode cache: k_cache [batch, n_kv_heads, cache_cap, head_dim],
 *     v_cache [batch, n_kv_heads, cache_cap, v_head_dim], len [batch] int32.
 *     Slots 0..n_meta-1 hold the meta positions; position p >= n_meta lives in slot
 *     n_meta + (p - n_meta) mod (cache_cap - n_meta), a ring. len[b] = positions
 *     held so far (meta included). NULL k_cache: no decode cache. A producer's
 *     prefill fills it (meta + the newest cache_cap - n_meta positions) and sets
 *     len; a producer's decode appends one position and increments len; a
 *     consumer's decode reads positions 0..len-1. */
typedef struct hymba_kv {
    void*    k_seq;
    void*    v_seq;
    int32_t  seq_cap;
    void*    k_cache;
    void*    v_cache;
    int32_t* len;
    int32_t  cache_cap;
    int32_t  batch;
    int32_t  n_meta;
    int32_t  n_kv_heads;
    int32_t  head_dim;
    int32_t  v_head_dim;
    int32_t  dtype;      /* HYMBA_F32 for fp32 layers, HYMBA_F16 for bf16 layers */
    int32_t  window;     /* attention span of the producer (<= 0: global) */
} hymba_kv;

/* Recurrent state of one layer's Mamba heads (device, caller-owned):
 * h [batch, d_inner, d_state] fp32; conv [batch, d_inner, d_conv] fp32 holding
 * the last d_conv pre-conv inputs, oldest first. */
typedef struct hymba_ssm_state {
    float* h;
    float* conv;
} hymba_ssm_state;

/* Prefill of B sequences of T user tokens through one layer.
 *   x: device [B, T, d_model] dtype, or [B, n_meta+T, d_model] with HYMBA_X_HAS_META.
 *   y: device [B, n_meta+T, d_model] dtype (meta rows included, so stacks compose);
 *      x and y are fp32 instead when HYMBA_IO_F32 is set.
 *      y may equal x when HYMBA_X_HAS_META is set (in-place residual stacks);
 *      otherwise y and x must not overlap.
 *   kv: producer: k_seq/v_seq written (and the decode cache filled if k_cache);
 *       consumer: k_seq/v_seq read (fill them with the producer's prefill first).
 *   st: NULL, or the state to write: h and conv after the last row.
 *   workspace: device scratch of at least hymba_workspace_bytes(cfg, B, T,
 *       HYMBA_MODE_PREFILL) bytes, 256-byte aligned; contents are undefined after. */
int hymba_mixer_prefill(const hymba_layer_cfg* cfg, const hymba_layer_weights* w,
                        const void* x, int B, int T, int flags, void* y,
                        hymba_kv* kv, hymba_ssm_state* st,
                        void* workspace, size_t ws_bytes, void* stream);

/* One decode step: one new token per sequence; sequence b's token sits at position
 * len[b] (producer) or len[b]-1 (consumer). The sequences of a batch may be at
 * different positions: each keeps its own length, ring slot and state, so a batch of
 * sequences of different lengths decodes together with no padding (the 51cto
 * Hymba-1.5B article, section 4, notes that padded meta tokens and the sliding
 * window kept the released code at batch 1 for generation).
 *   x_t: device [B, d_model]; y_t: device [B, d_model] (may equal x_t); fp32 with
 *   HYMBA_IO_F32, else dtype. Flags: HYMBA_ADD_RESIDUAL, HYMBA_IO_F32.
 *   kv must hold a decode cache (k_cache, len); st is updated in place. A cache
 *   whose ring is too short for the layer's span makes the step record
 *   HYMBA_ERR_DEVICE_RANGE in the status word and write zeros for that row. */
int hymba_mixer_decode(const hymba_layer_cfg* cfg, const hymba_layer_weights* w,
                       const void* x_t, int B, int flags, void* y_t,
                       hymba_kv* kv, hymba_ssm_state* st,
                       void* workspace, size_t ws_bytes, void* stream);

/* The MLP of the Hymba block around the mixer (the 51cto Hymba-1.5B article, section 2,
 * gives its intermediate size, 5504; the form is the Llama-family pre-norm SiLU-gated
 * MLP): h += W_down (SiLU(W_gate n) * (W_up n)) with n = RMSNorm(h) * norm_w, on every
 * row of the fp32 residual stream h [rows, d_model] in place. A block is
 *   hymba_mixer_prefill/decode(... HYMBA_PRE_NORM | HYMBA_ADD_RESIDUAL ...), then hymba_mlp.
 * Weights (device, caller-owned) of the layer's dtype: w_gate, w_up [d_ff, d_model],
 * w_down [d_model, d_ff]; norm_w [d_model] fp32. d_ff a multiple of 64. A bf16 layer's
 * GEMMs take fp16 operands (the weights converted per call into the workspace); an
 * fp32 layer's run on CUDA cores. Workspace: hymba_mlp_workspace_bytes, 256-byte aligned. */
typedef struct hymba_mlp_weights {
    const float* norm_w;
    const void*  w_gate;
    const void*  w_up;
    const void*  w_down;
} hymba_mlp_weights;

int hymba_mlp(const hymba_layer_cfg* cfg, int d_ff, const hymba_mlp_weights* w, float* h, long long rows,
              void* workspace, size_t ws_bytes, void* stream);
size_t hymba_mlp_workspace_bytes(const hymba_layer_cfg* cfg, int d_ff, long long rows);

/* Cross-layer KV sharing: fill *consumer_out with the producer's buffers (pointer
 * copies, no device work, no new memory). Fails with HYMBA_ERR_KV_INCOMPATIBLE
 * when the consumer's KV shape differs, or when its attention span does not fit
 * the producer's ring (an SWA consumer with window > cache_cap - n_meta, or a
 * global consumer on a ring no longer than the producer's window). */
int hymba_kv_share(const hymba_kv* producer, const hymba_layer_cfg* consumer_cfg,
                   hymba_kv* consumer_out);

/* Workspace bytes for one call (0 if the configuration is invalid). For
 * HYMBA_MODE_DECODE, T is the cache_cap of the KV cache the step reads. */
size_t hymba_workspace_bytes(const hymba_layer_cfg* cfg, int B, int T, int mode);

/* Decode-state bytes of one layer for B sequences of up to max_T positions (meta
 * included): KV slots (producer only; n_meta + window, or max_T when global)
 * * (head_dim + v_head_dim) * element size (2 for bf16 layers, whose K/V are
 * fp16; 4 for fp32) * n_kv_heads * B, plus the fp32 SSM state, the fp32 conv state
 * and the int32 lengths. */
size_t hymba_cache_bytes(const hymba_layer_cfg* cfg, int B, int max_T);

/* KV bytes over several attention layers ("Jamba: Hybrid SSM-Transformer",
 * section 2 and Worked Example; "Lecture 04", section 8 kv_cache_gb):
 * batch * seq_len * n_attn_layers * n_kv_heads * (head_dim + v_head_dim) * dtype_bytes. */
uint64_t hymba_kv_bytes(int n_attn_layers, int n_kv_heads, int head_dim, int v_head_dim,
                        int64_t seq_len, int batch, int dtype_bytes);

/* SSM state bytes ("Lecture 04", section 8 ssm_state_gb):
 * n_layers * channels * d_state * batch * dtype_bytes. */
uint64_t hymba_ssm_state_bytes(int n_layers, int channels, int d_state, int batch,
                               int dtype_bytes);

/* Decode attention that allocates nothing and takes no workspace. The pages have no
 * counterpart: this entry point exists for callers that cannot call cudaMalloc or
 * hand the library a scratch buffer, for example a decode loop running inside
 * another runtime that owns every device allocation through its own pool, or a
 * latency-critical path where an allocation (which can synchronise the device) is
 * not allowed.
 *
 * It computes the attention step of hymba_mixer_decode on its own: for every sequence
 * b and query head, softmax attention of q[b] over the positions the decode cache
 * holds, the newest being the query's own (position len[b] - 1), limited to the meta
 * block plus the layer's window (or everything, for a global layer), with GQA.
 *   q:  device [B, n_q_heads * head_dim], row stride ldq elements, after RoPE; element
 *       type of the cache (fp16 for bf16 layers, fp32 for fp32 layers).
 *   kv: a decode cache (k_cache, v_cache, len) as filled by prefill/decode.
 *   o:  device [B, n_q_heads * v_head_dim], same element type.
 * The partial results of its key splits live in one file-scope device array of 8 MiB
 * (every GPU that loads the library holds it until the process exits). Requests with
 * B * n_q_heads * ceil(cache_cap / 256) * (v_head_dim + 4) * 4 bytes above that return
 * HYMBA_ERR_SCRATCH_LIMIT and queue no work. The first call on a device looks up the
 * array's device address (with that device current); make that first call before any
 * stream capture. All calls share the one array, and every call writes each partial
 * before reading it, so nothing needs clearing between calls; but calls whose kernels
 * overlap on the GPU (other streams, other host threads) race on it, so the caller
 * must order them. */
int hymba_attn_decode_static(const hymba_layer_cfg* cfg, const void* q, int64_t ldq, const hymba_kv* kv,
                             void* o, int B, void* stream);

/* Synchronises `stream`, then returns and clears the status word of the current
 * device: HYMBA_OK, HYMBA_ERR_DEVICE_TIMEOUT or HYMBA_ERR_DEVICE_RANGE; or
 * HYMBA_ERR_CUDA if the synchronisation itself failed. */
int hymba_get_device_status(void* stream);

/* Where the first bounded device wait that ran out gave up (after a call reported
 * HYMBA_ERR_DEVICE_TIMEOUT): out[0] 1 if a record exists, out[1..3] the block index
 * (x, y, z), out[4] the role (0 TMA producer, 1 MMA issuer, 2 epilogue/softmax,
 * 4 hymba_debug_stalled_wait; 3 is not used: the decode attention's copies are waited
 * for by the hardware's own copy-group wait, which always ends), out[5] the step (k-block
 * or key block), out[6] the barrier (or stage). Synchronises the device and clears the
 * record. Requires n >= 7. */
int hymba_get_device_diag(int32_t* out, int n);

/* Failure-path testing. Every device wait of the library that waits for progress
 * (an mbarrier phase a copy, an MMA or another role completes) gives up after a limit
 * of SM clock cycles (default 2e8, about 0.1 s), records HYMBA_ERR_DEVICE_TIMEOUT and
 * where it happened, and its block then waits (with the default limit) for the copies
 * and MMAs it already issued before it exits, so the context stays usable.
 * hymba_debug_set_wait_limit sets that limit for the current device (0 restores the
 * default; synchronises the device first). hymba_debug_stalled_wait queues one block
 * that waits, with that limit, on an mbarrier nothing arrives on: the wait runs out and
 * the status word then reads HYMBA_ERR_DEVICE_TIMEOUT, role 4. */
int hymba_debug_set_wait_limit(long long cycles);
int hymba_debug_stalled_wait(void* stream);

/* Layout of the workspace of one call, for callers that inspect the stage outputs
 * after a prefill (tests do): out[0] total bytes, out[1] byte offset of the
 * projection P [rows, ld_p] dtype (columns Q | (K V, unused) | x | z | B | C | dt_low),
 * out[2] ld_p in elements, out[3] offset of Delta [rows, d_inner] fp32 (not written
 * when a bf16 prefill computes Delta inside its scan kernel: dt_rank <= 128 and a
 * multiple of 4, and B * d_inner / 64 at least twice the SM count), out[4] of the
 * attention output O [rows, n_q_heads*v_head_dim] dtype, out[5] of y_pre = C.h + D xc
 * [rows, d_inner] dtype (before the SiLU(z) gate), out[6] of the fused U [rows,
 * d_inner] dtype, out[7] of the RoPE table, out[8] of the decode split partials,
 * out[9] the decode split count. rows = B * (n_meta + T) for prefill, B for decode
 * (where T is the cache_cap of the KV cache). A decode step writes neither Delta (it
 * stays in the SSM step's registers) nor O: its attention stays as the split partials
 * [B, n_q_heads, splits, v_head_dim + 4] fp32 (per split: the unnormalised sum of
 * p v, the split's max logit in base 2, the sum of p, and two pad words so that each
 * record starts on a 16-byte boundary), which the fusion merges.
 * Requires n >= 10. */
int hymba_workspace_layout(const hymba_layer_cfg* cfg, int B, int T, int mode, int64_t* out, int n);

/* Static description of a status code. */
const char* hymba_strerror(int code);

/* Opt-in per-kernel timing. While enabled, every kernel the library queues is
 * bracketed by CUDA events on its own stream. hymba_trace_collect synchronises
 * the device, writes up to max_records (name, milliseconds) pairs in launch order
 * (names are static strings) and returns how many it wrote; records beyond the
 * internal pool (8192) are dropped. Not thread-safe against concurrent
 * enable/collect; calls in between may come from any thread. */
int hymba_trace_enable(int on);
int hymba_trace_collect(const char** names, float* ms, int max_records);

/* Restrict tracing to the launches of one kernel name (as reported by
 * hymba_trace_collect; at most 63 characters), or trace every launch again with
 * NULL. Events between launches serialise the device-side overlap of consecutive
 * kernels, so a timing run traces only the kernel it reports. Returns
 * HYMBA_ERR_INVALID_ARG for a longer name. */
int hymba_trace_only(const char* name);

/* Number of kernels the library has queued since load (all entry points). */
uint64_t hymba_launch_count(void);

/* Measurement: throughput of the units that bound the library's CUDA-core kernels on
 * the current device, in results per clock per SM of the slowest SM (one 1024-thread
 * block per SM, 8 independent dependency chains per thread, timed with clock64):
 * out[0] exp2 in fp32 (ex2.approx.f32, the MUFU unit: the scan's state decays and the
 * softmax's exponentials), out[1] exp2 on fp16 pairs (ex2.approx.f16x2, counted per
 * half), out[2] fp32 FMA results of packed FFMA2 (two per instruction). Synchronises
 * `stream`; uses a fixed device array of the library (no allocation). Requires n >= 3. */
int hymba_probe_unit_rates(double* out, int n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* HYMBA_H */
