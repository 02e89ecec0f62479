// Host-side launchers of the library's kernels (one kernel per launcher).
#pragma once
#include "common.cuh"
#include "epilogue.cuh"

namespace hymba {

// Launch context (stream, status word, SM count) of the current device.
int launch_context(cudaStream_t stream, Ctx* ctx);

// C = A B^T on CUDA cores (fp32 accumulate); A [M, K] (row stride lda), Bw [N, K]
// (row stride ldb); the result goes through epi_run64.
template <typename TA, typename TO>
int launch_gemm_simt(const Ctx& ctx, const char* name, const TA* A, long long lda, const TA* Bw, long long ldb,
                     int M, int N, int K, const EpiArgs<TO>& e);

// C = A B^T on the tcgen05 tensor cores (bf16 or fp16 in, fp32 accumulate in TMEM).
// Requirements: lda, ldb multiples of 8 elements, A and Bw 16-byte aligned. With A0
// (M0 > 0 rows, same lda) the launch also covers A0's rows, handed to the epilogue
// as meta rows (in-projection only): one launch for the meta and the user rows.
template <typename TA, typename TO>
int launch_gemm_tc(const Ctx& ctx, const char* name, const TA* A, long long lda, const TA* Bw, long long ldb,
                   int M, int N, int K, const EpiArgs<TO>& e, const TA* A0 = nullptr, int M0 = 0);

// Causal GQA attention over the meta prefix + window, CUDA cores.
template <typename T>
int launch_attn_prefill_simt(const Ctx& ctx, const T* P, long long ldP, const T* k_seq,
                             const T* v_seq, int kcap, T* O, int B, int Tp, int H, int G,
                             int dv, int n_meta, int window);

// Causal GQA attention over the meta prefix + window, tcgen05 tensor cores (bf16).
int launch_attn_prefill_tc(const Ctx& ctx, const f16* P, long long ldP, const f16* k_seq,
                           const f16* v_seq, int kcap, f16* O, int B, int Tp, int H, int G,
                           int dv, int n_meta, int window);

// Depthwise causal conv + SiLU + selective scan over the T' rows of every sequence,
// Delta from `delta` [rows, di] fp32; hp > 0 (the SSD form, hp channels per head, a
// multiple of 8): `delta` [rows, di / hp] and A_log [di / hp], one value per head.
template <typename T>
int launch_conv_scan_prefill(const Ctx& ctx, const T* P, long long ldP, int col_x, int col_B,
                             int col_C, const float* delta, const float* conv_w,
                             const float* conv_b, const float* A_log, const float* D, T* ypre,
                             float* h_out, float* conv_out, int B, int Tp, int di, int hp);

// The same for 16-bit intermediates with Delta computed in the kernel (dt_rank <= 128, a
// multiple of 4), one thread per channel pair and state half: for batches where
// B * d_inner fills the GPU (scan_wide_applies).
bool scan_wide_applies(int B, int di, int dt_rank, int sm_count);
int launch_conv_scan_wide(const Ctx& ctx, const f16* P, long long ldP, int col_x, int col_B, int col_dt, int dt_rank,
                          const f16* wdt, int ld_wdt, const float* b_dt, const float* conv_w, const float* conv_b,
                          const float* A_log, const float* D, f16* ypre, float* h_out, float* conv_out, int B, int Tp,
                          int di);

// conv + SiLU and the SSD-form scan (scalar A and Delta per SSM head of 64 channels) as
// chunked tensor-core matmuls, fp16 operands; delta [rows, ld_delta] per head.
bool ssd_scan_applies(int di, int ssm_heads);
int launch_ssd_scan(const Ctx& ctx, const f16* P, long long ldP, int col_x, int col_B, const float* delta,
                    int ld_delta, const float* conv_w, const float* conv_b, const float* A_log, const float* D,
                    f16* ypre, float* h_out, float* conv_out, int B, int Tp, int di, int ssm_heads);

// RMSNorm of both branches, SiLU(z) gate, beta scaling and average (U [rows, di]) or
// concatenation (U [rows, di + H*dv] = [Mamba | attention]); one row per block.
// Decode only: y_init [rows, d_model] is set to y_res (or zero) for a split-K output
// projection that adds its partial sums to it.
// The attention branch is O [rows, H*dv], or, when `part` is given, the decode
// attention's split partials [rows, H, n_split, dv + 2] merged on the fly (O unused).
// A consumer's adapted shared V (v_scale, v_bias [G, dv], both or neither) is applied
// to the attention output before its norm.
template <typename I, typename T>
int launch_fuse(const Ctx& ctx, const I* O, const float* part, int n_split, int H, int G, int dv, bool concat,
                const I* ypre, const I* P, long long ldP, int col_z, const float* g_attn, const float* g_ssm,
                const float* beta1, const float* beta2, const float* v_scale, const float* v_bias, T* U,
                int rows, int di, float eps, int* len_inc, float* y_init = nullptr, const float* y_res = nullptr,
                int d_model = 0);


// The RoPE table and the zero-padded 16-bit copy of W_dt [rows, cols] -> [rows, ld_dst],
// in one launch.
template <typename TS, typename TD>
int launch_prefill_prep(const Ctx& ctx, float2* tab, int Tp, int dh, float base, const TS* w, int rows, int cols,
                        TD* wdst, int ld_dst);

// The RoPE table of a decode step's new positions ([B, dh/2] (cos, sin)) and a copy
// of the [rows, cols] matrix w converted to TD into [rows, ld_dst] (zero-padded; the
// decode step's input rows when they arrive in another type; rows = 0: none), in one
// launch.
template <typename TS, typename TD>
int launch_decode_prep(const Ctx& ctx, float2* tab, const int* len, int pos_offset, int B, int dh, float base,
                       const TS* w, int rows, int cols, TD* wdst, int ld_dst);

// dst [rows, cols] = g * src / sqrt(mean(src^2) + eps) per row (cols <= 4096, a
// multiple of 8; 16-byte aligned rows).
template <typename TS, typename TD>
int launch_rmsnorm_rows(const Ctx& ctx, const TS* src, const float* g, TD* dst, long long rows, int cols, float eps);

// Copy a [rows, cols] matrix into a zero-padded [rows, ld_dst] one of type TD.
template <typename TS, typename TD>
int launch_pad_copy(const Ctx& ctx, const TS* src, int rows, int cols, TD* dst, int ld_dst);

// Fill the decode cache of a producer from its prefill sequence K/V and set len = Tp.
template <typename T>
int launch_cache_fill(const Ctx& ctx, const T* k_seq, const T* v_seq, int seq_cap, T* k_cache,
                      T* v_cache, int cache_cap, int* len, int B, int G, int dh, int dv,
                      int n_meta, int Tp);

// Decode attention: one query per (sequence, head) over the cache; split over keys,
// partial results in `part` [B, H, n_split, dv + 2] fp32, then combined into O
// (O == nullptr: left as partials for the fusion kernel to merge).
template <typename T>
int launch_attn_decode(const Ctx& ctx, const T* P, long long ldP, const T* k_cache,
                       const T* v_cache, int cache_cap, const int* len, int pos_offset,
                       float* part, int n_split, T* O, int B, int H, int G, int dv, int n_meta,
                       int window);

// One SSM decode step per (sequence, channel): Delta = softplus(dt_low W_dt^T + b_dt)
// from the projection row's dt_low columns, conv-state shift, conv, SiLU, scan step on
// h in place, y_pre = C.h + D xc. W_dt is [di, dt_rank] in the layer's weight type.
// The decode attention (split partials) and the SSM step of a layer in one launch
// (16-bit layers): the same arguments as the two launches above.
template <typename TW>
int launch_decode_attn_ssm(const Ctx& ctx, const f16* P, long long ldP, const f16* k_cache, const f16* v_cache,
                           int cache_cap, const int* len, int pos_offset, float* part, int n_split, int B, int H,
                           int G, int dv, int n_meta, int window, int col_x, int col_B, int col_C, int col_dtl,
                           const TW* w_dt, const float* b_dt, int dt_rank, const float* conv_w, const float* conv_b,
                           const float* A_log, const float* D, float* h, float* conv, f16* ypre, int di, int hp);

template <typename T, typename TW>
int launch_ssm_decode(const Ctx& ctx, const T* P, long long ldP, int col_x, int col_B, int col_C,
                      int col_dtl, const TW* w_dt, const float* b_dt, int dt_rank,
                      const float* conv_w, const float* conv_b, const float* A_log, const float* D,
                      float* h, float* conv, T* ypre, int B, int di, int hp);

}  // namespace hymba
