/*
 * ssa.h -- C ABI of the BLASST skip-softmax attention library for NVIDIA
 * B200 (sm_100a).
 *
 * The method (Model-Optimizer README "Skip-Softmax Sparse Attention for
 * Diffusion Models", introduction and "Threshold Modes"; Model-Optimizer
 * commit page, "Triton kernels"): non-causal FlashAttention over 128 x 128
 * tiles in which a KV tile whose scores all sit far below the running softmax
 * max is skipped outright -- no V load, no exponentials, no accumulation.
 * "Far below" is log2(lambda) in the log2 score domain, with
 * lambda = threshold_scale_factor / seq_len_kv computed per sequence
 * (README, "Threshold Modes", calibrated row; TRT-LLM VisualGen docs,
 * "Skip Softmax Attention": the kernel consumes threshold_scale_factor and
 * combines it with the sequence length at run time).
 *
 * Rules this library fixes where the pages are silent:
 *   s2[r,c]  = fp32(q_r . k_c) * fp32(softmax_scale * log2 e)
 *   d_j      = max over valid rows r of fp32(max_c s2[r,c] - m_r), where m_r
 *              is the running max over the KV tiles kept BEFORE tile j
 *              (d_0 = +inf); columns past the sequence end count as -inf and
 *              rows past it do not vote;
 *   skip j  <=> d_j < L, L = fp32(log2(threshold_scale_factor / S_kv));
 *   threshold_scale_factor <= 0 disables skipping (L = -inf).
 *
 * Layout. Q, K, V and out are bf16, packed varlen [total_tokens, H, D]
 * (row-major, D contiguous), D in {64, 128}; sequence b occupies rows
 * cu_seqlens[b] .. cu_seqlens[b+1]-1 (self-attention: S_q = S_kv). Its query
 * blocks are 128 rows each; the "global q-block" index numbers them over the
 * batch in order (sequence 0's blocks first). Per-unit outputs are indexed
 * [head][global q-block]; ssa_num_qblocks() gives their count Q.
 *
 * Ownership and streams. Every pointer argument is caller-owned; device
 * pointers must stay valid until the work on `stream` completes. `stream` is
 * a cudaStream_t (NULL = legacy default stream). The compute entry points
 * validate their arguments on the host, return a negative status before any
 * launch when they are wrong, enqueue work on `stream` and return without
 * synchronising. Errors a kernel detects (an inconsistent cu_seqlens, a
 * device wait that ran past its time limit) are recorded in a per-device
 * status word that ssa_get_error() reads. Q, K, V and out must be 16-byte
 * aligned. Every pointer documented as a device pointer must be device (or
 * managed) memory of the current device: the entry points check this with
 * cudaPointerGetAttributes before any launch and return SSA_ERR_INVALID_ARG
 * otherwise.
 *
 * Per-unit outputs. The caller sizes them from ssa_num_qblocks() (on a host
 * copy of cu_seqlens) and passes that count as num_qblocks; their inner
 * sizes follow from max_seqlen and n_thresholds. The kernels count the
 * q-blocks again from the device copy of cu_seqlens and, when the counts
 * differ (or a sequence is longer than max_seqlen where the diagnostics are
 * sized from it), write nothing at all and record SSA_ERR_DEVICE_ARG, so an
 * undersized buffer is never overrun. num_qblocks is ignored when no
 * per-unit output is given; a negative value with one is SSA_ERR_INVALID_ARG.
 *
 * Work order. For batches of up to 32 sequences the kernels start the
 * longest sequence's query blocks first (ties by position in the batch);
 * results do not depend on the order.
 */
#ifndef SSA_H_
#define SSA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SSA_OK = 0,
  SSA_ERR_INVALID_ARG = -1, /* bad pointer, size or value (host check)      */
  SSA_ERR_UNSUPPORTED = -2, /* head_dim not 64/128, misaligned pointer      */
  SSA_ERR_CUDA = -3,        /* a CUDA runtime or launch error               */
  SSA_ERR_TIMEOUT = -4,     /* a device-side wait exceeded its time limit   */
  SSA_ERR_DEVICE_ARG = -5   /* the kernel found cu_seqlens inconsistent (or
                               with num_qblocks / max_seqlen); nothing written */
};

#define SSA_TILE 128          /* Br = Bc = 128                                 */
#define SSA_MAX_THRESHOLDS 32 /* most thresholds one calibration call counts  */

/*
 * Skip-softmax attention forward (commit page, "Triton kernels": the
 * inference kernel with tile skipping and runtime sparsity counters).
 *   q, k, v      device bf16 [total_tokens, num_heads, head_dim]
 *   cu_seqlens   device int32 [batch + 1], non-decreasing, cu_seqlens[batch]
 *                <= total_tokens
 *   max_seqlen   >= every sequence length (sizes the debug outputs)
 *   softmax_scale   <= 0 selects 1/sqrt(head_dim)
 *   threshold_scale_factor  lambda * S_kv; <= 0 runs dense attention
 *   out          device bf16 [total_tokens, num_heads, head_dim]; rows of
 *                every sequence are written, nothing else is touched
 *   skip_counter device int32 [num_heads][Q] or NULL: tiles skipped per unit
 *                (plain stores, no atomics)
 *   num_qblocks  Q, the count skip_counter was sized for (see "Per-unit
 *                outputs" above)
 * Returns SSA_OK or a negative status.
 */
int ssa_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch, int total_tokens,
            int max_seqlen, int num_heads, int head_dim, float softmax_scale, float threshold_scale_factor,
            void* out, int32_t* skip_counter, int num_qblocks, void* stream);

/*
 * ssa_fwd plus per-tile diagnostics, for tests. T = ceil(max_seqlen / 128).
 *   decision_bitmap  device uint32 [num_heads][Q][ceil(T/32)] or NULL: bit
 *                    (j & 31) of word (j >> 5) is 1 when KV tile j was skipped
 *   tile_stat        device float [num_heads][Q][T] or NULL: the statistic
 *                    d_j of every tile (+inf for tile 0; entries past the
 *                    sequence's last tile are left untouched)
 * With threshold_scale_factor <= 0 the statistics follow the dense trajectory.
 */
int ssa_fwd_ex(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch, int total_tokens,
               int max_seqlen, int num_heads, int head_dim, float softmax_scale, float threshold_scale_factor,
               void* out, int32_t* skip_counter, int num_qblocks, uint32_t* decision_bitmap, float* tile_stat,
               void* stream);

/*
 * Calibration pass (commit page, "Triton kernels": full attention that counts
 * how many tiles would be skipped at each of N thresholds at once, with
 * per-program output buffers and no atomics; threshold trials from
 * Model-Optimizer PR #1166, "Usage").
 *   thresholds    HOST float [n_thresholds], raw lambda values (> 0), each
 *                 compared as log2(lambda); 1 <= n_thresholds <= 32
 *   out           device bf16, the dense attention output
 *   counts        device int32 [num_heads][Q][n_thresholds]: per unit, the
 *                 number of KV tiles j >= 1 with d_j < log2(lambda_k) on the
 *                 dense trajectory. For lambda_k <= 1 this equals ssa_fwd's
 *                 skip count at threshold_scale_factor = lambda_k * S_kv.
 *   num_qblocks   Q, the count `counts` was sized for
 */
int ssa_calibrate(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                  int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                  const float* thresholds, int n_thresholds, void* out, int32_t* counts, int num_qblocks,
                  void* stream);

/*
 * ssa_calibrate plus the statistic behind every count, for tests (the
 * calibration kernel's per-program buffers, commit page "Triton kernels"):
 *   tile_stat  device float [num_heads][Q][T], T = ceil(max_seqlen / 128), or
 *              NULL: d_j of every tile on the dense trajectory (+inf for tile
 *              0; entries past the sequence's last tile are left untouched),
 *              so that counts[.][.][k] = #{ j : tile_stat[.][.][j] < log2(lambda_k) }.
 */
int ssa_calibrate_ex(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                     int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                     const float* thresholds, int n_thresholds, void* out, int32_t* counts, int num_qblocks,
                     float* tile_stat, void* stream);

/*
 * ssa_fwd_ex with 8-bit Q and K: S = Q K^T runs on E4M3 operands (OCP FP8,
 * no infinities; tcgen05 kind::f8f6f4) while V, P and the output stay bf16.
 * The TRT-LLM docs ("VisualGen Sparse Attention (Beta)", "User
 * Configuration") state that skip-softmax composes with quantised Q/K
 * attention; its pull-request page ("Benchmark") reports FP8 speed-ups.
 * Reading: one scale per tensor, so the real Q is q_descale * decode(q) and
 * likewise for K, and the scores are
 *   s2[r,c] = fp32(decode(q_r) . decode(k_c)) * fp32(softmax_scale * q_descale * k_descale * log2 e)
 * with every rule of ssa_fwd unchanged after that.
 *   q, k        device E4M3 bytes [total_tokens, num_heads, 128] (head_dim must be 128)
 *   v, out      device bf16 [total_tokens, num_heads, 128]
 *   q_descale, k_descale  > 0, finite
 *   skip_counter, num_qblocks, decision_bitmap, tile_stat  as in ssa_fwd_ex
 *                (the three buffers each nullable)
 * Returns SSA_OK or a negative status (SSA_ERR_UNSUPPORTED for head_dim != 128).
 */
int ssa_fwd_fp8(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch, int total_tokens,
                int max_seqlen, int num_heads, int head_dim, float softmax_scale, float q_descale, float k_descale,
                float threshold_scale_factor, void* out, int32_t* skip_counter, int num_qblocks,
                uint32_t* decision_bitmap, float* tile_stat, void* stream);

/*
 * ssa_fwd_fp8 with V in E4M3 as well, and P rounded to E4M3 for the P.V
 * product: both MMAs run on 8-bit operands (tcgen05 kind::f8f6f4). The
 * TRT-LLM pull-request page ("Benchmark") reports skip-softmax speed-ups with
 * FP8 and NVFP4 attention; the docs ("User Configuration") name skip-softmax
 * combined with quantised attention. Reading, where the pages are silent:
 * one scale per tensor (real V = v_descale * decode(v)); the skip rule and
 * its running max m are those of ssa_fwd; each row takes its probabilities
 * against an integer reference r >= m that moves to ceil(m) as soon as m
 * passes it (rescaling O and l by the exact power of two 2^(r_old - r_new)),
 * P = 2^(s2 - r + 8) in (0, 256], the P.V product uses P rounded to the
 * nearest E4M3 value while the row sum l adds the unrounded P, and the output
 * is v_descale * O / l in bf16.
 *   q, k, v     device E4M3 bytes [total_tokens, num_heads, 128]
 *   out         device bf16 [total_tokens, num_heads, 128]
 *   q_descale, k_descale, v_descale  > 0, finite
 *   other arguments as in ssa_fwd_fp8
 */
int ssa_fwd_fp8_qkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                    int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                    float q_descale, float k_descale, float v_descale, float threshold_scale_factor, void* out,
                    int32_t* skip_counter, int num_qblocks, uint32_t* decision_bitmap, float* tile_stat,
                    void* stream);

/*
 * ssa_calibrate with E4M3 Q, K and V: the dense pass of ssa_fwd_fp8_qkv and its
 * counts (which depend on Q and K only, so they equal ssa_calibrate_fp8's).
 * Arguments as in ssa_calibrate_fp8, plus v_descale.
 */
int ssa_calibrate_fp8_qkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                          int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                          float q_descale, float k_descale, float v_descale, const float* thresholds,
                          int n_thresholds, void* out, int32_t* counts, int num_qblocks, void* stream);

/*
 * Per-tensor E4M3 quantisation for ssa_fwd_fp8: y[i] = E4M3(fp32(x[i] * inv_scale)),
 * round to nearest even, saturating to +-448 (a caller with amax = max|x|
 * passes inv_scale = 448 / amax and then q_descale = 1 / inv_scale).
 *   x  device bf16 [n], 16-byte aligned;  y  device bytes [n], 8-byte aligned
 * Returns SSA_OK, SSA_ERR_INVALID_ARG (n < 0, inv_scale not finite and > 0,
 * NULL with n > 0) or SSA_ERR_UNSUPPORTED (misaligned pointer).
 */
int ssa_quantize_fp8(const void* x, void* y, int64_t n, float inv_scale, void* stream);

/*
 * ssa_calibrate with 8-bit Q and K: the dense pass and its counts on the
 * scores ssa_fwd_fp8 defines (E4M3 Q, K with per-tensor descales; V and out
 * bf16; head_dim 128). For lambda_k <= 1 the count equals ssa_fwd_fp8's skip
 * count at threshold_scale_factor = lambda_k * S_kv. Arguments as in
 * ssa_calibrate and ssa_fwd_fp8.
 */
int ssa_calibrate_fp8(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                      int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                      float q_descale, float k_descale, const float* thresholds, int n_thresholds, void* out,
                      int32_t* counts, int num_qblocks, void* stream);

/*
 * threshold_scale_factor = a * exp(b * target_sparsity) (README, "Calibrated
 * threshold"; TRT-LLM VisualGen docs, "Checkpoint Config"). Returns NaN when
 * a <= 0, target_sparsity is outside [0, 1] or an argument is not finite.
 * A caller holding log_a passes exp(log_a).
 */
double ssa_resolve(double a, double b, double target_sparsity);

/*
 * Log-space least-squares fit of ln(scale_factor) = ln(a) + b * sparsity
 * (commit page, "Calibration": fit_logspace minimises relative error and the
 * observed sparsity range is recorded for extrapolation warnings). Points
 * with sparsity outside (0, 1) or scale_factor <= 0 are ignored. Writes a, b
 * and the observed [s_min, s_max] of the points used. Host arrays. Returns
 * SSA_OK, or SSA_ERR_INVALID_ARG when fewer than two distinct usable
 * sparsities remain or a pointer is NULL.
 */
int ssa_fit_logspace(const double* sparsity, const double* scale_factor, int n, double* a, double* b, double* s_min,
                     double* s_max);

/* Number of 128-row query blocks Q over the batch, from a HOST copy of
 * cu_seqlens; negative status when it is inconsistent. */
int ssa_num_qblocks(const int32_t* cu_seqlens_host, int batch);

/* Synchronise `stream`, then return this device's kernel status (SSA_OK,
 * SSA_ERR_TIMEOUT, SSA_ERR_DEVICE_ARG or SSA_ERR_CUDA) and clear the bits it
 * read, atomically on the device: an error that a kernel on another stream
 * records meanwhile is kept for the next call, not lost. */
int ssa_get_error(void* stream);

/* Static description of a status code. */
const char* ssa_status_string(int status);

/* Diagnostic for failure detection: runs the kernels' bounded mbarrier wait
 * (the one every producer/consumer wait uses) on a barrier nothing arrives
 * on, giving up after limit_ns (1 .. 1e9). Writes device int[3]: completed
 * (expected 0), abort flag raised (expected 1), microseconds waited. The
 * wait also records SSA_ERR_TIMEOUT in the device status word, which
 * ssa_get_error() then returns and clears. No fault, no hang. */
int ssa_wait_timeout_check(int* result, int64_t limit_ns, void* stream);

/* Text of the last CUDA error this library saw on the calling host thread
 * (the cause behind an SSA_ERR_CUDA); "no error" if none. Static storage. */
const char* ssa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H_ */
