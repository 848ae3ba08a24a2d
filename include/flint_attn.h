/*
 * flint_attn.h - C ABI of a B200 (sm_100a) library for Flint's sink-aware
 * sliding/full GQA attention, forward and backward.
 *
 * What the calls compute (the passages that define it):
 *   - Per-head RMSNorm of q and k with eps = rms_norm_eps (1e-6 by default):
 *     Flint layers page (nemo_automodel.components.models.flint.layers),
 *     FlintAttention class summary (separate Q/K/V projections, an RMSNorm per
 *     head, RoPE on selected layers, learned sinks), attributes q_norm,
 *     k_norm, eps; Flint config page
 *     (nemo_automodel.components.models.flint.config), FlintConfig.rms_norm_eps.
 *     Reading: one weight vector [D] for q and one for k, shared by all heads,
 *     applied as w * x / sqrt(mean(x^2) + eps).
 *   - NeoX RoPE over all head channels on sliding layers, none on full layers:
 *     FlintAttention._apply_rope (channel j rotates with channel j + D/2) and the
 *     FlintConfig docstring. Frequencies theta^(-2j/D); positions restart at 0
 *     in every document (FlintAttention.forward, position_ids for THD).
 *     RMSNorm is applied first, then RoPE.
 *   - Causal window that includes the current token; window <= 0 is unbounded:
 *     FlintConfig docstring and sliding_window; attention utils page
 *     (nemo_automodel.components.attention.utils),
 *     preprocess_args_and_kwargs_for_attn (its window_size convention).
 *   - THD packing: documents given by cu_doc_lens int32 [num_docs + 1], the
 *     cu_seqlens format of preprocess_args_and_kwargs_for_attn; attention never
 *     crosses a document boundary.
 *   - GQA: query head h reads KV head h / (H / Hk).
 *   - One learned FP32 sink logit per query head, unscaled, entering only the
 *     softmax denominator with a zero value: _FlintSinkParameters.forward and
 *     FlintAttention.forward (the sink is one more softmax category, whose
 *     value vector is zero).
 *     LSE_i = ln(e^{sink_h} + sum_j e^{z_ij}),  O_i = sum_j e^{z_ij - LSE_i} v_j,
 *     z_ij = softmax_scale * q_hat_i . k_hat_j.
 *   - Backward: gradients of sum(dO * O) w.r.t. q, k, v (raw inputs, before
 *     norm and RoPE), both norm weights and the sinks. The learned-sink training
 *     kernel is named on the Flint layers page (module docstring).
 *     d sink_h = -sum_i e^{sink_h - LSE_i} (dO_i . O_i).
 *
 * Conventions for every call:
 *   - All tensor arguments are DEVICE pointers owned by the caller, contiguous,
 *     row-major, 16-byte aligned. The library allocates no memory. Calls run on
 *     the device current when they are made; one process may drive several
 *     devices, from several host threads. State kept between calls, per device:
 *     the SM count, each kernel's raised dynamic shared-memory limit (set at the
 *     first call that launches it there), and, for
 *     flint_attn_bwd_preprocess_static only, the address of a fixed scratch
 *     array in device memory (see there).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Results are ready when the stream is synchronised.
 *   - Argument errors are returned before any launch (no GPU work is queued).
 *     A failed launch returns FLINT_ERR_CUDA. Device-side waits are bounded:
 *     a wait that runs out sets a status word in the workspace, which
 *     flint_attn_check_status() turns into FLINT_ERR_TIMEOUT.
 *   - Layouts: q, out, dout, dq [T, H, D]; k, v, dk, dv [T, Hk, D];
 *     q_norm_w, k_norm_w [D]; sink, dsink [H] fp32; lse [H, T] fp32;
 *     dq_norm_w, dk_norm_w [D] fp32.
 *   - An empty batch (T = 0; documents of length 0) is valid: the [T, ...]
 *     tensors (q, k, v, out, lse, dout, dq, dk, dv) may then be null. The
 *     forward writes nothing; the backward writes zero dsink and norm-weight
 *     gradients.
 *   - dtype FLINT_BF16: q, k, v, dout and the norm weights are bfloat16; out,
 *     dq, dk, dv are bfloat16, or float32 with params->fp32_out. The attention
 *     contractions run on tcgen05 tensor cores with FP32 accumulation; their
 *     operands (q_hat, k_hat, v, P, and in the backward dout and dS) are IEEE
 *     fp16, whose 10-bit mantissa keeps their rounding well below bf16's.
 *     |v| and |dout| must stay below 65504 (larger values saturate).
 *     dtype FLINT_FP32: all tensors are float32. With G = 1, 2, 4, 8 or 16 the
 *     attention contractions run on tcgen05 tensor cores at FP32 accuracy:
 *     each operand x enters as two fp16 parts, hi = fp16(x) and
 *     lo = fp16(x - hi), and each product takes three MMAs (hi*hi + hi*lo +
 *     lo*hi) with FP32 accumulation; v and dout are scaled by powers of two
 *     (as above), so any float32 magnitude is taken. RMSNorm, RoPE, the
 *     softmax and every reduction run in FP32. Other group sizes run every
 *     step in FP32 on CUDA cores (no padded calls there).
 */
#ifndef FLINT_ATTN_H
#define FLINT_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FLINT_OK = 0,
  FLINT_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad cu_doc_lens bound */
  FLINT_ERR_UNSUPPORTED = 2,   /* valid but not implemented: head_dim != 128, G not in {1,2,4,8,16} */
  FLINT_ERR_WORKSPACE = 3,     /* workspace smaller than flint_attn_workspace_bytes() */
  FLINT_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  FLINT_ERR_TIMEOUT = 5        /* a device-side wait ran out (see flint_attn_check_status) */
} flint_status_t;

typedef enum { FLINT_BF16 = 0, FLINT_FP32 = 1 } flint_dtype_t;

typedef struct {
  int32_t total_tokens;   /* T = cu_doc_lens[num_docs]; 0 <= T < 2^31 / H / D */
  int32_t num_docs;       /* N >= 1; zero-length documents are allowed */
  int32_t num_q_heads;    /* H, a multiple of num_kv_heads */
  int32_t num_kv_heads;   /* Hk >= 1; G = H / Hk must be 1, 2, 4, 8 or 16 (tensor-core
                             paths; FP32 inputs without compute_f16 take any G, other
                             values on CUDA cores) */
  int32_t head_dim;       /* D; must be 128 */
  int32_t window;         /* > 0: key j visible from query i iff 0 <= i - j < window
                             (the current token included); <= 0: full causal */
  int32_t use_rope;       /* nonzero: NeoX RoPE on all D channels after RMSNorm */
  float rope_theta;       /* RoPE base (> 0 when use_rope) */
  float rms_eps;          /* RMSNorm epsilon (Flint: 1e-6) */
  float softmax_scale;    /* 0 => 1/sqrt(head_dim) */
  int32_t dtype;          /* flint_dtype_t */
  int32_t fp32_out;       /* nonzero => out (forward, and as passed to the backward) and
                             dq, dk, dv are float32; zero => same type as q. FP32 inputs
                             always use float32 (but see compute_f16). */
  int32_t compute_f16;    /* FP32 inputs only (else FLINT_ERR_INVALID_ARG): the fp16
                             attention boundary of attention_compute_dtype='fp16' (Flint
                             config page: an fp16 QKV/kernel-output boundary inside
                             otherwise FP32 compute). RMSNorm and RoPE run in FP32; q_hat,
                             k_hat, v (and dout in the backward) enter the tcgen05
                             tensor-core path as fp16, and out is written as IEEE fp16
                             (float32 with fp32_out). dq, dk, dv and the norm-weight and
                             sink gradients stay float32. G must be 1, 2, 4, 8 or 16. */
} flint_attn_params_t;

/* Bytes of device workspace a call needs (backward = 0 for flint_attn_fwd,
 * 1 for flint_attn_bwd). Returns 0 if the params are invalid. The workspace
 * must be 256-byte aligned and is not used after the call's kernels finish. */
size_t flint_attn_workspace_bytes(const flint_attn_params_t* params, int backward);

/* Forward: O and LSE.
 *   q [T,H,D], k [T,Hk,D], v [T,Hk,D], q_norm_w [D], k_norm_w [D]  (dtype)
 *   sink [H] fp32, cu_doc_lens [num_docs+1] int32 (device, non-decreasing,
 *   cu_doc_lens[0] = 0, cu_doc_lens[num_docs] = T; not checked on the device)
 *   out [T,H,D] (dtype, or float32 with fp32_out), lse [H,T] fp32 (natural log). */
flint_status_t flint_attn_fwd(const flint_attn_params_t* params,
                              const void* q, const void* k, const void* v,
                              const void* q_norm_w, const void* k_norm_w,
                              const float* sink, const int32_t* cu_doc_lens,
                              void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Backward of sum(dout * out) for out = flint_attn_fwd(...).
 *   out, lse: the forward's results for the same inputs; dout [T,H,D] (dtype).
 *   out must have the type the forward wrote (float32 with fp32_out): D = dO . O
 *   is formed from it, and the bf16 rounding of O is the largest error source
 *   of the sink and norm-weight gradients.
 *   Writes dq [T,H,D], dk [T,Hk,D], dv [T,Hk,D] (gradients w.r.t. the RAW q, k,
 *   v; float32 with fp32_out, else the input type), dq_norm_w, dk_norm_w [D]
 *   fp32, dsink [H] fp32. Outputs are overwritten, not accumulated. q and k are
 *   re-normalised and re-rotated inside (nothing from the forward besides out
 *   and lse is needed). */
flint_status_t flint_attn_bwd(const flint_attn_params_t* params,
                              const void* q, const void* k, const void* v,
                              const void* q_norm_w, const void* k_norm_w,
                              const float* sink, const int32_t* cu_doc_lens,
                              const void* out, const float* lse, const void* dout,
                              void* dq, void* dk, void* dv,
                              float* dq_norm_w, float* dk_norm_w, float* dsink,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ---- Padding ------------------------------------------------------------
 * flint_attn_fwd / flint_attn_bwd with trailing padding in every document: a
 * BSHD attention_mask as the attention utils page
 * (nemo_automodel.components.attention.utils) hands it to TE, which takes
 * trailing padding only. BSHD [B, S] is cu_doc_lens = [0, S, 2S, ..., B*S].
 *   valid_lens [num_docs] int32 (device): document d's first valid_lens[d]
 *   tokens are real (clamped to [0, length]); the rest are padding.
 * Padded queries and keys are excluded while the sink stays valid (Flint
 * layers page, FlintAttention.forward): a padded row gets out = 0 and
 * lse = sink_h; real rows see only real keys; every gradient row at a padded
 * token (dq, dk, dv) is zero, and padded rows add nothing to dsink or the
 * norm-weight gradients. RoPE positions still count from the document start,
 * so real tokens are unaffected by the padding after them. Same workspace as
 * the unpadded calls; the tensor-core paths only (FLINT_ERR_UNSUPPORTED for
 * FLINT_FP32 inputs whose G is not 1, 2, 4, 8 or 16). Other arguments as in
 * flint_attn_fwd / flint_attn_bwd. */
flint_status_t flint_attn_fwd_padded(const flint_attn_params_t* params,
                                     const void* q, const void* k, const void* v,
                                     const void* q_norm_w, const void* k_norm_w,
                                     const float* sink, const int32_t* cu_doc_lens,
                                     const int32_t* valid_lens, void* out, float* lse,
                                     void* workspace, size_t workspace_bytes, void* stream);

flint_status_t flint_attn_bwd_padded(const flint_attn_params_t* params,
                                     const void* q, const void* k, const void* v,
                                     const void* q_norm_w, const void* k_norm_w,
                                     const float* sink, const int32_t* cu_doc_lens,
                                     const int32_t* valid_lens, const void* out,
                                     const float* lse, const void* dout,
                                     void* dq, void* dk, void* dv,
                                     float* dq_norm_w, float* dk_norm_w, float* dsink,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* ---- Decode over a KV cache ----------------------------------------------
 * The forward of one NEW token per sequence, for serving (the pages mention
 * serving kernels on the Flint layers page, module docstring, and a KV cache
 * through use_cache on the Flint config page). It computes exactly what
 * flint_attn_fwd computes for the last token of each sequence, with the earlier
 * tokens' keys and values taken from caches instead of recomputed:
 *   sequence b has cache_lens[b] = p tokens cached (positions 0..p-1); its new
 *   token is at position p. q_hat = RoPE_p(RMSNorm(q)) and k_hat =
 *   RoPE_p(RMSNorm(k)) as in the forward; k_hat and v are first written into
 *   slot p of k_cache / v_cache (rounded to bf16), then the new query attends
 *   to slots j with max(0, p - W + 1) <= j <= p (W <= 0: 0..p), plus the sink:
 *   LSE = ln(e^{sink_h} + sum_j e^{z_j}), O = sum_j e^{z_j - LSE} v_j.
 * Layouts: q [B, H, D]; k, v [B, Hk, D] (raw projections of the new token,
 *   bfloat16); q_norm_w, k_norm_w [D] bf16; sink [H] fp32; cache_lens [B] int32
 *   (device); k_cache, v_cache [B, Hk, C, D] bfloat16, head-major per sequence
 *   (slot j of KV head g of sequence b at ((b * Hk + g) * C + j) * D); k_cache
 *   holds normalised, rotated keys. out [B, H, D] (bf16, or float32 with
 *   fp32_out); lse [B, H] fp32 (natural log).
 * Only dtype FLINT_BF16 is supported (FLINT_ERR_UNSUPPORTED otherwise); H/Hk
 *   must be <= 16. Slot p must exist (0 <= p < C): a sequence whose cache_lens
 *   entry is out of range is skipped on the device (out and lse are left
 *   untouched, nothing is written to its cache) and the status word records it;
 *   flint_attn_check_status() then returns FLINT_ERR_INVALID_ARG.
 * The caches are read and written in place; the call does not allocate.
 * Asynchronous on `stream`. */
typedef struct {
  int32_t batch;            /* B >= 1 sequences, one new token each */
  int32_t cache_capacity;   /* C >= 1 slots per (sequence, KV head) */
  int32_t num_q_heads;      /* H */
  int32_t num_kv_heads;     /* Hk; H % Hk == 0, H / Hk <= 16 */
  int32_t head_dim;         /* D; must be 128 */
  int32_t window;           /* > 0: keys p-W+1..p visible; <= 0: unbounded */
  int32_t use_rope;         /* NeoX RoPE at position p */
  float rope_theta;
  float rms_eps;            /* 1e-6 in the Flint config */
  float softmax_scale;      /* 0 => 1/sqrt(head_dim) */
  flint_dtype_t dtype;      /* FLINT_BF16 */
  int32_t fp32_out;         /* out in float32 instead of bf16 */
} flint_decode_params_t;

/* Bytes of device workspace flint_attn_decode needs (0 if the params are
 * invalid). 256-byte aligned; not used after the call's kernels finish. */
size_t flint_attn_decode_workspace_bytes(const flint_decode_params_t* params);

flint_status_t flint_attn_decode(const flint_decode_params_t* params,
                                 const void* q, const void* k, const void* v,
                                 const void* q_norm_w, const void* k_norm_w,
                                 const float* sink, const int32_t* cache_lens,
                                 void* k_cache, void* v_cache,
                                 void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Largest num_q_heads flint_attn_bwd_preprocess_static accepts. */
#define FLINT_STATIC_MAX_HEADS 128

/* Backward preprocess without a workspace and without allocating: writes
 * d_rowsum [H,T] fp32 (D_i = dout_i . out_i per row) and dsink [H] fp32, the
 * same values flint_attn_bwd computes for its own use. The source pages have
 * no counterpart of this call; it exists for callers that cannot allocate
 * device memory where they run (a fixed-budget serving loop, a plugin that is
 * given tensors but no workspace, a path where cudaMalloc/cudaFree would
 * synchronise the device).
 *   params: total_tokens, num_q_heads, head_dim (128), dtype, fp32_out and
 *   compute_f16 are read; they fix the type of out exactly as for flint_attn_bwd
 *   (float32 with fp32_out or for FP32 inputs; IEEE fp16 for FP32 inputs with
 *   compute_f16 and without fp32_out; else bfloat16), and dout has the input
 *   type. compute_f16 with BF16 inputs is FLINT_ERR_INVALID_ARG;
 *   num_q_heads <= FLINT_STATIC_MAX_HEADS, else FLINT_ERR_WORKSPACE (both
 *   before any launch).
 *   out, dout [T,H,D], lse [H,T] fp32, sink [H] fp32: device inputs.
 *   d_rowsum [H,T], dsink [H]: device outputs (overwritten). With T = 0 the
 *   [T, ...] pointers (out, dout, lse, d_rowsum) may be null; dsink is zeroed.
 * Its scratch is a fixed 592 KiB array in device memory, held by every GPU that
 * loads the library until exit and shared by all calls: calls whose kernels
 * overlap on the GPU (unordered streams) race on it. The first call on a device
 * looks the array up with that device current and keeps its address for the
 * rest of the process; make it before any stream capture on that device, and
 * do not call this entry point on a device again after cudaDeviceReset (the
 * kept address belongs to the reset context). Asynchronous on `stream`. */
flint_status_t flint_attn_bwd_preprocess_static(const flint_attn_params_t* params,
                                                const void* out, const void* dout,
                                                const float* lse, const float* sink,
                                                float* d_rowsum, float* dsink, void* stream);

/* Synchronises `stream`, reads and clears the device status word in
 * `workspace` (written by bounded device waits), and returns FLINT_OK or
 * FLINT_ERR_TIMEOUT (FLINT_ERR_INVALID_ARG for a flint_attn_decode workspace
 * whose call met an out-of-range cache_lens entry). It returns FLINT_ERR_CUDA
 * if the stream itself reports an error, or if a backward kernel found its
 * dynamic shared memory not 1024-byte aligned and did no work (its tiles need
 * that alignment; not expected). */
flint_status_t flint_attn_check_status(void* workspace, void* stream);

/* ---- Measurement aids (not needed to compute anything) --------------------
 * flint_attn_profile_enable(1): later calls bracket each of their kernel
 * launches with a pair of CUDA events recorded on the call's stream (events are
 * created on first use and reused; no device memory is allocated).
 * flint_attn_profile_collect(): synchronises the recorded events, adds each
 * launch's duration into per-kernel totals and frees the event slots; then
 * fills up to max_kernels entries of names / total_ms / launches and returns
 * the number of kernel kinds. flint_attn_profile_reset() zeroes the totals.
 * flint_attn_launch_count(): kernels this library has launched since it was
 * loaded (counted whether or not profiling is enabled). Host-thread-safe. */
void flint_attn_profile_enable(int enable);
int flint_attn_profile_collect(int max_kernels, const char** names, double* total_ms,
                               long long* launches);
void flint_attn_profile_reset(void);
long long flint_attn_launch_count(void);

/* Diagnostic: y[i] = the kernels' FMA-pipe evaluation of 2^x[i] (range
 * reduction + degree-3 minimax polynomial; relative error <= 7.5e-5 for
 * x >= -125, inputs below -125 are clamped to it). x, y: device fp32 [n],
 * n even. Asynchronous on `stream`. */
flint_status_t flint_attn_exp2_poly(const float* x, float* y, int32_t n, void* stream);

/* Self-test of failure detection, without a GPU fault. One warp waits, through
 * the same bounded mbarrier wait that every pipelined kernel uses, on a
 * shared-memory barrier that completes only if arrive_first != 0, and gives
 * up after wait_cycles SM clock cycles (1 <= wait_cycles <= 4e9, the kernels'
 * own limit). status: caller-owned device int32[64], 256-byte aligned, with
 * status[0] = 0 on entry (the layout of a workspace's status word). A wait
 * that runs out sets a timeout bit in status[0], so a following
 * flint_attn_check_status(status, stream) returns FLINT_ERR_TIMEOUT (and
 * clears the word); status[1] = 1 if the wait completed, 0 if it gave up. The
 * kernel exits normally either way and the CUDA context stays usable.
 * Asynchronous on `stream`. FLINT_ERR_INVALID_ARG for a null or misaligned
 * status pointer or a limit out of range (before any launch); FLINT_ERR_CUDA
 * if the launch fails. */
flint_status_t flint_attn_selftest_wait(int64_t wait_cycles, int32_t arrive_first,
                                        int32_t* status, void* stream);

/* Static description of a status code. */
const char* flint_status_string(flint_status_t status);

/* Library version string, e.g. "flint_attn 0.1 sm_100a". */
const char* flint_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLINT_ATTN_H */
