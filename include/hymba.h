/*
 * hymba.h - C ABI of libhymba.so, the B200 (sm_100a) implementation of the Hymba
 * hybrid-head mixer forward pass (prefill and decode) and its cross-layer KV sharing.
 *
 * The method (cited by page title and section; [JJ] and [MC] below):
 *   [JJ] juejin.cn post "NVIDIA提出Hymba网络，Mamba+Attenation解决transformer的长序列低效难题"
 *     §数学表示 1   meta tokens R prepended: X~ = [R, X]
 *     §数学表示 2   one input projection W_in = [W_Q, W_K, W_V, W_SSM, W_G]
 *     §数学表示 3   attention heads, eq. (1): softmax(Q K^T) V
 *     §数学表示 4   SSM heads, eq. (2): alpha_ij = C_i prod exp(A Delta_k) B_j Delta_j,
 *                   gated by G
 *     §数学表示 5   per-branch normalisation, beta1/beta2 rescale, average, W_out
 *     §Hymba 的整体架构  global attention in the first/middle/last blocks, sliding-window
 *                   attention elsewhere, adjacent SWA blocks share one KV cache
 *   [MC] model card "Hymba-1.5B-Base" §模型架构: GQA, RoPE, 16 SSM states, meta tokens visible
 *     to every later token even under sliding-window attention.
 * Readings where the pages are silent (1/sqrt(D) scale and causal mask; window = the last
 * `window` positions including the query; half-split RoPE; Euler discretisation
 * exp(Delta A), Delta B; no D skip term; SiLU gate; RMSNorm; W_out over the concatenation
 * of both normalised branches times 1/2) are the ones the fp64 oracle states.
 *
 * Conventions for every entry point
 *   - Returns HYMBA_OK (0) or an HYMBA_ERR_* code; hymba_last_error() gives a message
 *     (thread-local, valid until the next call from the same thread).
 *   - The library never allocates device memory.  The caller passes device pointers it
 *     owns (inputs, outputs, weights, caches, workspace); the library keeps no pointer after
 *     a call returns.
 *   - Work is enqueued on `stream` (a cudaStream_t) and is asynchronous; no entry point
 *     synchronises except hymba_status_read.  Calls may be captured in a CUDA graph.
 *   - bf16 tensors are raw bfloat16 bits (uint16_t), row-major, contiguous unless a
 *     leading dimension is given.  fp32 tensors are float, row-major.
 *   - Device pointers must be 16-byte aligned; the workspace must be 256-byte aligned.
 *   - Errors found on the device (a bounded wait that timed out) are OR'ed into a status
 *     word at the start of the workspace and read with hymba_status_read.
 */
#ifndef HYMBA_H
#define HYMBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  HYMBA_OK = 0,
  HYMBA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
  HYMBA_ERR_UNSUPPORTED = 2,  /* shape outside what the kernels implement, or not sm_100 */
  HYMBA_ERR_WORKSPACE = 3,    /* workspace smaller than hymba_mixer_workspace_size */
  HYMBA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (message has details) */
  HYMBA_ERR_TIMEOUT = 5,      /* status word: a device-side bounded wait gave up */
  HYMBA_ERR_FP16_RANGE = 6,   /* status word: a value stored in fp16 (queries, keys, values, the
                                 KV cache, FFN activations) had |v| >= 65520 and became +-inf */
};

enum { HYMBA_KV_OWN = 0, HYMBA_KV_PRODUCER = 1, HYMBA_KV_CONSUMER = 2 };
enum { HYMBA_CACHE_SWA = 0, HYMBA_CACHE_GLOBAL = 1 };
enum { HYMBA_MODE_PREFILL = 0, HYMBA_MODE_DECODE = 1, HYMBA_MODE_PREFILL_HOST = 2 };

typedef uint16_t hymba_bf16;
typedef uint16_t hymba_f16;   /* IEEE half bits */
typedef struct CUstream_st* hymba_stream; /* identical to cudaStream_t; NULL = legacy stream */

/* One mixer layer's sizes ([MC] §模型架构, [JJ] §数学表示).
 * Supported: head_dim 64, d_state 16, d_conv 4, d_model % 8 == 0, d_inner % 64 == 0 and
 * d_inner <= 4096, n_q_heads * head_dim <= 2048, n_q_heads % n_kv_heads == 0 with at most 6
 * query heads per KV head, dt_rank % 4 == 0 and dt_rank + 2*d_state <= 256, window >= 1,
 * n_meta >= 0.  Anything else is refused with HYMBA_ERR_UNSUPPORTED / HYMBA_ERR_INVALID_ARG
 * before a kernel is launched. */
typedef struct hymba_layer_cfg {
  int d_model;     /* d */
  int n_q_heads;   /* Hq */
  int n_kv_heads;  /* Hkv (GQA: query head h reads KV head h*Hkv/Hq) */
  int head_dim;    /* D */
  int d_inner;     /* Di, SSM channels */
  int d_state;     /* S */
  int d_conv;      /* causal conv width */
  int dt_rank;     /* R */
  int window;      /* W: a query sees the last W positions (itself included) plus the meta tokens */
  int n_meta;      /* M meta tokens */
  int is_global;   /* 1: full causal attention; 0: sliding window + meta */
  int kv_role;     /* HYMBA_KV_OWN / PRODUCER (writes the shared cache) / CONSUMER (reads it) */
  float rope_base; /* RoPE base (theta_j = base^(-2j/D)) */
  float norm_eps;  /* RMSNorm epsilon */
} hymba_layer_cfg;

/* One layer's weights, all device pointers.
 *   meta    [M, d]            bf16  meta tokens R
 *   w_in    [P, d]            bf16  rows [Q (Hq*D) | K (Hkv*D) | V (Hkv*D) | x (Di) | z (Di)];
 *                                   a consumer layer has no K and V rows (P = Hq*D + 2*Di)
 *   conv_w  [Di, 4]           fp32  causal conv taps, tap 3 multiplies the current input
 *   conv_b  [Di]              fp32
 *   w_x     [R + 2S, Di]      bf16  rows [dt_low (R) | B (S) | C (S)]
 *   w_dt    [Di, w_dt_ld]     fp32  first R columns used; w_dt_ld >= R, w_dt_ld % 4 == 0
 *   dt_bias [Di]              fp32  Delta = softplus(dt_low W_dt^T + dt_bias)
 *   A       [Di, S]           fp32  (negative) state matrix
 *   g_attn  [Hq*D]            fp32  beta1
 *   g_ssm   [Di]              fp32  beta2
 *   w_out   [d, Hq*D + Di]    fp16  output projection.  It multiplies the normalised,
 *                                   rescaled branch outputs, which the library keeps in fp16:
 *                                   after RMSNorm every value is at most sqrt(width)*|beta|/2
 *                                   in magnitude, so fp16 cannot overflow and rounds 8x finer
 *                                   than bf16.  bf16 weights convert to fp16 exactly when
 *                                   6.1e-5 <= |w| <= 65504. */
typedef struct hymba_layer_weights {
  const hymba_bf16* meta;
  const hymba_bf16* w_in;
  const float* conv_w;
  const float* conv_b;
  const hymba_bf16* w_x;
  const float* w_dt;
  int w_dt_ld;
  const float* dt_bias;
  const float* A;
  const float* g_attn;
  const float* g_ssm;
  const hymba_f16* w_out;
} hymba_layer_weights;

/* A KV cache, shared by a producer/consumer pair of adjacent SWA layers or owned by one
 * layer ([JJ] §Hymba 的整体架构).  All device pointers, fp16, K stored after RoPE.  The
 * attention operands are fp16: keys, values and probabilities of a normalised-input layer
 * sit far inside fp16's range, where it rounds 8x finer than bf16.
 *   kind HYMBA_CACHE_SWA:
 *     meta_k, meta_v  [B, M, Hkv, D]   keys/values of the meta tokens
 *     ring_k, ring_v  [B, W, Hkv, D]   input position p (>= M) lives in slot (p - M) mod W
 *     k, v            [B, max_tokens, Hkv, D]  prefill view: the producer's prefill writes
 *                     every position here, the consumer's prefill reads it (may be shared
 *                     between caches when layers run in order)
 *   kind HYMBA_CACHE_GLOBAL:
 *     k, v            [B, max_tokens, Hkv, D]  position p at row p (prefill and decode)
 */
typedef struct hymba_kv_cache {
  int kind;
  int batch;
  int n_kv_heads;
  int head_dim;
  int n_meta;
  int window;
  int max_tokens;
  hymba_f16* meta_k;
  hymba_f16* meta_v;
  hymba_f16* ring_k;
  hymba_f16* ring_v;
  hymba_f16* k;
  hymba_f16* v;
} hymba_kv_cache;

/* Library version (major*10000 + minor*100 + patch). */
int hymba_version(void);

/* Message of the last error raised on this thread ("" if none). */
const char* hymba_last_error(void);

/* Bytes of workspace one prefill (mode HYMBA_MODE_PREFILL, n_tokens rows per sequence), one
 * prefill from host buffers (HYMBA_MODE_PREFILL_HOST: the prefill's workspace plus device
 * copies of the input and the output) or one decode step (HYMBA_MODE_DECODE; for a global
 * layer n_tokens is the cache's max_tokens, otherwise ignored) needs.  x_has_meta: see
 * prefill. */
int hymba_mixer_workspace_size(const hymba_layer_cfg* cfg, int batch, int n_tokens, int x_has_meta, int mode,
                               size_t* bytes);

/* Zero the status word of a workspace (call once after allocating it). */
int hymba_workspace_init(void* workspace, size_t ws_bytes, hymba_stream stream);

/* Synchronise `stream`, copy the workspace status word to *status and clear it.  *status is
 * 0, or HYMBA_ERR_TIMEOUT when a device-side wait gave up, else HYMBA_ERR_FP16_RANGE when a
 * value outside fp16's range was stored (the outputs of that call are then not finite; the
 * layer's inputs must be normalised, as the block's RMSNorm does), else HYMBA_ERR_INVALID_ARG
 * when a device-side index check skipped an access. */
int hymba_status_read(void* workspace, hymba_stream stream, int* status);

/* Plan and carve the KV caches of an n_layers stack ([JJ] §Hymba 的整体架构: adjacent SWA
 * blocks share one cache; global blocks keep their own).  Layers are walked in order; an
 * SWA layer followed by an SWA layer opens a pair (producer, consumer); an SWA layer whose
 * successor is global or absent keeps its own cache.
 *   base        sizes (n_kv_heads, head_dim, n_meta, window) shared by all layers
 *   is_global   [n_layers] host array, 1 = full attention
 *   batch, max_tokens   sequences and maximum positions (meta included) per sequence
 *   dev_buf     device buffer to carve, or NULL to only compute *bytes_needed and the plan
 *   layer_cache_id, layer_kv_role   [n_layers] host outputs
 *   caches      [max_caches] host outputs (filled when dev_buf != NULL), *n_caches = count
 * All SWA caches share one prefill view (k, v).  No kernel runs; nothing is zeroed. */
int hymba_kv_share_alloc(const hymba_layer_cfg* base, int n_layers, const uint8_t* is_global, int batch,
                         int max_tokens, void* dev_buf, size_t buf_bytes, size_t* bytes_needed,
                         int* layer_cache_id, int* layer_kv_role, hymba_kv_cache* caches, int max_caches,
                         int* n_caches);

/* Prefill of one mixer layer over `batch` sequences ([JJ] §数学表示 1-6).
 *   x          x_has_meta == 0: [B, n_tokens, d] input tokens; the meta tokens are prepended
 *              (T = M + n_tokens).  x_has_meta == 1: [B, n_tokens, d] rows that already
 *              start with the meta positions (T = n_tokens), as inside a stack.
 *   kv         own/producer: K (after RoPE) and V of every position are written to kv->k/v
 *              (max_tokens >= T) and, for an SWA cache, the meta rows and the last W
 *              positions to meta_k/v and ring_k/v.  consumer: reads kv->k/v.
 *   ssm_state_out  [B, Di, S] fp32 final SSM state, or NULL
 *   conv_state_out [B, Di, 3] fp32 last three conv inputs, or NULL
 *   residual   [B, T, d] bf16 added to the output, or NULL
 *   out        [B, T, d] bf16 (all rows, meta rows included)
 * Errors: INVALID_ARG (null/misaligned pointer, batch or n_tokens < 1, max_tokens < T),
 * UNSUPPORTED (shape, device), WORKSPACE (too small), CUDA. */
int hymba_mixer_prefill(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x,
                        int x_has_meta, int batch, int n_tokens, hymba_kv_cache* kv, float* ssm_state_out,
                        float* conv_state_out, const hymba_bf16* residual, hymba_bf16* out, void* workspace,
                        size_t ws_bytes, hymba_stream stream);

/* A layer's meta-token prefix, computed once ([JJ] §深入理解元 Tokens: the meta tokens are
 * fixed at inference, so what they produce can be computed offline).  The meta rows never
 * see the input rows (they come first and attention is causal), so these are the same for
 * every input: the keys (after RoPE) and values of the M meta positions, and the SSM and
 * conv states after the M meta rows.  A consumer layer's k/v are its producer's. */
typedef struct hymba_meta_prefix {
  hymba_f16* k;        /* [M, Hkv, D] fp16 */
  hymba_f16* v;        /* [M, Hkv, D] fp16 */
  float* ssm_state;    /* [Di, S] fp32 */
  float* conv_state;   /* [Di, 3] fp32: the last three conv inputs of the meta rows */
} hymba_meta_prefix;

/* Bytes of device memory one layer's prefix occupies (k, v, ssm_state, conv_state). */
int hymba_meta_prefix_size(const hymba_layer_cfg* cfg, size_t* bytes);

/* Compute a layer's prefix: one prefill of its M meta rows alone.
 *   meta_rows  [M, d] bf16: the meta rows of this layer's input (the meta tokens R for a
 *              single layer; the residual stream's meta rows, normalised, inside a stack)
 *   buf        device buffer of hymba_meta_prefix_size bytes, 256-byte aligned; *prefix
 *              receives pointers into it
 *   producer   for a consumer layer (kv_role 2), its producer's prefix: the meta keys and
 *              values it reads (and that *prefix then points to); NULL otherwise
 *   meta_out   [M, d] bf16: the layer's output rows for the meta positions
 *   workspace  as hymba_mixer_prefill for batch 1, n_tokens = M, x_has_meta = 1.
 * Errors as hymba_mixer_prefill; INVALID_ARG when n_meta == 0. */
int hymba_meta_prefix_build(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* meta_rows,
                            void* buf, size_t buf_bytes, const hymba_meta_prefix* producer,
                            hymba_meta_prefix* prefix, hymba_bf16* meta_out, void* workspace, size_t ws_bytes,
                            hymba_stream stream);

/* hymba_mixer_prefill from a precomputed prefix: x [B, n_tokens, d] holds only the input
 * rows (positions M .. M + n_tokens - 1), and only those rows are computed.  The prefix's
 * meta K/V are copied into the cache (the prefill view's rows 0..M-1 and, for an SWA cache,
 * its meta rows; a consumer reads its producer's), the conv and the scan start from the
 * prefix's states.  residual and out are [B, n_tokens, d].  ssm_state_out / conv_state_out
 * as hymba_mixer_prefill.  Workspace: hymba_mixer_workspace_size (mode PREFILL, the same
 * n_tokens, x_has_meta 0) suffices.  Errors as hymba_mixer_prefill. */
int hymba_mixer_prefill_prefix(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x,
                               int batch, int n_tokens, const hymba_meta_prefix* prefix, hymba_kv_cache* kv,
                               float* ssm_state_out, float* conv_state_out, const hymba_bf16* residual,
                               hymba_bf16* out, void* workspace, size_t ws_bytes, hymba_stream stream);

/* hymba_mixer_prefill with the input and the output in HOST memory: x_host [B, n_tokens, d]
 * and out_host [B, T, d] bf16 (page-locked memory lets the copies run asynchronously and
 * overlap other streams' work; pageable memory works but the copies then block the host).
 * Enqueued on `stream`: the copy of x_host into the workspace, the prefill, the copy of the
 * output to out_host.  The workspace (mode HYMBA_MODE_PREFILL_HOST) holds the device copies.
 * Weights, the KV cache and the states stay in device memory.  No residual.  Errors as
 * hymba_mixer_prefill. */
int hymba_mixer_prefill_host(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x_host,
                             int x_has_meta, int batch, int n_tokens, hymba_kv_cache* kv, float* ssm_state_out,
                             float* conv_state_out, hymba_bf16* out_host, void* workspace, size_t ws_bytes,
                             hymba_stream stream);

/* One decode step for `batch` sequences that all sit at position `position` (= M + number
 * of tokens already in the context; the pages' released model generates with equal-length
 * sequences).  x [B, d] bf16.  own/producer: the new K (after RoPE) and V go to ring slot
 * (position - M) mod W (SWA) or row `position` (global) before attending; consumer: the
 * producer's step must already have run.  ssm_state [B, Di, S] and conv_state [B, Di, 3]
 * fp32 are read and updated in place.  residual [B, d] or NULL; out [B, d] bf16.
 * Errors as prefill; INVALID_ARG also when position < M or (global) position >= max_tokens. */
int hymba_mixer_decode(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x, int batch,
                       int position, hymba_kv_cache* kv, float* ssm_state, float* conv_state,
                       const hymba_bf16* residual, hymba_bf16* out, void* workspace, size_t ws_bytes,
                       hymba_stream stream);

/* The decode step for a batch whose sequences sit at different positions: sequence b's new
 * token is at positions[b] (device memory, int32 [batch]), with n_meta <= positions[b] <=
 * max_position (and, for a global layer, < kv->max_tokens).  Everything else as
 * hymba_mixer_decode: each sequence's RoPE angle, ring slot (positions[b] - M) mod W (or
 * global row positions[b]) and attended keys (the meta tokens plus its own filled window,
 * or its rows 0..positions[b]) are its own.  This goes beyond the released model, which the
 * jxzklqfsx.com news article (§4) notes cannot generate for padded batches with meta tokens
 * and SWA.  max_position (host) sizes the attention's key splits.  A position outside those
 * bounds is recorded in the status word (HYMBA_ERR_INVALID_ARG from hymba_status_read) and
 * that sequence's cache is left unwritten; its outputs are then undefined. */
int hymba_mixer_decode_ragged(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x,
                              int batch, const int* positions, int max_position, hymba_kv_cache* kv,
                              float* ssm_state, float* conv_state, const hymba_bf16* residual, hymba_bf16* out,
                              void* workspace, size_t ws_bytes, hymba_stream stream);

/* Byte offsets, inside a prefill workspace, of the stage buffers of the last prefill (for
 * stage-by-stage checks).  Layouts (rows r = b*T + t):
 *   q      [B*T, Hq*D]  fp16  queries after RoPE
 *   xz     [B*T, 2*Di]  bf16  in_proj x | z columns
 *   xc     [B*T, Di]    bf16  SiLU(conv(x))
 *   xbc    [B*T, ld_xbc] fp32 x_proj output: dt_low | B | C
 *   dt_pre [B*T, Di]    bf16  dt_low W_dt^T (the scan applies softplus(. + dt_bias) in fp32)
 *   y      [B*T, Di]    bf16  scan output before the gate
 *   o      [B*T, Hq*D]  fp32  attention output
 *   u      [B*T, Hq*D+Di] fp16 normalised, rescaled, averaged branches (out_proj input)
 * scan_chunks / scan_chunk_len: the time chunks the selective scan is cut into (the last
 * chunk may be shorter). */
typedef struct hymba_stage_layout {
  size_t q, xz, xc, xbc, dt_pre, y, o, u;
  int ld_xbc;
  int scan_chunks, scan_chunk_len;
} hymba_stage_layout;
int hymba_mixer_stage_layout(const hymba_layer_cfg* cfg, int batch, int n_tokens, int x_has_meta,
                             hymba_stage_layout* out);

/* Byte offsets, inside a decode workspace, of the stage buffers of the last decode step (for
 * stage-by-stage checks).  max_tokens: the cache's max_tokens (it sizes a global layer's
 * attention splits).  Layouts (B sequences, P = in_proj width):
 *   proj      in_split slices of [B, P] fp32, slice stride proj_slice_stride elements: the
 *             in_proj output [q | k | v | x | z] is the sum of the slices in slice order
 *   xc        [B, Di]  bf16  SiLU(conv) of the new token
 *   xbc_part  xproj_split slices of [B, ld_xbc] fp32, slice stride xbc_slice_stride
 *             elements: x_proj's [dt_low | B | C] is the sum of the slices in slice order
 *   y         [B, Di]  fp32  gated SSM output */
typedef struct hymba_decode_stages {
  size_t proj, xc, xbc_part, y;
  long long proj_slice_stride, xbc_slice_stride;
  int in_split, xproj_split, ld_proj, ld_xbc;
} hymba_decode_stages;
int hymba_decode_stage_layout(const hymba_layer_cfg* cfg, int batch, int max_tokens, hymba_decode_stages* out);

/* C[M, N] = A[M, K] * B[N, K]^T (+ residual[M, N]) on the tcgen05 GEMM, bf16 in/out, fp32
 * accumulation.  K % 8 == 0, N % 8 == 0.  status_ws: a workspace (>= 256 bytes) whose
 * status word receives device-side errors. */
int hymba_gemm_bf16(const hymba_bf16* A, const hymba_bf16* B, const hymba_bf16* residual, hymba_bf16* C, int M,
                    int N, int K, void* status_ws, hymba_stream stream);

/* Stack harness pieces (one Hymba block = x + mixer(norm(x)), then + FFN(norm(.))):
 * out[r, :] = x[r, :] / sqrt(mean(x[r, :]^2) + eps) * gain, rows x d bf16. */
int hymba_rmsnorm(const hymba_bf16* x, const float* gain, int rows, int d, float eps, hymba_bf16* out,
                  hymba_stream stream);

/* SwiGLU FFN with residual: out = residual + W_down (SiLU(W_gate h) * (W_up h)).
 *   h [rows, d] bf16; w_gate_up [2F, d] bf16 with gate and up rows interleaved in blocks of
 *   32 (rows 64i..64i+31 = gate rows 32i.., rows 64i+32..64i+63 = up rows 32i..);
 *   w_down [d, F] fp16; act [rows, F] fp16 scratch (the activations feed the down
 *   projection in fp16, 8x finer than bf16 for these O(1) values); residual [rows, d] bf16 or
 *   NULL; out [rows, d] bf16; F % 64 == 0, d % 8 == 0. */
int hymba_ffn_swiglu(const hymba_bf16* h, const hymba_bf16* w_gate_up, const hymba_f16* w_down, int rows, int d,
                     int F, hymba_f16* act, const hymba_bf16* residual, hymba_bf16* out, void* status_ws,
                     hymba_stream stream);

/* The same FFN for a few rows (a decode step: rows = sequences, 1..256): the weights are the M
 * operand of the tensor-core GEMMs, so that their rows spread the weight streaming over the
 * SMs, and K is split into fp32 slices summed in a fixed order.  The same function as
 * hymba_ffn_swiglu; gate and up are kept in fp32 until the activation (fp16).  The workspace
 * (hymba_ffn_workspace_size) holds the slices, the activations and the status word. */
int hymba_ffn_workspace_size(int rows, int d, int F, size_t* bytes);
int hymba_ffn_swiglu_decode(const hymba_bf16* h, const hymba_bf16* w_gate_up, const hymba_f16* w_down, int rows,
                            int d, int F, const hymba_bf16* residual, hymba_bf16* out, void* workspace,
                            size_t ws_bytes, hymba_stream stream);

/* The decode steps of a block's two sublayers with the next sublayer's input norm fused into
 * their last kernel ([JJ] §Hymba 的整体架构: x + mixer(norm(x)), then + FFN(norm(.))): as
 * hymba_mixer_decode and hymba_ffn_swiglu_decode, and in the same final pass over each row
 *   norm_out[r, :] = out[r, :] / sqrt(mean(out[r, :]^2) + norm_eps) * norm_gain
 * (out as stored, bf16; norm_gain [d] fp32, 16-byte aligned; norm_out [rows, d] bf16, not
 * aliasing out or the input), which is what hymba_rmsnorm computes from out.  out itself is
 * bit for bit what the plain call writes.  d_model <= 4096.
 * Errors: as the plain calls; HYMBA_ERR_INVALID_ARG for a NULL, misaligned or aliasing norm
 * argument, HYMBA_ERR_UNSUPPORTED for d_model above 4096. */
int hymba_mixer_decode_norm(const hymba_layer_cfg* cfg, const hymba_layer_weights* weights, const hymba_bf16* x,
                            int batch, int position, hymba_kv_cache* kv, float* ssm_state, float* conv_state,
                            const hymba_bf16* residual, hymba_bf16* out, const float* norm_gain, float norm_eps,
                            hymba_bf16* norm_out, void* workspace, size_t ws_bytes, hymba_stream stream);
int hymba_ffn_swiglu_decode_norm(const hymba_bf16* h, const hymba_bf16* w_gate_up, const hymba_f16* w_down, int rows,
                                 int d, int F, const hymba_bf16* residual, hymba_bf16* out, const float* norm_gain,
                                 float norm_eps, hymba_bf16* norm_out, void* workspace, size_t ws_bytes,
                                 hymba_stream stream);

/* L2 prefetch hint for read-only device ranges that a later kernel on another stream (or
 * later on this one) will stream, e.g. the weights of a decode step's projections while the
 * latency-bound attention and scan kernels before them run.  ranges[i] / bytes[i]: up to 8
 * device pointers (16-byte aligned) and sizes, both arrays on the host; the call only enqueues
 * one kernel that issues bulk L2 prefetches of 32 KB pieces and returns without waiting for
 * them.  No result is defined and no memory is written: a hint the hardware may drop.
 * Errors: HYMBA_ERR_INVALID_ARG for n_ranges outside 1..8, a null or misaligned pointer. */
int hymba_l2_prefetch(const void* const* ranges, const size_t* bytes, int n_ranges, hymba_stream stream);

/* Meta-token prefix of a stack's residual stream ([JJ] §数学表示 1: X~ = [R, X]):
 * out[b] = [meta; x[b]], meta [n_meta, d], x [B, n_tokens, d], out [B, n_meta + n_tokens, d],
 * all bf16, d % 8 == 0. */
int hymba_prepend_meta(const hymba_bf16* meta, const hymba_bf16* x, int batch, int n_meta, int n_tokens, int d,
                       hymba_bf16* out, hymba_stream stream);

/* Upper bound, in nanoseconds, of every device-side wait on an mbarrier (default 2e9).
 * A wait that runs out records HYMBA_ERR_TIMEOUT in the status word and the kernel returns. */
int hymba_set_wait_limit_ns(unsigned long long ns);

/* Launch a kernel whose only wait is on a barrier nothing ever arrives at, so that the
 * bounded wait runs out; the status word of `workspace` then reads HYMBA_ERR_TIMEOUT.
 * Exercises the timeout path without faulting or hanging the device. */
int hymba_selftest_wait_timeout(void* workspace, size_t ws_bytes, hymba_stream stream);

/* hymba_mixer_decode without a workspace argument, for callers that cannot allocate device
 * memory where they run a decode step (a serving loop that must not take cudaMalloc's
 * device synchronisation between tokens, or a plugin whose host runtime owns all device
 * memory and hands it only inputs and outputs).  The pages have no counterpart: this is a deployment
 * convenience of this library.  Arguments and results are those of hymba_mixer_decode.
 *   - Scratch: a built-in 32 MiB device array (every GPU that loads the library holds it
 *     until exit).  A step that needs more (hymba_mixer_workspace_size, mode DECODE, with
 *     n_tokens = kv->max_tokens) is rejected with HYMBA_ERR_WORKSPACE; Hymba-1.5B-sized SWA
 *     layers fit up to batch 64.
 *   - The first call on each device looks up the array's device address; make that first
 *     call before any stream capture.
 *   - Every call on a device uses the same array: calls that can overlap on the GPU (for
 *     example on two streams of one device) race on it; the caller must serialise them.
 *   - The status word at the start of the array is cleared at every call and cannot be
 *     read, so device-side errors of this variant (a bounded wait that runs out, an fp16
 *     overflow) are not reported.  After such an error the step's outputs, states and new
 *     cache slot are undefined, with no sign of it; a caller that must detect errors uses
 *     hymba_mixer_decode and reads its workspace's status word.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
int hymba_mixer_decode_noalloc(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x,
                               int batch, int position, hymba_kv_cache* kv, float* ssm_state, float* conv_state,
                               const hymba_bf16* residual, hymba_bf16* out, hymba_stream stream);

/* Kernel-level timing: while enabled, every kernel the library launches is bracketed by a
 * pair of CUDA events on its stream (the events are created on the host by the first
 * hymba_profile_begin; no device memory is allocated).  hymba_profile_end synchronises on
 * the recorded events and returns, in launch order, each kernel's name and elapsed time.
 * At most max_records launches are recorded; not thread-safe.
 * hymba_profile_read stops recording and returns the same records without clearing them:
 * after the launches were captured into a CUDA graph, every replay re-records the events,
 * and a read after each replay gives that replay's kernel times without host launch gaps.
 * hymba_profile_end then clears the records. */
typedef struct hymba_prof_record {
  char name[24];
  float ms;
} hymba_prof_record;
int hymba_profile_begin(int max_records);
int hymba_profile_read(hymba_prof_record* out, int max_records, int* n_records);
int hymba_profile_end(hymba_prof_record* out, int max_records, int* n_records);

#ifdef __cplusplus
}
#endif
#endif /* HYMBA_H */
