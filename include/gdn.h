/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated delta-rule linear-attention layer
 * ("Gated DeltaNet", the linear-attention layer of Qwen3-Next).
 *
 * Per value head, with an fp32 state S in R^{d_k x d_v} (row-major, d_v contiguous), each
 * token t does
 *     S <- exp(g_t) S ;  S <- S + beta_t k_t (v_t - S^T k_t)^T ;  o_t = S^T q_t
 * (llama.cpp compare b7429..b7432, "Optimization: Qwen3 next autoregressive pass",
 *  src/models/qwen3next.cpp, build_delta_net_autoregressive). Longer inputs use the
 * equivalent chunked WY/UT form (same page, build_delta_net_chunking; chunk 64 as
 * QWEN3NEXT_CHUNK_SIZE in ik_llama.cpp src/llama-delta-net.cpp).
 *
 * Conventions shared by every entry point
 *  - All array pointers are DEVICE pointers owned by the caller; the library allocates
 *    nothing and keeps no pointer after a call returns (except the decode pipeline below,
 *    which takes host buffers and holds its arrays between calls).
 *  - Every call only enqueues work on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns without synchronising, except gdn_device_status.
 *  - Arrays are dense and row-major in the shapes given; every array pointer must be
 *    16-byte aligned (GDN_EALIGN otherwise).
 *  - Argument errors found on the host return a negative status and launch nothing.
 *    Errors that need device data (a slot id out of range or repeated, inconsistent
 *    cu_seqlens) are found by the kernels: the offending sequence is skipped and the
 *    first such error is recorded in a per-device status word read by gdn_device_status.
 *    A slot id repeated within one call is kept by its first sequence, which is processed
 *    normally; every later sequence with that slot is skipped entirely (its pool rows are
 *    not touched, its outputs are not written) and GDN_ESLOT is recorded.
 *  - GQA is grouped by default: value head h reads key head h / (H_v / H_k)
 *    (ik_llama.cpp src/llama-delta-net.cpp, build_layer_attn_linear_core, the repeat on
 *    the fused ssm_beta_alpha path); gdn_dims.layout selects the tiled mapping and the
 *    fused beta/alpha gate input of the other weight family.
 *  - Sequences are packed into one token stream with cu_seqlens[n_seqs+1] (int32,
 *    cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seqs] = T_total). Sequence n owns
 *    state pool row slot_ids[n]; slot ids within one call must be distinct. reset[n] != 0
 *    (or reset == NULL meaning all zero) starts sequence n from a zero recurrent state and
 *    a zero conv state, the counterpart of the pages' state reset at position 0
 *    (ik_llama.cpp, build_layer_attn_linear_core / build_layer_attn_linear).
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* gdn_stream_t;

/* Status codes. */
enum {
  GDN_OK = 0,
  GDN_EINVAL = -1,       /* bad shape, count, dtype or null pointer */
  GDN_ESLOT = -2,        /* slot id out of range or repeated within one call (device) */
  GDN_EALIGN = -3,       /* an array pointer is not 16-byte aligned */
  GDN_ECUDA = -4,        /* a CUDA launch or runtime call failed */
  GDN_ETIMEOUT = -5,     /* a bounded device-side wait gave up (device) */
  GDN_EWORKSPACE = -6,   /* workspace missing or smaller than gdn_prefill_workspace_size */
  GDN_EUNSUPPORTED = -7  /* valid but unsupported combination (e.g. head dim) */
};

/* Element types. */
enum { GDN_F32 = 0, GDN_BF16 = 1, GDN_F16 = 2 };

/* Layouts of the two families of Qwen3-Next GGUF weights (ik_llama.cpp
 * src/llama-delta-net.cpp, build_layer_attn_linear_core), combinable bit flags:
 *  - GDN_GQA_TILED: value head h reads key head h % H_k (the ggml_repeat_4d of q and k on
 *    the path with separate ssm_alpha / ssm_beta weights). Default: grouped, h / (H_v/H_k)
 *    (the repeat on the fused ssm_beta_alpha path).
 *  - GDN_GATES_MIXED_BA: the gate inputs come as the fused ssm_beta_alpha projection, one
 *    array [T][H_k][2 r] (r = H_v / H_k) holding per key head first the r beta logits, then
 *    the r alpha values, of the value heads h = hk r + j, j < r; it is passed as `a`, and `b`
 *    must be NULL. Default: separate a (alpha) and b (beta logits), each [T][H_v]. */
enum { GDN_LAYOUT_DEFAULT = 0, GDN_GQA_TILED = 1 << 0, GDN_GATES_MIXED_BA = 1 << 1 };

/* Layer shape. Supported: d_k, d_v in {32, 64, 128}; H_v a multiple of H_k;
 * d_conv in 0..4 (0 = no conv stage). conv_dim = 2*H_k*d_k + H_v*d_v. */
typedef struct gdn_dims {
  int32_t n_slots; /* rows of the recurrent-state and conv-state pools */
  int32_t H_k;     /* key heads (ssm_n_group) */
  int32_t H_v;     /* value heads (ssm_dt_rank) */
  int32_t d_k;     /* key head dim (ssm_d_state) */
  int32_t d_v;     /* value head dim (ssm_d_inner / H_v) */
  int32_t d_conv;  /* conv taps (ssm_d_conv, 4 in Qwen3-Next) */
  int32_t layout;  /* GDN_LAYOUT_DEFAULT or GDN_GQA_TILED | GDN_GATES_MIXED_BA */
} gdn_dims;

/* Prefill flags. */
enum {
  GDN_PREFILL_DEFAULT = 0,
  GDN_PREFILL_SIMT = 1u << 0, /* force the fp32 SIMT chunked kernel */
  /* bit 1 is reserved (rejected with GDN_EINVAL) */
  /* gdn_chunked_prefill: every sequence through the token-by-token kernel (the state held in
   * registers across a sequence's tokens, fp32 arithmetic), whatever its length; no
   * workspace needed. gdn_layer_prefill: the caller promises that every sequence has at most
   * 16 tokens (a multi-token step): only the short-sequence path runs, the record and scan
   * kernels are not launched, and a longer sequence is skipped with GDN_EINVAL recorded; the
   * workspace is then gdn_prefill_workspace_size(..., GDN_PREFILL_RECURRENT) bytes. */
  GDN_PREFILL_RECURRENT = 1u << 2,
  /* for gdn_prefill_workspace_size only: also room for the fp32 output that gdn_layer_prefill
   * gates into o when it is given an output gate (so o is rounded once, after the gate) */
  GDN_PREFILL_OUT_GATE = 1u << 3,
  /* tensor-core path: the state scan with one CTA per (sequence, value head) holding the
   * whole 128 x 128 state. Without this flag or GDN_PREFILL_TC_TILE_SCAN the call chooses:
   * the whole-head scan when the tile scan would need more than two waves of CTAs
   * (4 n_seqs H_v > 2 x the SM count), else the tile scan. */
  GDN_PREFILL_TC_HEAD_SCAN = 1u << 4,
  /* tensor-core path: the state scan with one CTA per (sequence, value head, 32-column tile)
   * (4 per head: more parallel, each chunk step about 2.5 times shorter; the faster choice
   * for a few sequences). Not combinable with GDN_PREFILL_TC_HEAD_SCAN. */
  GDN_PREFILL_TC_TILE_SCAN = 1u << 5
};

/*
 * Output gate of the layer (ik_llama.cpp src/llama-delta-net.cpp,
 * build_layer_attn_linear_core: llm_build_norm(o, ssm_norm, LLM_NORM_RMS), then
 * ggml_fused_mul_unary(z, ., SILU)): for every token t and value head h,
 *   out[t][h][:] = o[t][h][:] / sqrt(mean_j o[t][h][j]^2 + eps) * norm_w[:] * SiLU(z[t][h][:])
 * with the RMS taken over the d_v values of that head and norm_w shared by all heads.
 */
typedef struct gdn_out_gate {
  const void* z;        /* [T][H_v][d_v], same token order as o */
  int32_t z_dtype;      /* GDN_F32 or GDN_BF16 */
  const float* norm_w;  /* [d_v] fp32 */
  float eps;            /* >= 0 (the model's RMS-norm epsilon) */
} gdn_out_gate;

/*
 * gdn_conv_step -- the layer front for a packed batch of sequences.
 * Pages: ik_llama.cpp src/llama-delta-net.cpp, build_layer_attn_linear_core (ggml_ssm_conv
 * over [conv_states; x], SiLU over the whole conv output, q|k|v views, ggml_l2_norm of q
 * and k with eps, conv state write-back) and qwen3next.cpp build_layer_attn_linear
 * (gate = softplus(alpha + ssm_dt) * ssm_a; beta = sigmoid(b); q scaled by 1/sqrt(d)).
 *
 * Per token t of sequence n and channel c, with x_ext = [conv_state rows (oldest first);
 * the sequence's x rows]:
 *   y[c] = sum_j conv_w[c][j] * x_ext[t + j][c]  (tap d_conv-1 is the current token)
 *   u = y * sigmoid(y)                             (SiLU on q, k and v)
 *   q = u_q / sqrt(|u_q|^2 + eps) * q_scale ; k = u_k / sqrt(|u_k|^2 + eps) ; v = u_v
 *   g = -exp(A_log[h]) * softplus(a[t][h] + dt_bias[h]) ; beta = sigmoid(b[t][h])
 * and conv_state[slot] becomes the last d_conv-1 rows of x_ext.
 * With d_conv == 0 the conv and SiLU stages are skipped (u = x); conv_w and conv_state
 * must then be NULL.
 *
 *   x           [T_total][conv_dim], channel order q|k|v, x_dtype F32 or BF16
 *   conv_w      [conv_dim][d_conv] fp32 (NULL iff d_conv == 0)
 *   conv_state  [n_slots][d_conv-1][conv_dim], conv_state_dtype F32 or BF16, updated in
 *               place; NULL iff d_conv <= 1. Rolled bit-exactly (no rounding).
 *   cu_seqlens  [n_seqs+1] int32, or NULL when every sequence holds one token (T_total must
 *               then equal n_seqs; token n belongs to sequence n)
 *   a, b        [T_total][H_v] fp32 (with GDN_GATES_MIXED_BA: a = [T_total][H_k][2 r],
 *               b = NULL);  A_log, dt_bias [H_v] fp32
 *   q, k        [T_total][H_k][d_k];  v [T_total][H_v][d_v]; qkv_dtype F32, F16 or BF16
 *   g, beta     [T_total][H_v] fp32
 * Returns GDN_OK or a negative status; asynchronous on stream.
 */
int gdn_conv_step(const gdn_dims* dims, const void* x, int32_t x_dtype, const float* conv_w,
                  void* conv_state, int32_t conv_state_dtype, const int32_t* cu_seqlens,
                  const int32_t* slot_ids, const uint8_t* reset, int32_t n_seqs,
                  int64_t T_total, const float* a, const float* b, const float* A_log,
                  const float* dt_bias, float eps, float q_scale, void* q, void* k, void* v,
                  int32_t qkv_dtype, float* g, float* beta, gdn_stream_t stream);

/*
 * gdn_decode_step -- one token for each of n_seqs sequences (the autoregressive step).
 * Pages: qwen3next.cpp build_delta_net_autoregressive (n_seq_tokens == 1 dispatch in
 * build_layer_attn_linear).
 * Token n belongs to sequence n and updates state[slot_ids[n]] in place. The state is read
 * once and written once: o = exp(g) S0^T q + delta (k.q), delta = beta (v - exp(g) S0^T k),
 * S = exp(g) S0 + k delta^T, which equals the pages' step exactly in real arithmetic.
 *
 *   q, k   [n_seqs][H_k][d_k];  v [n_seqs][H_v][d_v]; qkv_dtype F32, F16 or BF16
 *          (q already L2-normalised and scaled, k L2-normalised: gdn_conv_step output)
 *   g, beta [n_seqs][H_v] fp32
 *   state  [n_slots][H_v][d_k][d_v] fp32, in place
 *   slot_ids [n_seqs] int32; reset [n_seqs] uint8 or NULL
 *   o      [n_seqs][H_v][d_v], o_dtype F32 or BF16 (round to nearest even)
 */
int gdn_decode_step(const gdn_dims* dims, const void* q, const void* k, const void* v,
                    int32_t qkv_dtype, const float* g, const float* beta, float* state,
                    const int32_t* slot_ids, const uint8_t* reset, int32_t n_seqs, void* o,
                    int32_t o_dtype, gdn_stream_t stream);

/*
 * gdn_layer_decode -- the whole single-token layer step for n_seqs sequences in one call: the
 * front (gdn_conv_step with one token per sequence, fp32 q/k/v) and then the decode step
 * (gdn_decode_step), with bit for bit the results of those two calls. Two ways, chosen by
 * batch size:
 *  - small batches (n_seqs * H_v * d_v / 32 <= 8 x the SM count) at d_k = d_v = 128,
 *    d_conv = 4, H_v = H_k or 2 H_k: ONE kernel, each CTA computing the front values it
 *    needs (a thread-block cluster per key head shares the conv-state roll); the workspace
 *    is then unused;
 *  - otherwise the front kernel and then the decode kernel, which streams the recurrent
 *    state in while the front is still running (programmatic dependent launch;
 *    gdn_decode_step on its own waits for the kernel ahead of it first).
 * Pages: ik_llama.cpp src/llama-delta-net.cpp,
 * build_layer_attn_linear_core (conv, SiLU, L2 norm, conv-state write-back) and
 * qwen3next.cpp build_delta_net_autoregressive (the n_seq_tokens == 1 step).
 *   x [n_seqs][conv_dim] (x_dtype F32 or BF16), conv_w, conv_state, slot_ids, reset, a, b
 *       ([n_seqs][H_v]), A_log, dt_bias, eps, q_scale: as gdn_conv_step
 *   state, o, o_dtype: as gdn_decode_step
 *   workspace / workspace_bytes: device scratch for the fp32 q, k, v, g, beta (and, with a
 *       gate, o) of the step, at least gdn_decode_workspace_size(dims, n_seqs) bytes,
 *       16-byte aligned; its contents are overwritten (GDN_EWORKSPACE if missing or too
 *       small)
 *   gate: NULL, or the output gate (z [n_seqs][H_v][d_v]); o receives the gated output. On
 *       the one-kernel path it is applied inside that kernel (the column tiles of a head
 *       exchange their sums of squares within the cluster); on the two-kernel path the step
 *       writes fp32 o into the workspace and a third kernel gates it into o (o is rounded
 *       once either way).
 */
int gdn_layer_decode(const gdn_dims* dims, const void* x, int32_t x_dtype, const float* conv_w,
                     void* conv_state, int32_t conv_state_dtype, const int32_t* slot_ids,
                     const uint8_t* reset, int32_t n_seqs, const float* a, const float* b,
                     const float* A_log, const float* dt_bias, float eps, float q_scale,
                     float* state, void* o, int32_t o_dtype, void* workspace,
                     size_t workspace_bytes, const gdn_out_gate* gate, gdn_stream_t stream);

/* Workspace bytes gdn_layer_decode needs for n_seqs sequences (0 for invalid arguments). */
size_t gdn_decode_workspace_size(const gdn_dims* dims, int32_t n_seqs);

/* Kernels one gdn_layer_decode call launches for n_seqs sequences on the current device, with
 * (gated != 0) or without an output gate: 1 (the one-kernel path), 2 (front, then decode) or
 * 3 (front, decode, output gate); 0 for invalid arguments. */
int32_t gdn_layer_decode_launches(const gdn_dims* dims, int32_t n_seqs, int32_t gated);

/*
 * gdn_chunked_prefill -- the chunked gated delta rule over packed sequences.
 * Pages: qwen3next.cpp build_delta_net_chunking and the removed single-chunk path whose
 * comments give the per-chunk math: g_cum = cumsum(g); decay mask exp(g_cum_i - g_cum_j)
 * masked before exp; A = -(beta K K^T * decay) strictly lower; T = (I - A)^-1 (the
 * triangular solve); U = T (V*beta); W = T (K*beta*exp(g_cum)); P = (Q K^T * decay) on
 * the lower triangle with the diagonal; v_new = U - W S; o = (Q*exp(g_cum)) S + P v_new;
 * S = exp(g_last) S + (K*exp(g_last - g_cum))^T v_new.
 * Chunks never cross a sequence boundary; a sequence's last partial chunk is handled as
 * if zero-padded (g = 0, beta = 0), which leaves S unchanged. Inside a chunk each token's
 * gate enters the running sums as max(g, -40): such a token keeps at most exp(-40) = 4e-18
 * of the past (far below fp32 rounding), and the sums stay small enough for their
 * differences to stay accurate.
 *
 *   q, k, v, g, beta : as gdn_conv_step output for the T_total packed tokens
 *   state [n_slots][H_v][d_k][d_v] fp32, read at slot_ids[n] (or zero if reset[n]) and
 *         overwritten with the final state of sequence n
 *   chunk 16, 32 or 64
 *   o     [T_total][H_v][d_v], o_dtype F32 or BF16
 *   workspace / workspace_bytes: device scratch of at least gdn_prefill_workspace_size()
 *         bytes (may be NULL when that size is 0); 256-byte aligned.
 *   flags GDN_PREFILL_* ; qkv_dtype F32 selects the fp32 SIMT kernel, F16/BF16 the
 *         tensor-core kernel (unless GDN_PREFILL_SIMT).
 * Mixed batches: on the tensor-core path, sequences of at most 16 tokens (single decode
 * tokens, speculative or multi-token steps) run through a token-by-token kernel that keeps
 * the state in registers (the per-token step of build_delta_net_autoregressive), and longer
 * ones through the chunked kernels, in the same call; each kernel reads cu_seqlens on the
 * device and leaves the other's sequences alone. GDN_PREFILL_RECURRENT sends every sequence
 * through the token-by-token kernel.
 */
int gdn_chunked_prefill(const gdn_dims* dims, const void* q, const void* k, const void* v,
                        int32_t qkv_dtype, const float* g, const float* beta, float* state,
                        const int32_t* slot_ids, const int32_t* cu_seqlens,
                        const uint8_t* reset, int32_t n_seqs, int64_t T_total, int32_t chunk,
                        void* o, int32_t o_dtype, void* workspace, size_t workspace_bytes,
                        uint32_t flags, gdn_stream_t stream);

/* Workspace bytes gdn_chunked_prefill needs for these arguments (0 if none). */
size_t gdn_prefill_workspace_size(const gdn_dims* dims, int64_t T_total, int32_t n_seqs,
                                  int32_t chunk, int32_t qkv_dtype, uint32_t flags);

/*
 * gdn_layer_prefill -- the whole layer core for packed sequences in one call: the front
 * (gdn_conv_step) applied inside the chunked prefill's first kernel, from raw x, then the
 * chunked gated delta rule (gdn_chunked_prefill). No q, k, v, g or beta tensor is written.
 * Pages: ik_llama.cpp src/llama-delta-net.cpp build_layer_attn_linear_core (conv, SiLU,
 * L2 norm, conv-state write-back) and qwen3next.cpp build_delta_net_chunking; the same
 * arithmetic as the two calls, up to the order of the L2-norm sums.
 *   x, conv_w, conv_state, cu_seqlens, slot_ids, reset, a, b, A_log, dt_bias, eps, q_scale:
 *       as gdn_conv_step (the conv state is read, then overwritten with the last d_conv - 1
 *       rows of [old state; x] of each sequence)
 *   state, chunk, o, o_dtype, workspace, workspace_bytes: as gdn_chunked_prefill, the
 *       workspace sized by gdn_prefill_workspace_size(..., GDN_F16, 0)
 *   flags: 0, GDN_PREFILL_TC_HEAD_SCAN or GDN_PREFILL_TC_TILE_SCAN, and GDN_PREFILL_RECURRENT
 *       for a batch of short sequences only (see the flag)
 *   gate: NULL, or the output gate (z [T_total][H_v][d_v]): the prefill then writes its
 *       output in fp32 into the workspace and one more kernel writes the gated result into o
 *       (o is rounded once); the workspace must be sized with GDN_PREFILL_OUT_GATE.
 * Mixed batches: sequences of at most 16 tokens skip the chunk set-up. With few sequences
 * (n_seqs H_v d_v / 32 <= 8 x the SM count) and H_v = H_k or 2 H_k they run in one kernel
 * that computes their front itself (fp32) and keeps the state in registers across their
 * tokens (a thread-block cluster per key head shares the conv-state roll); with more, the
 * front kernel writes their fp16 q, k, v, g, beta to 16 compact rows per sequence in the
 * workspace (gdn_prefill_workspace_size counts them when n_seqs > 1) and the token-by-token
 * kernel runs them. The record and scan kernels take the longer sequences and are not
 * launched when no sequence can be longer (T_total <= 16).
 * Supported: d_k = d_v = 128, chunk 64, d_conv = 4, x and conv_state GDN_BF16 (the q, k, v
 * operands are fp16); GDN_EUNSUPPORTED otherwise.
 */
int gdn_layer_prefill(const gdn_dims* dims, const void* x, int32_t x_dtype, const float* conv_w,
                      void* conv_state, int32_t conv_state_dtype, const int32_t* cu_seqlens,
                      const int32_t* slot_ids, const uint8_t* reset, int32_t n_seqs,
                      int64_t T_total, const float* a, const float* b, const float* A_log,
                      const float* dt_bias, float eps, float q_scale, float* state, int32_t chunk,
                      void* o, int32_t o_dtype, void* workspace, size_t workspace_bytes,
                      uint32_t flags, const gdn_out_gate* gate, gdn_stream_t stream);

/*
 * gdn_gated_norm -- the output gate on its own: out = RMSNorm(o) * norm_w * SiLU(z) for
 * T_total tokens (see gdn_out_gate), e.g. after gdn_chunked_prefill or gdn_decode_step.
 *   o [T_total][H_v][d_v] (o_dtype F32 or BF16); out likewise (out_dtype F32 or BF16); out
 *   may equal o (in place).
 */
int gdn_gated_norm(const gdn_dims* dims, const void* o, int32_t o_dtype, const gdn_out_gate* gate,
                   void* out, int32_t out_dtype, int64_t T_total, gdn_stream_t stream);

/*
 * gdn_chunked_prefill_noalloc -- gdn_chunked_prefill on the tensor-core path for callers that
 * cannot allocate device memory for a workspace: for example code that runs inside a host
 * framework that owns every device allocation and offers no allocation hook, or a
 * latency-critical loop that must not call cudaMalloc/cudaFree (both can synchronise the
 * device). The pages have no counterpart of this entry point.
 * Same arguments and results as gdn_chunked_prefill without workspace / flags. Scratch comes
 * from a 64 MiB array in device global memory that the library reserves on every GPU that
 * loads it, for the life of the process; nothing is allocated per call. Limits and rules:
 *  - only the tensor-core configuration (d_k = d_v = 128, chunk 64, qkv_dtype GDN_F16),
 *    GDN_EUNSUPPORTED otherwise;
 *  - needs (ceil(T_total / 64) + n_seqs) * H_v * 73984 bytes <= 64 MiB (for H_v = 32 about
 *    28 chunk slots, e.g. one sequence of 1728 tokens), GDN_EWORKSPACE otherwise, before any
 *    launch;
 *  - all calls on a device share the array: calls that overlap on the GPU (other streams or
 *    host threads) race and corrupt each other's results; serialise them;
 *  - the first call on a device looks up the array's device address with that device
 *    current, so make it before any stream capture.
 */
int gdn_chunked_prefill_noalloc(const gdn_dims* dims, const void* q, const void* k,
                                const void* v, int32_t qkv_dtype, const float* g,
                                const float* beta, float* state, const int32_t* slot_ids,
                                const int32_t* cu_seqlens, const uint8_t* reset, int32_t n_seqs,
                                int64_t T_total, int32_t chunk, void* o, int32_t o_dtype,
                                gdn_stream_t stream);

/*
 * gdn_state_slot_copy -- state[dst[i]] = state[src[i]] and conv_state[dst[i]] =
 * conv_state[src[i]] for i < n, bit-exactly (fork a sequence's recurrent state).
 * Pages: the recurrent-state copy map s_copy of llama.cpp PR #16095
 * (llm_graph_input_rs::set_input). dst slots must be distinct and must not appear in src:
 * a pair whose dst repeats an earlier pair's dst, or appears anywhere in src, is skipped
 * (GDN_ESLOT is recorded); the other pairs are copied.
 *   state      [n_slots][H_v][d_k][d_v] fp32 (may be NULL to copy only conv_state)
 *   conv_state [n_slots][d_conv-1][conv_dim] of conv_state_dtype (may be NULL)
 *   src, dst   [n] int32 device arrays
 */
int gdn_state_slot_copy(const gdn_dims* dims, float* state, void* conv_state,
                        int32_t conv_state_dtype, const int32_t* src, const int32_t* dst,
                        int32_t n, gdn_stream_t stream);

/*
 * Decode pipeline with host buffers -- gdn_layer_decode fed from and returned to HOST memory,
 * each step's copies overlapped with the neighbouring steps' compute. It is the one part of
 * this ABI that keeps state between calls and takes host pointers: a pipeline object holds
 * the layer's device arrays (given once), a caller-owned device buffer with two sets of
 * staged inputs and outputs and the decode workspace, and two copy streams with their
 * events, which gdn_decode_pipe_create makes and gdn_decode_pipe_destroy releases.
 * Step s (gdn_decode_pipe_step) uses staging set s % 2: the input copy stream waits until the
 * compute of step s - 2 has read that set, then copies x, a, b, the slot ids and the reset
 * flags from the host into it (one copy each, or one for a packed input row); the compute
 * stream waits for those copies and
 * for the output copy of step s - 2 and runs gdn_layer_decode on the set; the output copy
 * stream then copies o to the host. Steps run in order on the compute stream (each reads the
 * state the previous one wrote); a step's input copy overlaps the previous step's compute and
 * its output copy the next step's. Host buffers must stay valid and unchanged until the
 * step's copies have run; pinned host memory (cudaHostAlloc, cudaHostRegister) keeps the
 * copies asynchronous. No output gate (use gdn_layer_decode for gated steps). A pipeline is
 * used by one host thread at a time; steps are issued on the device that was current at
 * creation (GDN_EINVAL from another).
 * Pages: as gdn_layer_decode.
 */
typedef struct gdn_decode_pipe gdn_decode_pipe;

/* Device buffer bytes a pipeline for n_seqs sequences needs (0 for invalid arguments). */
size_t gdn_decode_pipe_buffer_size(const gdn_dims* dims, int32_t n_seqs, int32_t x_dtype,
                                   int32_t o_dtype);

/*
 * gdn_decode_pipe_create -- a pipeline for steps of n_seqs sequences on the current device.
 *   dims, x_dtype, conv_w, conv_state, conv_state_dtype, A_log, dt_bias, eps, q_scale, state,
 *       o_dtype: as gdn_layer_decode; the device arrays are used by every step and must
 *       outlive the pipeline
 *   buffer / buffer_bytes: device memory of at least gdn_decode_pipe_buffer_size bytes,
 *       256-byte aligned, owned by the caller, used by the pipeline until it is destroyed
 *   compute: the stream the steps' kernels run on
 *   *pipe receives the pipeline. Returns GDN_OK, GDN_EINVAL / GDN_EALIGN / GDN_EWORKSPACE for
 *   bad arguments or GDN_ECUDA if a stream or event could not be created.
 */
int gdn_decode_pipe_create(const gdn_dims* dims, int32_t n_seqs, int32_t x_dtype,
                           const float* conv_w, void* conv_state, int32_t conv_state_dtype,
                           const float* A_log, const float* dt_bias, float eps, float q_scale,
                           float* state, int32_t o_dtype, void* buffer, size_t buffer_bytes,
                           gdn_stream_t compute, gdn_decode_pipe** pipe);

/*
 * gdn_decode_pipe_step -- enqueue one step (see above). HOST pointers: x [n_seqs][conv_dim]
 * (x_dtype), a [n_seqs][H_v] fp32 (with GDN_GATES_MIXED_BA: [n_seqs][H_k][2 r], and b NULL),
 * b [n_seqs][H_v] fp32, slot_ids [n_seqs] int32, reset [n_seqs] uint8 or NULL, o
 * [n_seqs][H_v][d_v] (o_dtype) receiving the step's output. Returns GDN_OK or the status of
 * the copies or of gdn_layer_decode; asynchronous.
 */
int gdn_decode_pipe_step(gdn_decode_pipe* pipe, const void* x, const float* a, const float* b,
                         const int32_t* slot_ids, const uint8_t* reset, void* o);

/*
 * gdn_decode_pipe_step_packed -- gdn_decode_pipe_step with x, a, b and the slot ids in ONE host
 * row (a single host-to-device copy): x at byte 0, then a, b (absent with GDN_GATES_MIXED_BA)
 * and the slot ids, each starting at the previous array's end rounded up to a multiple of 256
 * bytes; gdn_decode_pipe_packed_bytes gives the row's length (0 for invalid arguments). The
 * row must be one host allocation.
 */
size_t gdn_decode_pipe_packed_bytes(const gdn_dims* dims, int32_t n_seqs, int32_t x_dtype);
int gdn_decode_pipe_step_packed(gdn_decode_pipe* pipe, const void* in, const uint8_t* reset,
                                void* o);

/* Make the compute stream wait for every copy issued so far: once that stream is
 * synchronised after this call, every step's output is in host memory. */
int gdn_decode_pipe_flush(gdn_decode_pipe* pipe);

/* Wait for the pipeline's copy streams, then release its streams, events and object. The
 * buffer stays the caller's, who must not release it before the compute stream has passed the
 * last step (synchronise it, or order the release after it). NULL is a no-op. */
int gdn_decode_pipe_destroy(gdn_decode_pipe* pipe);

/*
 * gdn_device_status -- synchronise `stream`, then read (and if `clear`, reset to GDN_OK)
 * the status word the kernels of the current device write on a device-side error.
 * *status receives GDN_OK or the first recorded negative status. Returns GDN_OK or
 * GDN_ECUDA if the synchronisation or copy failed.
 */
int gdn_device_status(int32_t* status, int32_t clear, gdn_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* gdn_status_string(int32_t status);

/* ABI version of this header (incremented on incompatible change). */
int32_t gdn_abi_version(void);

/*
 * gdn_debug_set_wait_limit -- diagnostics: the bound, in SM clock cycles, of the device-side
 * waits of the tensor-core prefill's first kernel (the one that writes the workspace records)
 * for calls enqueued from now on; 0 restores the default of about one second. A wait that
 * runs out records GDN_ETIMEOUT, lets what the block already issued finish and ends the
 * block; the call's results are then undefined. It lets a test drive that path without a
 * fault. Process-wide; returns GDN_EINVAL for a negative limit.
 */
int32_t gdn_debug_set_wait_limit(int64_t cycles);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
