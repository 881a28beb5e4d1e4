// Host-side launch interfaces shared by the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

struct FrontArgs {
  const void* x; int x_dtype;
  const float* conv_w;
  void* conv_state; int conv_state_dtype;
  const int32_t* cu_seqlens; const int32_t* slot_ids; const uint8_t* reset;
  int n_seqs; int64_t T_total;
  const float* a; const float* b; const float* A_log; const float* dt_bias;
  float eps; float q_scale;
  void* q; void* k; void* v; int qkv_dtype;
  float* g; float* beta;
  int H_k, H_v, d_k, d_v, d_conv, n_slots;
  int layout;  // GDN_GQA_TILED | GDN_GATES_MIXED_BA
  int32_t* status;
  // > 0: only sequences of at most max_len tokens (the others are left alone, conv state
  // included), and token j of sequence n writes its q, k, v, g, beta at the compact row
  // n * max_len + j (front4_kernel only)
  int max_len;
};

struct DecodeArgs {
  const void* q; const void* k; const void* v; int qkv_dtype;
  const float* g; const float* beta;
  float* state; const int32_t* slot_ids; const uint8_t* reset; int n_seqs;
  void* o; int o_dtype;
  int H_k, H_v, d_k, d_v, n_slots;
  int layout;
  int32_t* status;
  // output gate fused into the one-kernel layer decode (z == nullptr: none): o receives
  // RMSNorm(o) * norm_w * SiLU(z), z [n_seqs][H_v][d_v]; decode_kernel takes none
  const void* z; int z_dtype; const float* norm_w; float norm_eps;
  // set by the launcher: L2 prefetch distance of decode_kernel in blocks (0: none)
  int pf_dist;
};

// The output gate as its own kernel: out = RMSNorm(o) * norm_w * SiLU(z) per row of d_v.
struct GateArgs {
  const void* o; int o_dtype;
  const void* z; int z_dtype;
  const float* norm_w; float eps;
  void* out; int out_dtype;
  int64_t rows; int d_v;
};

struct PrefillArgs {
  const void* q; const void* k; const void* v; int qkv_dtype;
  const float* g; const float* beta;
  float* state; const int32_t* slot_ids; const int32_t* cu_seqlens; const uint8_t* reset;
  int n_seqs; int64_t T_total; int chunk;
  void* o; int o_dtype;
  void* workspace; size_t workspace_bytes;
  int H_k, H_v, d_k, d_v, n_slots;
  int layout;
  uint32_t flags;  // GDN_PREFILL_*
  int32_t* status;
  // sequences of at most short_max tokens are left to the token-by-token kernel of the same
  // call (launch_recurrent); 0 = the chunked kernels take every sequence
  int short_max;
  // limit (SM clock cycles) of the record kernel's device-side waits; 0 = the default
  long long wait_cycles;
  // > 0 (token-by-token kernel): q, k, v, g, beta of token j of sequence n sit at the compact
  // row n * compact_rows + j (as the front writes them with max_len = compact_rows)
  int compact_rows;
  // layer prefill (gdn_layer_prefill): the prep computes q, k, v, g, beta from x itself and
  // the scan writes the new conv state; q, k, v, g, beta above are unused
  int fused;
  const void* x;            // [T_total][conv_dim] bf16
  const float* conv_w;      // [conv_dim][4]
  void* conv_state;         // [n_slots][3][conv_dim] bf16
  const float* fa; const float* fb;  // [T_total][H_v]
  const float* A_log; const float* dt_bias;
  float eps, q_scale;
};

struct SlotCopyArgs {
  float* state; void* conv_state; int conv_state_dtype;
  const int32_t* src; const int32_t* dst; int n;
  int64_t state_elems;      // floats per slot
  int64_t conv_bytes;       // bytes per slot of conv state
  int n_slots;
  int32_t* status;
};

cudaError_t launch_front(const FrontArgs& a, cudaStream_t s);
// after_front: the kernel just before this one on the stream is this library's front kernel
// (launched by gdn_layer_decode), so the state may be read before waiting for it.
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, bool after_front);
// gdn_layer_decode in one kernel (the front computed inside the decode step); for
// d_k = d_v = 128, d_conv = 4, H_v = H_k or 2 H_k (else cudaErrorNotSupported). f holds the
// front's inputs (its q, k, v, g, beta and cu_seqlens are unused).
bool layer_decode_fused_supported(const DecodeArgs& a, const FrontArgs& f);
// Supported and faster than the two-kernel path: small batches (measured crossover between
// 8 and 16 sequences at H_v = 32).
bool layer_decode_fused_preferred(const DecodeArgs& a, const FrontArgs& f);
cudaError_t launch_layer_decode(const DecodeArgs& a, const FrontArgs& f, cudaStream_t s);
cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s);
// Token-by-token recurrence (state in registers across a sequence's tokens); with
// max_len > 0 only sequences of at most max_len tokens are processed.
cudaError_t launch_recurrent(const PrefillArgs& a, int max_len, cudaStream_t s);
// Layer prefill (a.fused): sequences of at most max_len (<= 16) tokens in one kernel, the
// front computed inside; d_k = d_v = 128 and H_v = H_k or 2 H_k (else cudaErrorNotSupported).
bool layer_short_supported(const PrefillArgs& a);
cudaError_t launch_layer_short(const PrefillArgs& a, int max_len, cudaStream_t s);
cudaError_t launch_slot_copy(const SlotCopyArgs& a, cudaStream_t s);
cudaError_t launch_gated_norm(const GateArgs& a, cudaStream_t s);

// Tensor-core (tcgen05) chunked prefill; returns cudaErrorNotSupported for shapes it does
// not cover.
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s);

size_t prefill_tc_workspace(int H_v, int d_k, int d_v, int64_t T_total, int n_seqs, int chunk);
bool prefill_tc_supported(int d_k, int d_v, int chunk, int qkv_dtype);
// Same kernels with the library's fixed device scratch array instead of a workspace;
// cudaErrorInvalidValue when the call needs more than prefill_tc_noalloc_capacity() bytes.
cudaError_t launch_prefill_tc_noalloc(const PrefillArgs& a, cudaStream_t s);
size_t prefill_tc_noalloc_capacity();

}  // namespace gdn
