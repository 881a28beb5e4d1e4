// C-ABI entry points (include/gdn.h): host-side argument validation, dtype dispatch and
// launches on the caller's stream. Nothing here allocates device memory or synchronises,
// except gdn_device_status.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace {

// Diagnostics: the limit of the prefill record kernel's device-side waits (0 = its default).
std::atomic<long long> g_wait_cycles{0};

// Per-device status word written by kernels on device-side argument errors.
__device__ int32_t g_status_word;

constexpr int kMaxDevices = 64;
int32_t* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;

int32_t* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int32_t*>(p);
  }
  return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
bool qkv_dtype_ok(int t) { return t == GDN_F32 || t == GDN_BF16 || t == GDN_F16; }
bool io_dtype_ok(int t) { return t == GDN_F32 || t == GDN_BF16; }
size_t dtype_size(int t) { return t == GDN_F32 ? 4 : 2; }

int check_dims(const gdn_dims* d) {
  if (!d) return GDN_EINVAL;
  if (d->n_slots <= 0 || d->H_k <= 0 || d->H_v <= 0 || d->H_v % d->H_k != 0) return GDN_EINVAL;
  if (d->d_conv < 0 || d->d_conv > 4) return GDN_EINVAL;
  if (d->d_k <= 0 || d->d_v <= 0) return GDN_EINVAL;
  if (!head_dim_ok(d->d_k) || !head_dim_ok(d->d_v)) return GDN_EUNSUPPORTED;
  if (d->H_v > 65535) return GDN_EUNSUPPORTED;
  if (d->layout & ~(GDN_GQA_TILED | GDN_GATES_MIXED_BA)) return GDN_EINVAL;
  return GDN_OK;
}

// An output gate argument: z and norm_w present and aligned, dtypes and eps valid.
int gate_check(const gdn_out_gate* g) {
  if (!g) return GDN_OK;
  if (!g->z || !g->norm_w || !io_dtype_ok(g->z_dtype) || !(g->eps >= 0.0f)) return GDN_EINVAL;
  if (!aligned16(g->z) || !aligned16(g->norm_w)) return GDN_EALIGN;
  return GDN_OK;
}

// The gate inputs: separate a and b, or (GDN_GATES_MIXED_BA) the fused array as a, b NULL.
bool gates_ok(const gdn_dims* d, const float* a, const float* b) {
  if (d->layout & GDN_GATES_MIXED_BA) return a != nullptr && b == nullptr;
  return a != nullptr && b != nullptr;
}

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return GDN_OK;
  if (e == cudaErrorNotSupported) return GDN_EUNSUPPORTED;
  return GDN_ECUDA;
}

// Sequences of at most this many tokens (single decode tokens, speculative or multi-token
// steps) take the token-by-token kernel; longer ones the chunked tensor-core kernels.
constexpr int kShortMax = 16;

// The tensor-core chunked prefill with mixed batches split on the device: the token-by-token
// kernel takes the sequences of at most kShortMax tokens, the chunked kernels the others. Each
// kernel reads cu_seqlens and skips the other's sequences, so one call serves any mix. From
// the host sizes alone: one sequence longer than kShortMax needs no token-by-token launch, and
// a batch of at most kShortMax tokens needs no chunked launch.
cudaError_t launch_tc_routed(gdn::PrefillArgs pa, cudaStream_t s, bool noalloc) {
  const bool maybe_short = pa.n_seqs > 1 || pa.T_total <= kShortMax;
  const bool maybe_long = pa.T_total > kShortMax;
  if (maybe_short) {
    cudaError_t e = gdn::launch_recurrent(pa, kShortMax, s);
    if (e != cudaSuccess || !maybe_long) return e;
    pa.short_max = kShortMax;
  }
  return noalloc ? gdn::launch_prefill_tc_noalloc(pa, s) : gdn::launch_prefill_tc(pa, s);
}

}  // namespace

extern "C" {

int gdn_conv_step(const gdn_dims* dims, const void* x, int32_t x_dtype, const float* conv_w,
                  void* conv_state, int32_t conv_state_dtype, const int32_t* cu_seqlens,
                  const int32_t* slot_ids, const uint8_t* reset, int32_t n_seqs,
                  int64_t T_total, const float* a, const float* b, const float* A_log,
                  const float* dt_bias, float eps, float q_scale, void* q, void* k, void* v,
                  int32_t qkv_dtype, float* g, float* beta, gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  if (n_seqs < 0 || T_total < 0) return GDN_EINVAL;
  if (n_seqs == 0) return GDN_OK;
  if (!io_dtype_ok(x_dtype) || !qkv_dtype_ok(qkv_dtype)) return GDN_EINVAL;
  const int R = dims->d_conv > 0 ? dims->d_conv - 1 : 0;
  if (dims->d_conv > 0 && !conv_w) return GDN_EINVAL;
  if (dims->d_conv == 0 && conv_w) return GDN_EINVAL;
  if (R > 0) {
    if (!conv_state || !io_dtype_ok(conv_state_dtype) || !slot_ids) return GDN_EINVAL;
  } else if (conv_state) {
    return GDN_EINVAL;
  }
  if (!cu_seqlens && T_total != n_seqs) return GDN_EINVAL;  // NULL: one token per sequence
  if (!gates_ok(dims, a, b) || !A_log || !dt_bias || !q || !k || !v || !g || !beta)
    return GDN_EINVAL;
  if (T_total > 0 && !x) return GDN_EINVAL;
  if (!(eps >= 0.0f)) return GDN_EINVAL;
  const void* ptrs[] = {x, conv_w, conv_state, a, b, q, k, v, g, beta, A_log, dt_bias};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_EALIGN;
  if (T_total == 0 && R == 0) return GDN_OK;
  gdn::FrontArgs fa{};
  fa.x = x; fa.x_dtype = x_dtype; fa.conv_w = conv_w;
  fa.conv_state = conv_state; fa.conv_state_dtype = conv_state_dtype;
  fa.cu_seqlens = cu_seqlens; fa.slot_ids = slot_ids; fa.reset = reset;
  fa.n_seqs = n_seqs; fa.T_total = T_total;
  fa.a = a; fa.b = b; fa.A_log = A_log; fa.dt_bias = dt_bias; fa.eps = eps; fa.q_scale = q_scale;
  fa.q = q; fa.k = k; fa.v = v; fa.qkv_dtype = qkv_dtype; fa.g = g; fa.beta = beta;
  fa.H_k = dims->H_k; fa.H_v = dims->H_v; fa.d_k = dims->d_k; fa.d_v = dims->d_v;
  fa.d_conv = dims->d_conv; fa.n_slots = dims->n_slots; fa.layout = dims->layout;
  fa.status = status_ptr();
  if (!fa.status) return GDN_ECUDA;
  return from_cuda(gdn::launch_front(fa, reinterpret_cast<cudaStream_t>(stream)));
}

int gdn_decode_step(const gdn_dims* dims, const void* q, const void* k, const void* v,
                    int32_t qkv_dtype, const float* g, const float* beta, float* state,
                    const int32_t* slot_ids, const uint8_t* reset, int32_t n_seqs, void* o,
                    int32_t o_dtype, gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  if (n_seqs < 0 || n_seqs > 65535) return GDN_EINVAL;
  if (n_seqs == 0) return GDN_OK;
  if (!qkv_dtype_ok(qkv_dtype) || !io_dtype_ok(o_dtype)) return GDN_EINVAL;
  if (!q || !k || !v || !g || !beta || !state || !slot_ids || !o) return GDN_EINVAL;
  const void* ptrs[] = {q, k, v, g, beta, state, o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_EALIGN;
  gdn::DecodeArgs da{};
  da.q = q; da.k = k; da.v = v; da.qkv_dtype = qkv_dtype; da.g = g; da.beta = beta;
  da.state = state; da.slot_ids = slot_ids; da.reset = reset; da.n_seqs = n_seqs;
  da.o = o; da.o_dtype = o_dtype;
  da.H_k = dims->H_k; da.H_v = dims->H_v; da.d_k = dims->d_k; da.d_v = dims->d_v;
  da.n_slots = dims->n_slots; da.layout = dims->layout;
  da.status = status_ptr();
  if (!da.status) return GDN_ECUDA;
  return from_cuda(gdn::launch_decode(da, reinterpret_cast<cudaStream_t>(stream), false));
}

namespace {
// fp32 q, k, v, g, beta of a decode step, each array 256-byte aligned in the workspace
struct DecodeWs {
  size_t q, k, v, g, beta, o32, total;
};
size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
DecodeWs decode_ws(const gdn_dims* d, int32_t n) {
  DecodeWs w{};
  const size_t qk = round256((size_t)n * d->H_k * d->d_k * 4);
  const size_t vv = round256((size_t)n * d->H_v * d->d_v * 4);
  const size_t gg = round256((size_t)n * d->H_v * 4);
  w.q = 0; w.k = qk; w.v = 2 * qk; w.g = 2 * qk + vv; w.beta = w.g + gg;
  w.o32 = w.beta + gg;  // fp32 o before the output gate (two-kernel path with a gate)
  w.total = w.o32 + vv;
  return w;
}
}  // namespace

int32_t gdn_layer_decode_launches(const gdn_dims* dims, int32_t n_seqs, int32_t gated) {
  if (check_dims(dims) != GDN_OK || n_seqs <= 0 || n_seqs > 65535) return 0;
  gdn::DecodeArgs da{};
  da.H_k = dims->H_k; da.H_v = dims->H_v; da.d_k = dims->d_k; da.d_v = dims->d_v;
  da.n_seqs = n_seqs;
  gdn::FrontArgs fa{};
  fa.d_conv = dims->d_conv;
  if (gdn::layer_decode_fused_preferred(da, fa)) return 1;
  return gated ? 3 : 2;
}

size_t gdn_decode_workspace_size(const gdn_dims* dims, int32_t n_seqs) {
  if (check_dims(dims) != GDN_OK || n_seqs <= 0) return 0;
  return decode_ws(dims, n_seqs).total;
}

int gdn_layer_decode(const gdn_dims* dims, const void* x, int32_t x_dtype, const float* conv_w,
                     void* conv_state, int32_t conv_state_dtype, const int32_t* slot_ids,
                     const uint8_t* reset, int32_t n_seqs, const float* a, const float* b,
                     const float* A_log, const float* dt_bias, float eps, float q_scale,
                     float* state, void* o, int32_t o_dtype, void* workspace,
                     size_t workspace_bytes, const gdn_out_gate* gate, gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  rc = gate_check(gate);
  if (rc != GDN_OK) return rc;
  if (n_seqs < 0 || n_seqs > 65535) return GDN_EINVAL;
  if (n_seqs == 0) return GDN_OK;
  if (!io_dtype_ok(x_dtype) || !io_dtype_ok(o_dtype)) return GDN_EINVAL;
  const int R = dims->d_conv > 0 ? dims->d_conv - 1 : 0;
  if (dims->d_conv > 0 && !conv_w) return GDN_EINVAL;
  if (dims->d_conv == 0 && conv_w) return GDN_EINVAL;
  if (R > 0) {
    if (!conv_state || !io_dtype_ok(conv_state_dtype)) return GDN_EINVAL;
  } else if (conv_state) {
    return GDN_EINVAL;
  }
  if (!x || !gates_ok(dims, a, b) || !A_log || !dt_bias || !state || !slot_ids || !o)
    return GDN_EINVAL;
  if (!(eps >= 0.0f)) return GDN_EINVAL;
  const void* ptrs[] = {x, conv_w, conv_state, a, b, A_log, dt_bias, state, o, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_EALIGN;
  const DecodeWs w = decode_ws(dims, n_seqs);
  if (!workspace || workspace_bytes < w.total) return GDN_EWORKSPACE;
  int32_t* status = status_ptr();
  if (!status) return GDN_ECUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* q = reinterpret_cast<float*>(ws + w.q);
  float* k = reinterpret_cast<float*>(ws + w.k);
  float* v = reinterpret_cast<float*>(ws + w.v);
  float* g = reinterpret_cast<float*>(ws + w.g);
  float* beta = reinterpret_cast<float*>(ws + w.beta);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  gdn::FrontArgs fa{};
  fa.x = x; fa.x_dtype = x_dtype; fa.conv_w = conv_w;
  fa.conv_state = conv_state; fa.conv_state_dtype = conv_state_dtype;
  fa.cu_seqlens = nullptr;  // one token per sequence
  fa.slot_ids = slot_ids; fa.reset = reset;
  fa.n_seqs = n_seqs; fa.T_total = n_seqs;
  fa.a = a; fa.b = b; fa.A_log = A_log; fa.dt_bias = dt_bias; fa.eps = eps; fa.q_scale = q_scale;
  fa.q = q; fa.k = k; fa.v = v; fa.qkv_dtype = GDN_F32; fa.g = g; fa.beta = beta;
  fa.H_k = dims->H_k; fa.H_v = dims->H_v; fa.d_k = dims->d_k; fa.d_v = dims->d_v;
  fa.d_conv = dims->d_conv; fa.n_slots = dims->n_slots; fa.layout = dims->layout;
  fa.status = status;
  gdn::DecodeArgs da{};
  da.q = q; da.k = k; da.v = v; da.qkv_dtype = GDN_F32; da.g = g; da.beta = beta;
  da.state = state; da.slot_ids = slot_ids; da.reset = reset; da.n_seqs = n_seqs;
  da.o = o; da.o_dtype = o_dtype;
  da.H_k = dims->H_k; da.H_v = dims->H_v; da.d_k = dims->d_k; da.d_v = dims->d_v;
  da.n_slots = dims->n_slots; da.layout = dims->layout;
  da.status = status;
  // small batches at the Qwen3-Next shape: one kernel computes the front inside the step (and
  // the output gate: the column tiles of a head share a cluster)
  if (gdn::layer_decode_fused_preferred(da, fa)) {
    if (gate) {
      da.z = gate->z; da.z_dtype = gate->z_dtype; da.norm_w = gate->norm_w;
      da.norm_eps = gate->eps;
    }
    return from_cuda(gdn::launch_layer_decode(da, fa, s));
  }
  rc = from_cuda(gdn::launch_front(fa, s));
  if (rc != GDN_OK) return rc;
  // with an output gate the step writes fp32 o into the workspace, gated into o afterwards
  float* o32 = reinterpret_cast<float*>(ws + w.o32);
  if (gate) { da.o = o32; da.o_dtype = GDN_F32; }
  // the front kernel was just launched on this stream (with a normal launch, so it started
  // after all earlier work): the decode may read the state before waiting for the front
  rc = from_cuda(gdn::launch_decode(da, s, true));
  if (rc != GDN_OK || !gate) return rc;
  gdn::GateArgs ga{};
  ga.o = o32; ga.o_dtype = GDN_F32; ga.z = gate->z; ga.z_dtype = gate->z_dtype;
  ga.norm_w = gate->norm_w; ga.eps = gate->eps; ga.out = o; ga.out_dtype = o_dtype;
  ga.rows = (int64_t)n_seqs * dims->H_v; ga.d_v = dims->d_v;
  return from_cuda(gdn::launch_gated_norm(ga, s));
}

namespace {
// fp32 output of a gated layer prefill, after the records in the workspace
size_t gate_out_bytes(const gdn_dims* d, int64_t T_total) {
  return round256((size_t)T_total * d->H_v * d->d_v * 4);
}
// Short sequences of a many-sequence layer prefill: their fp16 q, k, v and fp32 g, beta at
// kShortMax compact rows per sequence (after the records and the gate's o)
struct ShortWs {
  size_t q, k, v, g, beta, total;
};
ShortWs short_ws(const gdn_dims* d, int32_t n_seqs) {
  ShortWs w{};
  if (n_seqs <= 1) return w;
  const size_t rows = (size_t)n_seqs * kShortMax;
  const size_t qk = round256(rows * d->H_k * d->d_k * 2);
  const size_t vv = round256(rows * d->H_v * d->d_v * 2);
  const size_t gg = round256(rows * d->H_v * 4);
  w.q = 0; w.k = qk; w.v = 2 * qk; w.g = 2 * qk + vv; w.beta = w.g + gg; w.total = w.beta + gg;
  return w;
}
// Whether the layer prefill's short sequences take the one-kernel path (front inside, cluster
// per key head): small grids; past about one and a half waves the front kernel + token-by-token
// kernel pair is faster (as for the layer decode)
bool layer_short_one_kernel(const gdn::PrefillArgs& pa) {
  if (!gdn::layer_short_supported(pa)) return false;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return false;
  return (int64_t)pa.n_seqs * pa.H_v * (pa.d_v / 32) <= 8LL * sms;
}
}  // namespace

size_t gdn_prefill_workspace_size(const gdn_dims* dims, int64_t T_total, int32_t n_seqs,
                                  int32_t chunk, int32_t qkv_dtype, uint32_t flags) {
  if (check_dims(dims) != GDN_OK || T_total < 0 || n_seqs <= 0) return 0;
  if (flags & GDN_PREFILL_RECURRENT) {
    // gdn_layer_prefill with only short sequences: the gate's fp32 o and the compact rows
    // (gdn_chunked_prefill needs none with this flag)
    size_t need = (flags & GDN_PREFILL_OUT_GATE) ? gate_out_bytes(dims, T_total) : 0;
    const size_t sw = short_ws(dims, n_seqs).total;
    if (sw) need = round256(need) + sw;
    return need;
  }
  if ((flags & GDN_PREFILL_SIMT) || qkv_dtype == GDN_F32) return 0;
  if (!gdn::prefill_tc_supported(dims->d_k, dims->d_v, chunk, qkv_dtype)) return 0;
  size_t need = gdn::prefill_tc_workspace(dims->H_v, dims->d_k, dims->d_v, T_total, n_seqs, chunk);
  if (flags & GDN_PREFILL_OUT_GATE) need = round256(need) + gate_out_bytes(dims, T_total);
  // room for the short sequences of a many-sequence layer prefill
  const size_t sw = short_ws(dims, n_seqs).total;
  if (sw) need = round256(need) + sw;
  return need;
}

int gdn_chunked_prefill(const gdn_dims* dims, const void* q, const void* k, const void* v,
                        int32_t qkv_dtype, const float* g, const float* beta, float* state,
                        const int32_t* slot_ids, const int32_t* cu_seqlens,
                        const uint8_t* reset, int32_t n_seqs, int64_t T_total, int32_t chunk,
                        void* o, int32_t o_dtype, void* workspace, size_t workspace_bytes,
                        uint32_t flags, gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  if (n_seqs < 0 || n_seqs > 65535 || T_total < 0) return GDN_EINVAL;
  if (n_seqs == 0) return GDN_OK;
  if (chunk != 16 && chunk != 32 && chunk != 64) return GDN_EINVAL;
  if (!qkv_dtype_ok(qkv_dtype) || !io_dtype_ok(o_dtype)) return GDN_EINVAL;
  if (!state || !slot_ids || !cu_seqlens) return GDN_EINVAL;
  if (T_total > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_EINVAL;
  if (flags & ~(uint32_t)(GDN_PREFILL_SIMT | GDN_PREFILL_RECURRENT | GDN_PREFILL_TC_HEAD_SCAN |
                          GDN_PREFILL_TC_TILE_SCAN))
    return GDN_EINVAL;
  if ((flags & GDN_PREFILL_TC_HEAD_SCAN) && (flags & GDN_PREFILL_TC_TILE_SCAN)) return GDN_EINVAL;
  const void* ptrs[] = {q, k, v, g, beta, state, o, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_EALIGN;
  gdn::PrefillArgs pa{};
  pa.q = q; pa.k = k; pa.v = v; pa.qkv_dtype = qkv_dtype; pa.g = g; pa.beta = beta;
  pa.state = state; pa.slot_ids = slot_ids; pa.cu_seqlens = cu_seqlens; pa.reset = reset;
  pa.n_seqs = n_seqs; pa.T_total = T_total; pa.chunk = chunk; pa.o = o; pa.o_dtype = o_dtype;
  pa.workspace = workspace; pa.workspace_bytes = workspace_bytes;
  pa.H_k = dims->H_k; pa.H_v = dims->H_v; pa.d_k = dims->d_k; pa.d_v = dims->d_v;
  pa.n_slots = dims->n_slots; pa.layout = dims->layout;
  pa.wait_cycles = g_wait_cycles.load();
  pa.flags = flags;
  pa.status = status_ptr();
  if (!pa.status) return GDN_ECUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (flags & GDN_PREFILL_RECURRENT) return from_cuda(gdn::launch_recurrent(pa, 0, s));
  const bool simt = (flags & GDN_PREFILL_SIMT) || qkv_dtype == GDN_F32 ||
                    !gdn::prefill_tc_supported(dims->d_k, dims->d_v, chunk, qkv_dtype);
  if (simt) return from_cuda(gdn::launch_prefill_simt(pa, s));
  const size_t need =
      gdn::prefill_tc_workspace(dims->H_v, dims->d_k, dims->d_v, T_total, n_seqs, chunk);
  if (need > 0 && (!workspace || workspace_bytes < need)) return GDN_EWORKSPACE;
  return from_cuda(launch_tc_routed(pa, s, false));
}

int gdn_layer_prefill(const gdn_dims* dims, const void* x, int32_t x_dtype, const float* conv_w,
                      void* conv_state, int32_t conv_state_dtype, const int32_t* cu_seqlens,
                      const int32_t* slot_ids, const uint8_t* reset, int32_t n_seqs,
                      int64_t T_total, const float* a, const float* b, const float* A_log,
                      const float* dt_bias, float eps, float q_scale, float* state, int32_t chunk,
                      void* o, int32_t o_dtype, void* workspace, size_t workspace_bytes,
                      uint32_t flags, const gdn_out_gate* gate, gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  rc = gate_check(gate);
  if (rc != GDN_OK) return rc;
  if (n_seqs < 0 || n_seqs > 65535 || T_total < 0) return GDN_EINVAL;
  if (n_seqs == 0) return GDN_OK;
  if (chunk != 16 && chunk != 32 && chunk != 64) return GDN_EINVAL;
  if (!io_dtype_ok(x_dtype) || !io_dtype_ok(o_dtype) || !io_dtype_ok(conv_state_dtype))
    return GDN_EINVAL;
  if (!state || !slot_ids || !cu_seqlens || !conv_w || !conv_state || !gates_ok(dims, a, b) ||
      !A_log || !dt_bias)
    return GDN_EINVAL;
  if (T_total > 0 && (!x || !o)) return GDN_EINVAL;
  if (!(eps >= 0.0f)) return GDN_EINVAL;
  if (flags & ~(uint32_t)(GDN_PREFILL_OUT_GATE | GDN_PREFILL_TC_HEAD_SCAN |
                          GDN_PREFILL_TC_TILE_SCAN | GDN_PREFILL_RECURRENT))
    return GDN_EINVAL;
  if ((flags & GDN_PREFILL_TC_HEAD_SCAN) && (flags & GDN_PREFILL_TC_TILE_SCAN)) return GDN_EINVAL;
  const void* ptrs[] = {x, conv_w, conv_state, a, b, A_log, dt_bias, state, o, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_EALIGN;
  if (!gdn::prefill_tc_supported(dims->d_k, dims->d_v, chunk, GDN_F16) || dims->d_conv != 4 ||
      x_dtype != GDN_BF16 || conv_state_dtype != GDN_BF16)
    return GDN_EUNSUPPORTED;
  // GDN_PREFILL_RECURRENT: every sequence has at most kShortMax tokens (no records)
  const bool only_short = (flags & GDN_PREFILL_RECURRENT) != 0;
  const size_t rec = only_short ? 0 :
      gdn::prefill_tc_workspace(dims->H_v, dims->d_k, dims->d_v, T_total, n_seqs, chunk);
  const size_t base = gate ? round256(rec) + gate_out_bytes(dims, T_total) : rec;
  const ShortWs sw = short_ws(dims, n_seqs);
  const size_t need = sw.total ? round256(base) + sw.total : base;
  if (need > 0 && (!workspace || workspace_bytes < need)) return GDN_EWORKSPACE;
  gdn::PrefillArgs pa{};
  pa.qkv_dtype = GDN_F16;
  pa.state = state; pa.slot_ids = slot_ids; pa.cu_seqlens = cu_seqlens; pa.reset = reset;
  pa.n_seqs = n_seqs; pa.T_total = T_total; pa.chunk = chunk; pa.o = o; pa.o_dtype = o_dtype;
  pa.workspace = workspace; pa.workspace_bytes = workspace_bytes;
  pa.H_k = dims->H_k; pa.H_v = dims->H_v; pa.d_k = dims->d_k; pa.d_v = dims->d_v;
  pa.n_slots = dims->n_slots; pa.layout = dims->layout;
  pa.wait_cycles = g_wait_cycles.load();
  pa.flags = flags;
  pa.fused = 1;
  pa.x = x; pa.conv_w = conv_w; pa.conv_state = conv_state; pa.fa = a; pa.fb = b;
  pa.A_log = A_log; pa.dt_bias = dt_bias; pa.eps = eps; pa.q_scale = q_scale;
  pa.status = status_ptr();
  if (!pa.status) return GDN_ECUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // with an output gate the prefill writes fp32 into the workspace, gated into o afterwards
  float* o32 = gate ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round256(rec))
                    : nullptr;
  if (gate) { pa.o = o32; pa.o_dtype = GDN_F32; }
  // sequences of at most kShortMax tokens: one kernel with the front inside and the state in
  // registers; the record and scan kernels skip them (and are not launched when no sequence
  // can be longer)
  const bool maybe_short = n_seqs > 1 || T_total <= kShortMax || only_short;
  const bool maybe_long = T_total > kShortMax && !only_short;
  // a single sequence outside the one-kernel path's shapes has no short route
  if (only_short && !layer_short_one_kernel(pa) && sw.total == 0) return GDN_EUNSUPPORTED;
  if (maybe_short && layer_short_one_kernel(pa)) {
    rc = from_cuda(gdn::launch_layer_short(pa, kShortMax, s));
    if (rc != GDN_OK) return rc;
    pa.short_max = kShortMax;
  } else if (maybe_short && sw.total) {
    // the front of the short sequences only (compact rows in the workspace), then the
    // token-by-token kernel on them
    uint8_t* swp = static_cast<uint8_t*>(workspace) + round256(base);
    gdn::FrontArgs fa{};
    fa.x = x; fa.x_dtype = x_dtype; fa.conv_w = conv_w;
    fa.conv_state = conv_state; fa.conv_state_dtype = conv_state_dtype;
    fa.cu_seqlens = cu_seqlens; fa.slot_ids = slot_ids; fa.reset = reset;
    fa.n_seqs = n_seqs; fa.T_total = T_total;
    fa.a = a; fa.b = b; fa.A_log = A_log; fa.dt_bias = dt_bias; fa.eps = eps;
    fa.q_scale = q_scale;
    fa.q = swp + sw.q; fa.k = swp + sw.k; fa.v = swp + sw.v; fa.qkv_dtype = GDN_F16;
    fa.g = reinterpret_cast<float*>(swp + sw.g); fa.beta = reinterpret_cast<float*>(swp + sw.beta);
    fa.H_k = dims->H_k; fa.H_v = dims->H_v; fa.d_k = dims->d_k; fa.d_v = dims->d_v;
    fa.d_conv = dims->d_conv; fa.n_slots = dims->n_slots; fa.layout = dims->layout;
    fa.status = pa.status;
    fa.max_len = kShortMax;
    rc = from_cuda(gdn::launch_front(fa, s));
    if (rc != GDN_OK) return rc;
    gdn::PrefillArgs pr = pa;
    pr.fused = 0;
    pr.q = fa.q; pr.k = fa.k; pr.v = fa.v; pr.qkv_dtype = GDN_F16; pr.g = fa.g;
    pr.beta = fa.beta;
    pr.compact_rows = kShortMax;
    rc = from_cuda(gdn::launch_recurrent(pr, kShortMax, s));
    if (rc != GDN_OK) return rc;
    pa.short_max = kShortMax;
  }
  if (!only_short && (maybe_long || pa.short_max == 0)) {
    rc = from_cuda(gdn::launch_prefill_tc(pa, s));
    if (rc != GDN_OK) return rc;
  }
  if (!gate || T_total == 0) return GDN_OK;
  gdn::GateArgs ga{};
  ga.o = o32; ga.o_dtype = GDN_F32; ga.z = gate->z; ga.z_dtype = gate->z_dtype;
  ga.norm_w = gate->norm_w; ga.eps = gate->eps; ga.out = o; ga.out_dtype = o_dtype;
  ga.rows = T_total * dims->H_v; ga.d_v = dims->d_v;
  return from_cuda(gdn::launch_gated_norm(ga, s));
}

int gdn_gated_norm(const gdn_dims* dims, const void* o, int32_t o_dtype, const gdn_out_gate* gate,
                   void* out, int32_t out_dtype, int64_t T_total, gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  if (!gate || T_total < 0) return GDN_EINVAL;
  rc = gate_check(gate);
  if (rc != GDN_OK) return rc;
  if (!io_dtype_ok(o_dtype) || !io_dtype_ok(out_dtype)) return GDN_EINVAL;
  if (T_total == 0) return GDN_OK;
  if (!o || !out) return GDN_EINVAL;
  if (!aligned16(o) || !aligned16(out)) return GDN_EALIGN;
  gdn::GateArgs ga{};
  ga.o = o; ga.o_dtype = o_dtype; ga.z = gate->z; ga.z_dtype = gate->z_dtype;
  ga.norm_w = gate->norm_w; ga.eps = gate->eps; ga.out = out; ga.out_dtype = out_dtype;
  ga.rows = T_total * dims->H_v; ga.d_v = dims->d_v;
  return from_cuda(gdn::launch_gated_norm(ga, reinterpret_cast<cudaStream_t>(stream)));
}

int gdn_chunked_prefill_noalloc(const gdn_dims* dims, const void* q, const void* k,
                                const void* v, int32_t qkv_dtype, const float* g,
                                const float* beta, float* state, const int32_t* slot_ids,
                                const int32_t* cu_seqlens, const uint8_t* reset, int32_t n_seqs,
                                int64_t T_total, int32_t chunk, void* o, int32_t o_dtype,
                                gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  if (n_seqs < 0 || n_seqs > 65535 || T_total < 0) return GDN_EINVAL;
  if (n_seqs == 0) return GDN_OK;
  if (chunk != 16 && chunk != 32 && chunk != 64) return GDN_EINVAL;
  if (!qkv_dtype_ok(qkv_dtype) || !io_dtype_ok(o_dtype)) return GDN_EINVAL;
  if (!state || !slot_ids || !cu_seqlens) return GDN_EINVAL;
  if (T_total > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_EINVAL;
  const void* ptrs[] = {q, k, v, g, beta, state, o};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_EALIGN;
  if (!gdn::prefill_tc_supported(dims->d_k, dims->d_v, chunk, qkv_dtype)) return GDN_EUNSUPPORTED;
  if (gdn::prefill_tc_workspace(dims->H_v, dims->d_k, dims->d_v, T_total, n_seqs, chunk) >
      gdn::prefill_tc_noalloc_capacity())
    return GDN_EWORKSPACE;
  gdn::PrefillArgs pa{};
  pa.q = q; pa.k = k; pa.v = v; pa.qkv_dtype = qkv_dtype; pa.g = g; pa.beta = beta;
  pa.state = state; pa.slot_ids = slot_ids; pa.cu_seqlens = cu_seqlens; pa.reset = reset;
  pa.n_seqs = n_seqs; pa.T_total = T_total; pa.chunk = chunk; pa.o = o; pa.o_dtype = o_dtype;
  pa.H_k = dims->H_k; pa.H_v = dims->H_v; pa.d_k = dims->d_k; pa.d_v = dims->d_v;
  pa.n_slots = dims->n_slots; pa.layout = dims->layout;
  pa.wait_cycles = g_wait_cycles.load();
  pa.status = status_ptr();
  if (!pa.status) return GDN_ECUDA;
  return from_cuda(launch_tc_routed(pa, reinterpret_cast<cudaStream_t>(stream), true));
}

int gdn_state_slot_copy(const gdn_dims* dims, float* state, void* conv_state,
                        int32_t conv_state_dtype, const int32_t* src, const int32_t* dst,
                        int32_t n, gdn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != GDN_OK) return rc;
  if (n < 0 || n > 65535) return GDN_EINVAL;
  if (n == 0) return GDN_OK;
  if (!src || !dst) return GDN_EINVAL;
  if (!state && !conv_state) return GDN_EINVAL;
  if (conv_state && (!io_dtype_ok(conv_state_dtype) || dims->d_conv <= 1)) return GDN_EINVAL;
  if ((state && !aligned16(state)) || (conv_state && !aligned16(conv_state))) return GDN_EALIGN;
  gdn::SlotCopyArgs sa{};
  sa.state = state; sa.conv_state = conv_state; sa.conv_state_dtype = conv_state_dtype;
  sa.src = src; sa.dst = dst; sa.n = n;
  sa.state_elems = (int64_t)dims->H_v * dims->d_k * dims->d_v;
  const int64_t conv_dim = 2LL * dims->H_k * dims->d_k + (int64_t)dims->H_v * dims->d_v;
  sa.conv_bytes = conv_state ? (int64_t)(dims->d_conv - 1) * conv_dim *
                                   (int64_t)dtype_size(conv_state_dtype) : 0;
  sa.n_slots = dims->n_slots;
  sa.status = status_ptr();
  if (!sa.status) return GDN_ECUDA;
  return from_cuda(gdn::launch_slot_copy(sa, reinterpret_cast<cudaStream_t>(stream)));
}

int gdn_device_status(int32_t* status, int32_t clear, gdn_stream_t stream) {
  if (!status) return GDN_EINVAL;
  int32_t* p = status_ptr();
  if (!p) return GDN_ECUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ECUDA;
  int32_t host = 0;
  if (cudaMemcpy(&host, p, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDN_ECUDA;
  if (clear) {
    const int32_t zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return GDN_ECUDA;
  }
  *status = host;
  return GDN_OK;
}

const char* gdn_status_string(int32_t status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_EINVAL: return "GDN_EINVAL: invalid argument";
    case GDN_ESLOT: return "GDN_ESLOT: slot id out of range or repeated";
    case GDN_EALIGN: return "GDN_EALIGN: pointer not 16-byte aligned";
    case GDN_ECUDA: return "GDN_ECUDA: CUDA error";
    case GDN_ETIMEOUT: return "GDN_ETIMEOUT: device wait gave up";
    case GDN_EWORKSPACE: return "GDN_EWORKSPACE: workspace missing or too small";
    case GDN_EUNSUPPORTED: return "GDN_EUNSUPPORTED: unsupported shape or dtype";
  }
  return "GDN: unknown status";
}

int32_t gdn_abi_version(void) { return 2; }

int32_t gdn_debug_set_wait_limit(int64_t cycles) {
  if (cycles < 0) return GDN_EINVAL;
  g_wait_cycles.store(cycles);
  return GDN_OK;
}

}  // extern "C"
