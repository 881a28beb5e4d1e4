// Decode pipeline with host buffers (include/gdn.h, gdn_decode_pipe_*): the layer decode step
// fed from and returned to host memory. Two staging sets in a caller-owned device buffer let
// step s + 1's input copy and step s - 1's output copy run, on their own streams, while step s
// computes; the steps themselves stay in order on the compute stream, since each reads the
// recurrent and conv state the previous one wrote.
// Pages: as gdn_layer_decode (ik_llama.cpp src/llama-delta-net.cpp,
// build_layer_attn_linear_core; qwen3next.cpp build_delta_net_autoregressive).
#include <cuda_runtime.h>

#include <new>

#include "../../include/gdn.h"

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
bool io_dtype(int t) { return t == GDN_F32 || t == GDN_BF16; }
size_t esize(int t) { return t == GDN_F32 ? 4 : 2; }

// Bytes and offsets of one staging set, and of the whole buffer (two sets, then the decode
// workspace).
struct Layout {
  size_t x, a, b, slots, reset, o;   // bytes of each array
  size_t ox, oa, ob, os, orst, oo;   // offsets within a set
  size_t set, ws_off, ws, total;
};

bool layout_of(const gdn_dims* d, int32_t n, int32_t x_dtype, int32_t o_dtype, Layout* L) {
  if (!d || n <= 0 || n > 65535 || !io_dtype(x_dtype) || !io_dtype(o_dtype)) return false;
  if (d->H_k <= 0 || d->H_v <= 0 || d->d_k <= 0 || d->d_v <= 0) return false;
  const bool mixed = (d->layout & GDN_GATES_MIXED_BA) != 0;
  const size_t conv_dim = (size_t)(2 * d->H_k) * d->d_k + (size_t)d->H_v * d->d_v;
  L->x = (size_t)n * conv_dim * esize(x_dtype);
  L->a = (size_t)n * d->H_v * 4 * (mixed ? 2 : 1);  // [n][H_k][2 r] when fused
  L->b = mixed ? 0 : (size_t)n * d->H_v * 4;
  L->slots = (size_t)n * 4;
  L->reset = (size_t)n;
  L->o = (size_t)n * d->H_v * d->d_v * esize(o_dtype);
  L->ox = 0;
  L->oa = L->ox + up(L->x);
  L->ob = L->oa + up(L->a);
  L->os = L->ob + up(L->b);
  L->orst = L->os + up(L->slots);
  L->oo = L->orst + up(L->reset);
  L->set = L->oo + up(L->o);
  L->ws = gdn_decode_workspace_size(d, n);
  if (L->ws == 0) return false;
  L->ws_off = 2 * L->set;
  L->total = L->ws_off + up(L->ws);
  return true;
}

}  // namespace

struct gdn_decode_pipe {
  gdn_dims dims;
  int32_t n, x_dtype, cs_dtype, o_dtype;
  const float* conv_w;
  void* conv_state;
  const float* A_log;
  const float* dt_bias;
  float eps, q_scale;
  float* state;
  uint8_t* buf;
  Layout L;
  int device;
  cudaStream_t compute, in, out;
  cudaEvent_t in_ready[2], in_free[2], computed[2], out_done[2];
  long long step;
};

extern "C" {

size_t gdn_decode_pipe_buffer_size(const gdn_dims* dims, int32_t n_seqs, int32_t x_dtype,
                                   int32_t o_dtype) {
  Layout L;
  return layout_of(dims, n_seqs, x_dtype, o_dtype, &L) ? L.total : 0;
}

int gdn_decode_pipe_destroy(gdn_decode_pipe* pipe) {
  if (!pipe) return GDN_OK;
  int rc = GDN_OK;
  int cur = 0;
  const bool switched = cudaGetDevice(&cur) == cudaSuccess && cur != pipe->device &&
                        cudaSetDevice(pipe->device) == cudaSuccess;
  // the copies may still be reading or writing host memory and the staging sets
  if (pipe->in && cudaStreamSynchronize(pipe->in) != cudaSuccess) rc = GDN_ECUDA;
  if (pipe->out && cudaStreamSynchronize(pipe->out) != cudaSuccess) rc = GDN_ECUDA;
  for (int j = 0; j < 2; ++j) {
    cudaEvent_t* evs[] = {&pipe->in_ready[j], &pipe->in_free[j], &pipe->computed[j],
                          &pipe->out_done[j]};
    for (cudaEvent_t* e : evs)
      if (*e && cudaEventDestroy(*e) != cudaSuccess) rc = GDN_ECUDA;
  }
  if (pipe->in && cudaStreamDestroy(pipe->in) != cudaSuccess) rc = GDN_ECUDA;
  if (pipe->out && cudaStreamDestroy(pipe->out) != cudaSuccess) rc = GDN_ECUDA;
  if (switched) cudaSetDevice(cur);
  delete pipe;
  return rc;
}

int gdn_decode_pipe_create(const gdn_dims* dims, int32_t n_seqs, int32_t x_dtype,
                           const float* conv_w, void* conv_state, int32_t conv_state_dtype,
                           const float* A_log, const float* dt_bias, float eps, float q_scale,
                           float* state, int32_t o_dtype, void* buffer, size_t buffer_bytes,
                           gdn_stream_t compute, gdn_decode_pipe** pipe) {
  if (!pipe) return GDN_EINVAL;
  *pipe = nullptr;
  Layout L;
  if (!layout_of(dims, n_seqs, x_dtype, o_dtype, &L)) return GDN_EINVAL;
  if (!A_log || !dt_bias || !state || !(eps >= 0.0f)) return GDN_EINVAL;
  if (!buffer || buffer_bytes < L.total) return GDN_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(buffer) & (kAlign - 1)) != 0) return GDN_EALIGN;
  gdn_decode_pipe* p = new (std::nothrow) gdn_decode_pipe{};
  if (!p) return GDN_ECUDA;
  p->dims = *dims;
  p->n = n_seqs; p->x_dtype = x_dtype; p->cs_dtype = conv_state_dtype; p->o_dtype = o_dtype;
  p->conv_w = conv_w; p->conv_state = conv_state; p->A_log = A_log; p->dt_bias = dt_bias;
  p->eps = eps; p->q_scale = q_scale; p->state = state;
  p->buf = static_cast<uint8_t*>(buffer);
  p->L = L;
  p->compute = reinterpret_cast<cudaStream_t>(compute);
  bool ok = cudaGetDevice(&p->device) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->out, cudaStreamNonBlocking) == cudaSuccess;
  for (int j = 0; ok && j < 2; ++j) {
    cudaEvent_t* evs[] = {&p->in_ready[j], &p->in_free[j], &p->computed[j], &p->out_done[j]};
    for (cudaEvent_t* e : evs)
      ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    gdn_decode_pipe_destroy(p);
    return GDN_ECUDA;
  }
  *pipe = p;
  return GDN_OK;
}

}  // extern "C"

namespace {

// One step: inputs from separate host arrays, or (packed) from one host row holding them at
// the staging set's offsets (x, a, b, slot_ids are then pointers into that row).
int pipe_step(gdn_decode_pipe* p, bool packed, const void* x, const float* a, const float* b,
              const int32_t* slot_ids, const uint8_t* reset, void* o) {
  const Layout& L = p->L;
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != p->device) return GDN_EINVAL;
  const int j = (int)(p->step & 1);
  uint8_t* set = p->buf + (size_t)j * L.set;
  // inputs: once step s - 2 has read this set
  if (cudaStreamWaitEvent(p->in, p->in_free[j], 0) != cudaSuccess) return GDN_ECUDA;
  // one copy per array (or one for the whole packed row)
  struct Copy { void* dst; const void* src; size_t n; } in[] = {
      {set + L.ox, x, packed ? L.os + L.slots : L.x}, {set + L.oa, a, packed ? 0 : L.a},
      {set + L.ob, b, packed ? 0 : L.b}, {set + L.os, slot_ids, packed ? 0 : L.slots},
      {set + L.orst, reset, reset ? L.reset : 0}};
  for (const Copy& c : in)
    if (c.n && cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, p->in) != cudaSuccess)
      return GDN_ECUDA;
  if (cudaEventRecord(p->in_ready[j], p->in) != cudaSuccess) return GDN_ECUDA;
  // the step: after its inputs, and after step s - 2's output has left this set
  if (cudaStreamWaitEvent(p->compute, p->in_ready[j], 0) != cudaSuccess ||
      cudaStreamWaitEvent(p->compute, p->out_done[j], 0) != cudaSuccess)
    return GDN_ECUDA;
  const int rc = gdn_layer_decode(
      &p->dims, set + L.ox, p->x_dtype, p->conv_w, p->conv_state, p->cs_dtype,
      reinterpret_cast<const int32_t*>(set + L.os),
      reset ? reinterpret_cast<const uint8_t*>(set + L.orst) : nullptr, p->n,
      reinterpret_cast<const float*>(set + L.oa),
      L.b ? reinterpret_cast<const float*>(set + L.ob) : nullptr, p->A_log, p->dt_bias, p->eps,
      p->q_scale, p->state, set + L.oo, p->o_dtype, p->buf + L.ws_off, L.ws, nullptr,
      reinterpret_cast<gdn_stream_t>(p->compute));
  if (rc != GDN_OK) return rc;
  if (cudaEventRecord(p->in_free[j], p->compute) != cudaSuccess ||
      cudaEventRecord(p->computed[j], p->compute) != cudaSuccess)
    return GDN_ECUDA;
  // output: once the step has written it
  if (cudaStreamWaitEvent(p->out, p->computed[j], 0) != cudaSuccess ||
      cudaMemcpyAsync(o, set + L.oo, L.o, cudaMemcpyDeviceToHost, p->out) != cudaSuccess ||
      cudaEventRecord(p->out_done[j], p->out) != cudaSuccess)
    return GDN_ECUDA;
  ++p->step;
  return GDN_OK;
}

}  // namespace

extern "C" {

size_t gdn_decode_pipe_packed_bytes(const gdn_dims* dims, int32_t n_seqs, int32_t x_dtype) {
  Layout L;
  return layout_of(dims, n_seqs, x_dtype, GDN_BF16, &L) ? L.os + L.slots : 0;
}

int gdn_decode_pipe_step(gdn_decode_pipe* p, const void* x, const float* a, const float* b,
                         const int32_t* slot_ids, const uint8_t* reset, void* o) {
  if (!p || !x || !a || !slot_ids || !o) return GDN_EINVAL;
  if ((p->L.b != 0) != (b != nullptr)) return GDN_EINVAL;
  return pipe_step(p, false, x, a, b, slot_ids, reset, o);
}

int gdn_decode_pipe_step_packed(gdn_decode_pipe* p, const void* in, const uint8_t* reset,
                                void* o) {
  if (!p || !in || !o) return GDN_EINVAL;
  const uint8_t* row = static_cast<const uint8_t*>(in);
  const Layout& L = p->L;
  return pipe_step(p, true, row + L.ox, reinterpret_cast<const float*>(row + L.oa),
                   L.b ? reinterpret_cast<const float*>(row + L.ob) : nullptr,
                   reinterpret_cast<const int32_t*>(row + L.os), reset, o);
}

int gdn_decode_pipe_flush(gdn_decode_pipe* p) {
  if (!p) return GDN_EINVAL;
  for (int j = 0; j < 2; ++j)
    if (cudaStreamWaitEvent(p->compute, p->out_done[j], 0) != cudaSuccess) return GDN_ECUDA;
  return GDN_OK;
}

}  // extern "C"
