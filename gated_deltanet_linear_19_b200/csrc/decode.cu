// Single-token gated delta-rule step (the autoregressive path).
// Pages: qwen3next.cpp build_delta_net_autoregressive: S <- exp(g) S; kv = S^T k;
// delta = beta (v - kv); S <- S + k delta^T; o = S^T q.
//
// One pass over the state: with S0 the stored state and e = exp(g),
//   r = S0^T k, y = S0^T q (both from the same loads), delta = beta (v - e r),
//   S = e S0 + k delta^T, o = S^T q = e y + delta (k.q).
// HBM-bound: every state byte is read once and written once with 16-byte streaming
// accesses. A CTA owns a 32-column tile of one (sequence, value head) state: 128 threads =
// 8 column quads x 16 row groups, each thread holding DK/16 rows x 4 columns in registers.
// Column sums are reduced with warp shuffles (rows 4 apart share a column quad) and then
// across the 4 warps through shared memory.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int DEC_THREADS = 128;
constexpr int DEC_TILE = 32;  // value columns per CTA

// Cluster helpers for the fused output gate: the column tiles of one (sequence, value head)
// form a thread-block cluster and exchange their partial sums of squares of o.
__device__ __forceinline__ void st_cluster_f32(float* local, uint32_t rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(local))), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int DK, typename TQ, typename TO, bool EARLY, bool GATE>
__global__ void __launch_bounds__(DEC_THREADS)
decode_kernel(const DecodeArgs p) {
  constexpr int RPT = DK / 16;  // rows per thread
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 7;        // column quad within the tile
  const int rg = tid >> 3;       // row group 0..15: rows rg + 16 m
  const int b = blockIdx.z, h = blockIdx.y, tile = blockIdx.x;
  const int hk = khead_of(h, p.H_k, p.H_v, p.layout);
  const int d_v = p.d_v;
  // The grid is launched with programmatic stream serialization, so it may start before the
  // kernel ahead of it on the stream has finished. Without EARLY (gdn_decode_step, whose
  // predecessor is unknown) nothing is read before waiting for that kernel. With EARLY
  // (gdn_layer_decode) the predecessor is this library's front kernel, which writes only
  // q, k, v, g, beta and the conv state and itself started after all earlier work on the
  // stream: slot ids, reset flags and the state may be read at once, so the state streaming
  // overlaps the front.
  if constexpr (!EARLY) asm volatile("griddepcontrol.wait;" ::: "memory");

  const int slot = p.slot_ids[b];
  if (slot < 0 || slot >= p.n_slots) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  const bool rst = p.reset != nullptr && p.reset[b] != 0;

  float* S = p.state + (((int64_t)slot * p.H_v + h) * DK) * d_v + tile * DEC_TILE + cq * 4;
  float4 s[RPT];
  if (!rst) {
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = ld4_stream(S + (int64_t)(rg + 16 * m) * d_v);
  } else {
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // a slot repeated within the call: only its first sequence updates it (checked while the
  // state loads are in flight; the loaded values of a skipped sequence are discarded)
  if (block_slot_taken(p.slot_ids, b, slot)) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  // q, k, v, g, beta come from the kernel launched just before this one (the front)
  if constexpr (EARLY) asm volatile("griddepcontrol.wait;" ::: "memory");
  const TQ* kp = static_cast<const TQ*>(p.k) + ((int64_t)b * p.H_k + hk) * DK;
  const TQ* qp = static_cast<const TQ*>(p.q) + ((int64_t)b * p.H_k + hk) * DK;
  float kr[RPT], qr[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) { kr[m] = ld(kp + rg + 16 * m); qr[m] = ld(qp + rg + 16 * m); }
  const float e = expf(p.g[(int64_t)b * p.H_v + h]);
  const float bt = p.beta[(int64_t)b * p.H_v + h];
  const float4 vv = ld4(static_cast<const TQ*>(p.v) + ((int64_t)b * p.H_v + h) * d_v +
                        tile * DEC_TILE + cq * 4);

  float acc[9];  // r[4], y[4], k.q
#pragma unroll
  for (int i = 0; i < 9; ++i) acc[i] = 0.f;
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    acc[0] = fmaf(s[m].x, kr[m], acc[0]); acc[1] = fmaf(s[m].y, kr[m], acc[1]);
    acc[2] = fmaf(s[m].z, kr[m], acc[2]); acc[3] = fmaf(s[m].w, kr[m], acc[3]);
    acc[4] = fmaf(s[m].x, qr[m], acc[4]); acc[5] = fmaf(s[m].y, qr[m], acc[5]);
    acc[6] = fmaf(s[m].z, qr[m], acc[6]); acc[7] = fmaf(s[m].w, qr[m], acc[7]);
    acc[8] = fmaf(kr[m], qr[m], acc[8]);
  }
  // lanes l, l^8, l^16, l^24 share a column quad
#pragma unroll
  for (int i = 0; i < 9; ++i) {
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
  }
  __shared__ float red[4][8][9];
  if (lane < 8) {
#pragma unroll
    for (int i = 0; i < 9; ++i) red[warp][lane][i] = acc[i];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 9; ++i)
    acc[i] = red[0][cq][i] + red[1][cq][i] + red[2][cq][i] + red[3][cq][i];

  const float kq = acc[8];
  float dl[4], o[4];
  dl[0] = bt * (vv.x - e * acc[0]); dl[1] = bt * (vv.y - e * acc[1]);
  dl[2] = bt * (vv.z - e * acc[2]); dl[3] = bt * (vv.w - e * acc[3]);
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = fmaf(e, acc[4 + i], dl[i] * kq);

#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    float4 n;
    n.x = fmaf(e, s[m].x, kr[m] * dl[0]);
    n.y = fmaf(e, s[m].y, kr[m] * dl[1]);
    n.z = fmaf(e, s[m].z, kr[m] * dl[2]);
    n.w = fmaf(e, s[m].w, kr[m] * dl[3]);
    st4_stream(S + (int64_t)(rg + 16 * m) * d_v, n);
  }
  if constexpr (GATE) {
    // output gate: RMS over the whole value head (all column tiles of the cluster), then
    // o * inv_rms * norm_w * SiLU(z). Threads 0..7 (warp 0, rg == 0) hold the tile's 32 outputs.
    __shared__ float part[4];
    const int ntiles = d_v / DEC_TILE;
    float ss = 0.f;
    if (rg == 0) ss = o[0] * o[0] + o[1] * o[1] + o[2] * o[2] + o[3] * o[3];
    if (warp == 0) {
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      if (lane == 0)
        for (int r = 0; r < ntiles; ++r) st_cluster_f32(&part[tile], (uint32_t)r, ss);
    }
    // every CTA of the cluster reaches this point (the exits above depend only on the
    // sequence, which the whole cluster shares), and none writes to another after it
    cluster_sync_all();
    if (rg == 0) {
      float tot = 0.f;
      for (int r = 0; r < ntiles; ++r) tot += part[r];
      const float inv = 1.0f / sqrtf(tot / (float)d_v + p.norm_eps);
      const int64_t off = ((int64_t)b * p.H_v + h) * d_v + tile * DEC_TILE + cq * 4;
      float zf[4];
      if (p.z_dtype == GDN_BF16) {
        const float4 z4 = ld4(static_cast<const __nv_bfloat16*>(p.z) + off);
        zf[0] = z4.x; zf[1] = z4.y; zf[2] = z4.z; zf[3] = z4.w;
      } else {
        const float4 z4 = ld4(static_cast<const float*>(p.z) + off);
        zf[0] = z4.x; zf[1] = z4.y; zf[2] = z4.z; zf[3] = z4.w;
      }
      const float4 w4 = ld4(p.norm_w + tile * DEC_TILE + cq * 4);
      const float wf[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = o[i] * inv * wf[i] * silu_exact(zf[i]);
    }
  }
  if (rg == 0) {
    TO* op = static_cast<TO*>(p.o) + ((int64_t)b * p.H_v + h) * d_v + tile * DEC_TILE + cq * 4;
    st4(op, make_float4(o[0], o[1], o[2], o[3]));
  }
}

template <int DK, typename TQ, bool EARLY>
cudaError_t launch_o(const DecodeArgs& a, cudaStream_t s, dim3 grid) {
  // Programmatic stream serialization: the grid may begin while the preceding kernel is
  // still running; the kernel waits for it before reading what that kernel may write. With
  // the output gate, the column tiles of a (sequence, value head) form one cluster.
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = grid.x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  const bool gate = a.z != nullptr;
  cfg.numAttrs = gate ? 2 : 1;
  if (a.o_dtype == GDN_BF16)
    return gate ? cudaLaunchKernelEx(&cfg, decode_kernel<DK, TQ, __nv_bfloat16, EARLY, true>, a)
                : cudaLaunchKernelEx(&cfg, decode_kernel<DK, TQ, __nv_bfloat16, EARLY, false>, a);
  return gate ? cudaLaunchKernelEx(&cfg, decode_kernel<DK, TQ, float, EARLY, true>, a)
              : cudaLaunchKernelEx(&cfg, decode_kernel<DK, TQ, float, EARLY, false>, a);
}

template <int DK, bool EARLY>
cudaError_t launch_q(const DecodeArgs& a, cudaStream_t s, dim3 grid) {
  switch (a.qkv_dtype) {
    case GDN_F32: return launch_o<DK, float, EARLY>(a, s, grid);
    case GDN_BF16: return launch_o<DK, __nv_bfloat16, EARLY>(a, s, grid);
    case GDN_F16: return launch_o<DK, __half, EARLY>(a, s, grid);
  }
  return cudaErrorInvalidValue;
}

template <bool EARLY>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t s, dim3 grid) {
  switch (a.d_k) {
    case 32: return launch_q<32, EARLY>(a, s, grid);
    case 64: return launch_q<64, EARLY>(a, s, grid);
    case 128: return launch_q<128, EARLY>(a, s, grid);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, bool after_front) {
  dim3 grid(a.d_v / DEC_TILE, a.H_v, a.n_seqs);
  return after_front ? launch_d<true>(a, s, grid) : launch_d<false>(a, s, grid);
}

}  // namespace gdn
