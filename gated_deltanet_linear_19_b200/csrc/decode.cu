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
// L2 prefetch of the state one wave ahead: each block asks L2 for the state bytes of the
// block that many places after it in launch order (the number of blocks resident at once),
// which deepens the stream's pipeline beyond the registers of the resident blocks. Used for
// grids of at least kPrefetchMinWaves waves (64 sequences at H_v = 32: 48.9 -> 45.7 us per
// layer step, 32 sequences 26.3 -> 24.1 us); a grid of under three waves measured slower with
// it (16 sequences: 14.0 against 14.5 us), its first wave's loads meeting the prefetches.
// Distances from 0.8 to 1.5 waves measured alike.
constexpr int kPrefetchMinWaves = 4;
// No register cap: at about 95 registers 5 blocks run per SM; capping for 6 or 7 blocks per SM
// spills and measured slower (64-sequence layer step: 47.7 us uncapped, 48.1 us for 6 blocks,
// 51.3 us for 7).

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

// The step on one thread's part of the tile, from the loaded state s (rows rg + 16 m, columns
// 4 cq .. 4 cq + 3), k and q at those rows, e = exp(g), beta and v at the columns: reduces
// S0^T k, S0^T q and k.q over the tile's rows (xor shuffles over the lanes of a column quad,
// then the 4 warps through shared memory), streams the new state to S and leaves
// o = e S0^T q + delta (k.q) for the columns in o (valid in every thread).
template <int RPT>
__device__ __forceinline__ void state_step(const float4 (&s)[RPT], const float (&kr)[RPT],
                                           const float (&qr)[RPT], float e, float bt,
                                           float4 vv, float* S, int d_v, float (&o)[4]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 7, rg = tid >> 3;
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
  float dl[4];
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
}

// Output gate, fused: RMS over the whole value head (all column tiles, which form a cluster
// whose ranks rank0 .. rank0 + ntiles - 1 are the tiles 0 .. ntiles - 1 of this value head),
// then o * inv_rms * norm_w * SiLU(z). Threads 0..7 (warp 0, rg == 0) hold the tile's 32
// outputs. Every CTA of the cluster must call it (it holds a cluster barrier).
__device__ __forceinline__ void out_gate(float (&o)[4], const DecodeArgs& p, int b, int h,
                                         int tile, uint32_t rank0) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 7, rg = tid >> 3;
  const int d_v = p.d_v;
  __shared__ float part[4];
  const int ntiles = d_v / DEC_TILE;
  float ss = 0.f;
  if (rg == 0) ss = o[0] * o[0] + o[1] * o[1] + o[2] * o[2] + o[3] * o[3];
  if (warp == 0) {
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    if (lane == 0)
      for (int r = 0; r < ntiles; ++r) st_cluster_f32(&part[tile], rank0 + (uint32_t)r, ss);
  }
  // none of the CTAs writes to another after this barrier
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

template <int DK, typename TQ, typename TO, bool EARLY>
__global__ void __launch_bounds__(DEC_THREADS)
decode_kernel(const DecodeArgs p) {
  constexpr int RPT = DK / 16;  // rows per thread
  const int tid = threadIdx.x;
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
  prefetch_state_ahead<DK>(p.state, p.slot_ids, p.n_slots, p.H_v, d_v, p.pf_dist);
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

  float o[4];
  state_step<RPT>(s, kr, qr, e, bt, vv, S, d_v, o);
  if (rg == 0) {
    TO* op = static_cast<TO*>(p.o) + ((int64_t)b * p.H_v + h) * d_v + tile * DEC_TILE + cq * 4;
    st4(op, make_float4(o[0], o[1], o[2], o[3]));
  }
}

template <typename Kern>
DecodeArgs with_prefetch(const DecodeArgs& a, Kern kern, dim3 grid) {
  DecodeArgs b = a;
  const int res = resident_blocks(kern, DEC_THREADS);
  const int64_t blocks = (int64_t)grid.x * grid.y * grid.z;
  b.pf_dist = (res > 0 && blocks >= (int64_t)kPrefetchMinWaves * res) ? res : 0;
  return b;
}

template <int DK, typename TQ, bool EARLY>
cudaError_t launch_o(const DecodeArgs& a, cudaStream_t s, dim3 grid) {
  // Programmatic stream serialization: the grid may begin while the preceding kernel is
  // still running; the kernel waits for it before reading what that kernel may write.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.o_dtype == GDN_BF16) {
    auto kern = decode_kernel<DK, TQ, __nv_bfloat16, EARLY>;
    return cudaLaunchKernelEx(&cfg, kern, with_prefetch(a, kern, grid));
  }
  auto kern = decode_kernel<DK, TQ, float, EARLY>;
  return cudaLaunchKernelEx(&cfg, kern, with_prefetch(a, kern, grid));
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


// ------------------------------------------------------------------ one-kernel layer decode
// gdn_layer_decode for d_k = d_v = 128, d_conv = 4 and H_v = r H_k with r = 1 or 2: the front
// of the step and the state step in one kernel. Each CTA computes the front values it needs
// (the key head's q and k, its tile's 32 v channels, the value head's gates) with the same
// arithmetic, in the same order, as the front kernel's decode path (a warp holds one head's
// 128 channels, 4 per lane, the L2 norm reduced with xor shuffles), so the result is bit for
// bit that of gdn_conv_step followed by gdn_decode_step. A cluster holds the 4 column tiles of
// the r value heads of one key head: every CTA of it reads the key head's q and k conv state,
// so that part of the roll waits for a cluster barrier (arrived at right after the reads,
// waited for after the state step) and is split over the cluster's CTAs; the tile's v channels
// are read and rewritten by their CTA alone.
// Pages: ik_llama.cpp src/llama-delta-net.cpp build_layer_attn_linear_core (conv, SiLU,
// L2 norm, conv-state write-back) and qwen3next.cpp build_delta_net_autoregressive.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

template <typename TX, typename TS, typename TO, bool GATE>
__global__ void __launch_bounds__(DEC_THREADS)
layer_decode_kernel(const DecodeArgs p, const FrontArgs f) {
  constexpr int DK = 128, RPT = DK / 16;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 7, rg = tid >> 3;
  const int r = p.H_v / p.H_k;  // value heads per key head: the cluster is 4 tiles x r heads
  const int tile = blockIdx.x, b = blockIdx.z;
  const int hk = blockIdx.y / r, jv = blockIdx.y - hk * r;
  const int h = (p.layout & GDN_GQA_TILED) ? hk + jv * p.H_k : hk * r + jv;
  const int d_v = DK;
  // everything this kernel reads may have been written by the kernel ahead of it
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next kernel on the stream may be scheduled now: every kernel of this library that is
  // launched programmatically waits for its predecessor before reading anything it may write
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // exits depend on the sequence only, so a cluster leaves as a whole
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
  if (block_slot_taken(p.slot_ids, b, slot)) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  const uint32_t crank = cluster_rank();
  if (crank != (uint32_t)(tile + 4 * jv) && tid == 0) set_status(p.status, GDN_ECUDA);

  // ---- front: warps 0 and 1 the key head's q and k (lane = 4 channels), warp 2 lanes 0-7
  // the tile's v channels, warp 3 lane 0 the gates; the conv window is [state rows; x]
  const int64_t conv_dim = (int64_t)(2 * p.H_k + p.H_v) * DK;
  TS* cst = static_cast<TS*>(f.conv_state) + (int64_t)slot * 3 * conv_dim;
  const TX* xrow = static_cast<const TX*>(f.x) + (int64_t)b * conv_dim;
  __shared__ float qk_s[2][DK];
  __shared__ float v_s[DEC_TILE];
  __shared__ float gb_s[2];
  const bool fr = warp < 2 || (warp == 2 && lane < 8);
  int64_t c0 = 0;
  if (warp < 2) c0 = (int64_t)warp * p.H_k * DK + (int64_t)hk * DK + lane * 4;
  else if (warp == 2) c0 = 2LL * p.H_k * DK + (int64_t)h * DK + tile * DEC_TILE + lane * 4;
  float win[3][4], xs[4], y[4];
  if (fr) {
    float wa[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 w4 = *reinterpret_cast<const float4*>(f.conv_w + (c0 + j) * 4);
      wa[j][0] = w4.x; wa[j][1] = w4.y; wa[j][2] = w4.z; wa[j][3] = w4.w;
    }
#pragma unroll
    for (int sl = 0; sl < 3; ++sl) {
      const float4 v = rst ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(cst + sl * conv_dim + c0);
      win[sl][0] = v.x; win[sl][1] = v.y; win[sl][2] = v.z; win[sl][3] = v.w;
    }
    const float4 x4 = ld4(xrow + c0);
    xs[0] = x4.x; xs[1] = x4.y; xs[2] = x4.z; xs[3] = x4.w;
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float acc = wa[j][0] * win[0][j];
      acc = fmaf(wa[j][1], win[1][j], acc);
      acc = fmaf(wa[j][2], win[2][j], acc);
      acc = fmaf(wa[j][3], xs[j], acc);
      y[j] = acc * sigmoidf_(acc);  // SiLU
      ss = fmaf(y[j], y[j], ss);
    }
    if (warp < 2) {
      float tot = ss;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
      const float mul = (warp == 0 ? f.q_scale : 1.0f) / sqrtf(tot + f.eps);
#pragma unroll
      for (int j = 0; j < 4; ++j) qk_s[warp][lane * 4 + j] = y[j] * mul;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v_s[lane * 4 + j] = y[j] * 1.0f;
    }
  } else if (warp == 3 && lane == 0) {
    const float z = gate_alpha(f.a, b, h, p.H_k, p.H_v, p.layout) + f.dt_bias[h];
    const float g = -expf(f.A_log[h]) * softplusf_(z);
    gb_s[0] = expf(g);
    gb_s[1] = sigmoidf_(gate_beta_logit(f.a, f.b, b, h, p.H_k, p.H_v, p.layout));
  }
  // this CTA has read the old conv state (the values are in registers)
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (warp == 2 && lane < 8) {
    // the tile's v channels: new rows = old rows 1, 2 and x (read by this CTA alone)
    st4(cst + c0, make_float4(win[1][0], win[1][1], win[1][2], win[1][3]));
    st4(cst + conv_dim + c0, make_float4(win[2][0], win[2][1], win[2][2], win[2][3]));
    st4(cst + 2 * conv_dim + c0, make_float4(xs[0], xs[1], xs[2], xs[3]));
  }
  __syncthreads();

  float kr[RPT], qr[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) { kr[m] = qk_s[1][rg + 16 * m]; qr[m] = qk_s[0][rg + 16 * m]; }
  const float e = gb_s[0], bt = gb_s[1];
  const float4 vv = make_float4(v_s[cq * 4], v_s[cq * 4 + 1], v_s[cq * 4 + 2], v_s[cq * 4 + 3]);
  float o[4];
  state_step<RPT>(s, kr, qr, e, bt, vv, S, d_v, o);

  // every CTA of the cluster has read the key head's old q / k conv state: roll it, each CTA
  // its 256 / (4 r) channels (held by the lanes that computed them)
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (warp < 2 && (warp * 32 + lane) / (16 / r) == (int)crank) {
    st4(cst + c0, make_float4(win[1][0], win[1][1], win[1][2], win[1][3]));
    st4(cst + conv_dim + c0, make_float4(win[2][0], win[2][1], win[2][2], win[2][3]));
    st4(cst + 2 * conv_dim + c0, make_float4(xs[0], xs[1], xs[2], xs[3]));
  }
  if constexpr (GATE) out_gate(o, p, b, h, tile, (uint32_t)(4 * jv));
  if (rg == 0) {
    TO* op = static_cast<TO*>(p.o) + ((int64_t)b * p.H_v + h) * d_v + tile * DEC_TILE + cq * 4;
    st4(op, make_float4(o[0], o[1], o[2], o[3]));
  }
}

template <typename TX, typename TS, typename TO>
cudaError_t launch_ld_o(const DecodeArgs& a, const FrontArgs& f, cudaStream_t s) {
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 4;
  attr[1].val.clusterDim.y = a.H_v / a.H_k;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4, a.H_v, a.n_seqs);
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (a.z != nullptr) return cudaLaunchKernelEx(&cfg, layer_decode_kernel<TX, TS, TO, true>, a, f);
  return cudaLaunchKernelEx(&cfg, layer_decode_kernel<TX, TS, TO, false>, a, f);
}

template <typename TX, typename TS>
cudaError_t launch_ld_s(const DecodeArgs& a, const FrontArgs& f, cudaStream_t s) {
  if (a.o_dtype == GDN_BF16) return launch_ld_o<TX, TS, __nv_bfloat16>(a, f, s);
  return launch_ld_o<TX, TS, float>(a, f, s);
}
}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, bool after_front) {
  dim3 grid(a.d_v / DEC_TILE, a.H_v, a.n_seqs);
  return after_front ? launch_d<true>(a, s, grid) : launch_d<false>(a, s, grid);
}

bool layer_decode_fused_supported(const DecodeArgs& a, const FrontArgs& f) {
  return a.d_k == 128 && a.d_v == 128 && f.d_conv == 4 &&
         (a.H_v == a.H_k || a.H_v == 2 * a.H_k);
}

bool layer_decode_fused_preferred(const DecodeArgs& a, const FrontArgs& f) {
  if (!layer_decode_fused_supported(a, f)) return false;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return false;
  // Measured per layer step (H_v = 32): one kernel 5.1 / 8.7 / 16.7 / 77 us and two kernels
  // 7.4 / 9.7 / 13.7 / 47.7 us at 4 / 8 / 16 / 64 sequences. The one-kernel grid finishes a
  // cluster's 8 CTAs together and recomputes a key head's q and k in each of them, which
  // costs more than the second launch once the grid is past about one and a half waves.
  return (int64_t)a.n_seqs * a.H_v * (a.d_v / DEC_TILE) <= 8LL * sms;
}

cudaError_t launch_layer_decode(const DecodeArgs& a, const FrontArgs& f, cudaStream_t s) {
  if (!layer_decode_fused_supported(a, f)) return cudaErrorNotSupported;
  if (f.x_dtype == GDN_BF16) {
    if (f.conv_state_dtype == GDN_BF16) return launch_ld_s<__nv_bfloat16, __nv_bfloat16>(a, f, s);
    return launch_ld_s<__nv_bfloat16, float>(a, f, s);
  }
  if (f.conv_state_dtype == GDN_BF16) return launch_ld_s<float, __nv_bfloat16>(a, f, s);
  return launch_ld_s<float, float>(a, f, s);
}

}  // namespace gdn
