// Short sequences of a layer prefill (gdn_layer_prefill): sequences of at most max_len tokens
// (decode tokens, speculative or multi-token steps in a mixed batch) run the whole layer in one
// kernel, the front computed inside and the state kept in registers across the sequence's
// tokens; the chunked kernels of the same call take the longer sequences.
// Pages: ik_llama.cpp src/llama-delta-net.cpp build_layer_attn_linear_core (conv over
// [conv state; x], SiLU, L2 norm, conv-state write-back) and qwen3next.cpp
// build_delta_net_autoregressive (the per-token step), applied token after token;
// build_layer_attn_linear sends every sequence of more than one token to the chunked path,
// where short ones pay the chunk set-up.
//
// CTA = (32-column tile, value head, sequence), 128 threads; a cluster holds the 4 column tiles
// of the r = H_v / H_k value heads of one key head. Each CTA computes, for every token of its
// sequence, the key head's q and k (warps 0 and 1, a warp per head, 4 channels per lane, the
// L2 norm reduced with xor shuffles), its tile's 32 v channels (warp 2, lanes 0-7) and the
// value head's gates (warp 3), all in fp32, into shared memory; then it runs the decode step's
// one-pass form token after token (S read once, written once). After the tokens the conv
// window in each lane's registers holds the last d_conv - 1 rows of [conv state; x], the new
// conv state: the tile's v channels are written by their CTA (no other reads them), the key
// head's q and k channels, which every CTA of the cluster reads, after a cluster barrier and
// split over the cluster's CTAs.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int LS_THREADS = 128;
constexpr int LS_TILE = 32;
constexpr int LS_MAX = 16;  // tokens per sequence, at most

__device__ __forceinline__ uint32_t ls_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

template <typename TO>
__global__ void __launch_bounds__(LS_THREADS)
layer_short_kernel(const PrefillArgs p, int max_len) {
  constexpr int DK = 128, RPT = DK / 16;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 7, rg = tid >> 3;
  const int r = p.H_v / p.H_k;
  const int tile = blockIdx.x, n = blockIdx.z;
  const int hk = blockIdx.y / r, jv = blockIdx.y - hk * r;
  const int h = (p.layout & GDN_GQA_TILED) ? hk + jv * p.H_k : hk * r + jv;
  const int d_v = DK;
  const bool lead = tid == 0 && blockIdx.x == 0 && blockIdx.y == 0;

  // every exit below depends on the sequence only, so a cluster leaves as a whole
  const int64_t c0 = p.cu_seqlens[n], c1 = p.cu_seqlens[n + 1];
  if (c0 < 0 || c1 < c0 || c1 > p.T_total) {
    if (lead) set_status(p.status, GDN_EINVAL);
    return;
  }
  const int L = (int)(c1 - c0);
  if (L > max_len || L > LS_MAX) {
    // the chunked kernels of the same call take it; with GDN_PREFILL_RECURRENT (only short
    // sequences promised) there are none: an error
    if ((p.flags & GDN_PREFILL_RECURRENT) && lead) set_status(p.status, GDN_EINVAL);
    return;
  }
  const int slot = p.slot_ids[n];
  if (slot < 0 || slot >= p.n_slots) {
    if (lead) set_status(p.status, GDN_ESLOT);
    return;
  }
  if (block_slot_taken(p.slot_ids, n, slot)) {
    if (lead) set_status(p.status, GDN_ESLOT);
    return;
  }
  const bool rst = p.reset != nullptr && p.reset[n] != 0;
  float* S = p.state + (((int64_t)slot * p.H_v + h) * DK) * d_v + tile * LS_TILE + cq * 4;
  float4 s[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m)
    s[m] = rst ? make_float4(0.f, 0.f, 0.f, 0.f)
               : *reinterpret_cast<const float4*>(S + (int64_t)(rg + 16 * m) * d_v);

  // ---- front of the L tokens
  __shared__ __align__(16) float qk_s[LS_MAX][2][DK];
  __shared__ __align__(16) float v_s[LS_MAX][LS_TILE];
  __shared__ float e_s[LS_MAX], b_s[LS_MAX];
  const int64_t conv_dim = (int64_t)(2 * p.H_k + p.H_v) * DK;
  __nv_bfloat16* cst = static_cast<__nv_bfloat16*>(p.conv_state) + (int64_t)slot * 3 * conv_dim;
  const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
  const bool fr = warp < 2 || (warp == 2 && lane < 8);
  int64_t ch = 0;
  if (warp < 2) ch = (int64_t)warp * p.H_k * DK + (int64_t)hk * DK + lane * 4;
  else if (warp == 2) ch = 2LL * p.H_k * DK + (int64_t)h * DK + tile * LS_TILE + lane * 4;
  float win[3][4];  // the conv window: the last 3 rows of [conv state; x] seen so far
  if (fr) {
    float wa[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 w4 = *reinterpret_cast<const float4*>(p.conv_w + (ch + j) * 4);
      wa[j][0] = w4.x; wa[j][1] = w4.y; wa[j][2] = w4.z; wa[j][3] = w4.w;
    }
#pragma unroll
    for (int sl = 0; sl < 3; ++sl) {
      const float4 v = rst ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(cst + sl * conv_dim + ch);
      win[sl][0] = v.x; win[sl][1] = v.y; win[sl][2] = v.z; win[sl][3] = v.w;
    }
    for (int t = 0; t < L; ++t) {
      const float4 x4 = ld4(xg + (c0 + t) * conv_dim + ch);
      const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
      float y[4], ss = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float acc = wa[j][0] * win[0][j];
        acc = fmaf(wa[j][1], win[1][j], acc);
        acc = fmaf(wa[j][2], win[2][j], acc);
        acc = fmaf(wa[j][3], xs[j], acc);
        y[j] = acc * sigmoidf_(acc);  // SiLU
        ss = fmaf(y[j], y[j], ss);
        win[0][j] = win[1][j];
        win[1][j] = win[2][j];
        win[2][j] = xs[j];
      }
      if (warp < 2) {
        float tot = ss;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        const float mul = (warp == 0 ? p.q_scale : 1.0f) / sqrtf(tot + p.eps);
#pragma unroll
        for (int j = 0; j < 4; ++j) qk_s[t][warp][lane * 4 + j] = y[j] * mul;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) v_s[t][lane * 4 + j] = y[j];
      }
    }
  } else if (warp == 3 && lane < L) {
    const int64_t t = c0 + lane;
    const float z = gate_alpha(p.fa, t, h, p.H_k, p.H_v, p.layout) + p.dt_bias[h];
    e_s[lane] = expf(-expf(p.A_log[h]) * softplusf_(z));
    b_s[lane] = sigmoidf_(gate_beta_logit(p.fa, p.fb, t, h, p.H_k, p.H_v, p.layout));
  }
  // this CTA has read the old conv state (the values are in registers)
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (warp == 2 && lane < 8) {
    // the tile's v channels: read by this CTA alone
#pragma unroll
    for (int sl = 0; sl < 3; ++sl)
      st4(cst + sl * conv_dim + ch, make_float4(win[sl][0], win[sl][1], win[sl][2], win[sl][3]));
  }
  __syncthreads();

  // ---- the step, token after token (column sums double-buffered by token parity)
  __shared__ float red[2][4][8][9];
  for (int t = 0; t < L; ++t) {
    const int buf = t & 1;
    float kr[RPT], qr[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) { kr[m] = qk_s[t][1][rg + 16 * m]; qr[m] = qk_s[t][0][rg + 16 * m]; }
    const float e = e_s[t], bt = b_s[t];
    const float4 vv = *reinterpret_cast<const float4*>(&v_s[t][cq * 4]);
    float acc[9];  // S^T k [4], S^T q [4], k.q
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
#pragma unroll
    for (int i = 0; i < 9; ++i) {
      acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
      acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
    }
    if (lane < 8) {
#pragma unroll
      for (int i = 0; i < 9; ++i) red[buf][warp][lane][i] = acc[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 9; ++i)
      acc[i] = red[buf][0][cq][i] + red[buf][1][cq][i] + red[buf][2][cq][i] + red[buf][3][cq][i];
    const float kq = acc[8];
    float dl[4], o[4];
    dl[0] = bt * (vv.x - e * acc[0]); dl[1] = bt * (vv.y - e * acc[1]);
    dl[2] = bt * (vv.z - e * acc[2]); dl[3] = bt * (vv.w - e * acc[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = fmaf(e, acc[4 + i], dl[i] * kq);
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
      s[m].x = fmaf(e, s[m].x, kr[m] * dl[0]);
      s[m].y = fmaf(e, s[m].y, kr[m] * dl[1]);
      s[m].z = fmaf(e, s[m].z, kr[m] * dl[2]);
      s[m].w = fmaf(e, s[m].w, kr[m] * dl[3]);
    }
    if (rg == 0) {
      TO* op = static_cast<TO*>(p.o) + ((c0 + t) * p.H_v + h) * d_v + tile * LS_TILE + cq * 4;
      st4(op, make_float4(o[0], o[1], o[2], o[3]));
    }
  }
#pragma unroll
  for (int m = 0; m < RPT; ++m) *reinterpret_cast<float4*>(S + (int64_t)(rg + 16 * m) * d_v) = s[m];

  // every CTA of the cluster has read the key head's old q / k conv state: roll it, each CTA
  // its 256 / (4 r) channels (held by the lanes that computed them)
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  const int crank = (int)ls_cluster_rank();
  if (warp < 2 && (warp * 32 + lane) / (16 / r) == crank) {
#pragma unroll
    for (int sl = 0; sl < 3; ++sl)
      st4(cst + sl * conv_dim + ch, make_float4(win[sl][0], win[sl][1], win[sl][2], win[sl][3]));
  }
}

}  // namespace

bool layer_short_supported(const PrefillArgs& a) {
  return a.fused && a.d_k == 128 && a.d_v == 128 && (a.H_v == a.H_k || a.H_v == 2 * a.H_k);
}

cudaError_t launch_layer_short(const PrefillArgs& a, int max_len, cudaStream_t s) {
  if (!layer_short_supported(a) || max_len > LS_MAX) return cudaErrorNotSupported;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 4;
  attr[0].val.clusterDim.y = a.H_v / a.H_k;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4, a.H_v, a.n_seqs);
  cfg.blockDim = dim3(LS_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.o_dtype == GDN_BF16)
    return cudaLaunchKernelEx(&cfg, layer_short_kernel<__nv_bfloat16>, a, max_len);
  return cudaLaunchKernelEx(&cfg, layer_short_kernel<float>, a, max_len);
}

}  // namespace gdn
