// Token-by-token gated delta rule for short packed sequences (a few tokens each: speculative
// or multi-token decode steps), with the state held in registers across the sequence's tokens.
// Pages: qwen3next.cpp build_delta_net_autoregressive (the per-token step
// S <- exp(g) S; kv = S^T k; delta = beta (v - kv); S <- S + k delta^T; o = S^T q), applied
// token after token, where build_layer_attn_linear sends every sequence of more than one token
// to the chunked path; here short sequences skip the chunk set-up.
//
// Per token, with e = exp(g): r = S^T k and y = S^T q from the same registers,
// delta = beta (v - e r), S <- e S + k delta^T, o = e y + delta (k.q), exactly the decode
// step's one-pass form. The state tile is read once and written once per call, not once per
// token. A CTA owns a 32-column tile of one (sequence, value head) state: 128 threads = 8
// column quads x 16 row groups, DK/16 rows x 4 columns each in registers; column sums are
// reduced with shuffles and then across the 4 warps through shared memory (added once per
// token by 72 threads). The tokens' q, k, v, g and beta (at most RC_MAXT tokens) are staged
// in shared memory up front (q and k rows permuted so that a thread's rows load as vectors),
// so no global load sits inside the token loop. fp32 arithmetic throughout; the column sums
// and the state update as packed fp32 pairs (per lane the scalar operations).
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int RC_THREADS = 128;
constexpr int RC_TILE = 32;
constexpr int RC_MAXT = 16;  // tokens staged in shared memory at once

template <int DK, typename TQ, typename TO>
__global__ void __launch_bounds__(RC_THREADS)
recurrent_kernel(const PrefillArgs p, int max_len) {
  constexpr int RPT = DK / 16;  // rows per thread
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid & 7, rg = tid >> 3;
  const int tile = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int hk = khead_of(h, p.H_k, p.H_v, p.layout);
  const int d_v = p.d_v;
  const bool lead = tid == 0 && h == 0 && tile == 0;

  const int64_t c0 = p.cu_seqlens[n], c1 = p.cu_seqlens[n + 1];
  if (c0 < 0 || c1 < c0 || c1 > p.T_total) {
    if (lead) set_status(p.status, GDN_EINVAL);
    return;
  }
  // sequences longer than max_len belong to the chunked kernels of the same call (with
  // compact rows and GDN_PREFILL_RECURRENT, a layer prefill promised none: an error)
  if (max_len > 0 && c1 - c0 > max_len) {
    if (p.compact_rows > 0 && (p.flags & GDN_PREFILL_RECURRENT) && lead)
      set_status(p.status, GDN_EINVAL);
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
  float* S = p.state + (((int64_t)slot * p.H_v + h) * DK) * d_v + tile * RC_TILE + cq * 4;
  float4 s[RPT];
  if (!rst) {
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = *reinterpret_cast<const float4*>(S + (int64_t)(rg + 16 * m) * d_v);
  } else {
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  __shared__ float red[2][4][8][9];
  __shared__ __align__(16) float tot[8][12];  // the 4 warps' partials summed (9 of 12 used)
  __shared__ __align__(16) float qk_s[RC_MAXT][2][DK];
  __shared__ __align__(16) float v_s[RC_MAXT][RC_TILE];
  __shared__ float e_s[RC_MAXT], b_s[RC_MAXT];
  const TQ* qg = static_cast<const TQ*>(p.q);
  const TQ* kg = static_cast<const TQ*>(p.k);
  const TQ* vg = static_cast<const TQ*>(p.v);
  // row of the sequence's first token in q, k, v, g, beta
  const int64_t irow0 = p.compact_rows > 0 ? (int64_t)n * p.compact_rows : c0;
  for (int64_t tb = c0; tb < c1; tb += RC_MAXT) {
    const int nt = (int)(c1 - tb < RC_MAXT ? c1 - tb : RC_MAXT);
    const int64_t rb = irow0 + (tb - c0);
    __syncthreads();  // the previous group's values are no longer read
    for (int e = tid; e < nt * 2 * DK; e += RC_THREADS) {
      const int t = e / (2 * DK), w = (e / DK) & 1, d = e % DK;
      const TQ* src = w ? kg : qg;
      // row d at (d % 16) * RPT + d / 16: thread rg's rows rg + 16 m are consecutive
      qk_s[t][w][(d & 15) * RPT + (d >> 4)] = ld(src + ((rb + t) * p.H_k + hk) * DK + d);
    }
    for (int e = tid; e < nt * RC_TILE; e += RC_THREADS) {
      const int t = e / RC_TILE, c = e % RC_TILE;
      v_s[t][c] = ld(vg + ((rb + t) * p.H_v + h) * d_v + tile * RC_TILE + c);
    }
    if (tid < nt) {
      e_s[tid] = expf(p.g[(rb + tid) * p.H_v + h]);
      b_s[tid] = p.beta[(rb + tid) * p.H_v + h];
    }
    __syncthreads();
    for (int j = 0; j < nt; ++j) {
      const int64_t t = tb + j;
      const int buf = (int)((t - c0) & 1);
      float kr[RPT], qr[RPT];
#pragma unroll
      for (int m = 0; m < RPT; ++m) { kr[m] = qk_s[j][1][rg * RPT + m]; qr[m] = qk_s[j][0][rg * RPT + m]; }
      const float e = e_s[j];
      const float bt = b_s[j];
      const float4 vv = *reinterpret_cast<const float4*>(&v_s[j][cq * 4]);

      float acc[9];  // r[4], y[4], k.q
      {
        // column pairs (x, y) and (z, w) with packed fp32 FMAs: per lane the same operations
        // in the same order as one fmaf per column
        float2 a01 = make_float2(0.f, 0.f), a23 = a01, a45 = a01, a67 = a01;
        float a8 = 0.f;
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
          const float2 k2 = make_float2(kr[m], kr[m]), q2 = make_float2(qr[m], qr[m]);
          const float2 sxy = make_float2(s[m].x, s[m].y), szw = make_float2(s[m].z, s[m].w);
          a01 = fma2(sxy, k2, a01); a23 = fma2(szw, k2, a23);
          a45 = fma2(sxy, q2, a45); a67 = fma2(szw, q2, a67);
          a8 = fmaf(kr[m], qr[m], a8);
        }
        acc[0] = a01.x; acc[1] = a01.y; acc[2] = a23.x; acc[3] = a23.y;
        acc[4] = a45.x; acc[5] = a45.y; acc[6] = a67.x; acc[7] = a67.y; acc[8] = a8;
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
      // the 72 sums (8 column quads x 9) once, by 72 threads, in warp order; then each thread
      // reads its quad's 9 (the next token's first barrier orders these reads before tot is
      // written again)
      if (tid < 72) {
        const int q = tid / 9, i = tid - 9 * (tid / 9);
        tot[q][i] = red[buf][0][q][i] + red[buf][1][q][i] + red[buf][2][q][i] + red[buf][3][q][i];
      }
      __syncthreads();
      {
        const float4 t0 = *reinterpret_cast<const float4*>(&tot[cq][0]);
        const float4 t1 = *reinterpret_cast<const float4*>(&tot[cq][4]);
        acc[0] = t0.x; acc[1] = t0.y; acc[2] = t0.z; acc[3] = t0.w;
        acc[4] = t1.x; acc[5] = t1.y; acc[6] = t1.z; acc[7] = t1.w;
        acc[8] = tot[cq][8];
      }
      const float kq = acc[8];
      float dl[4], o[4];
      dl[0] = bt * (vv.x - e * acc[0]); dl[1] = bt * (vv.y - e * acc[1]);
      dl[2] = bt * (vv.z - e * acc[2]); dl[3] = bt * (vv.w - e * acc[3]);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = fmaf(e, acc[4 + i], dl[i] * kq);
      {
        const float2 e2 = make_float2(e, e);
        const float2 d01 = make_float2(dl[0], dl[1]), d23 = make_float2(dl[2], dl[3]);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
          const float2 k2 = make_float2(kr[m], kr[m]);
          const float2 xy = fma2(e2, make_float2(s[m].x, s[m].y), mul2(k2, d01));
          const float2 zw = fma2(e2, make_float2(s[m].z, s[m].w), mul2(k2, d23));
          s[m] = make_float4(xy.x, xy.y, zw.x, zw.y);
        }
      }
      if (rg == 0) {
        TO* op = static_cast<TO*>(p.o) + (t * p.H_v + h) * d_v + tile * RC_TILE + cq * 4;
        st4(op, make_float4(o[0], o[1], o[2], o[3]));
      }
    }
  }
#pragma unroll
  for (int m = 0; m < RPT; ++m) *reinterpret_cast<float4*>(S + (int64_t)(rg + 16 * m) * d_v) = s[m];
}

template <int DK, typename TQ>
cudaError_t launch_o(const PrefillArgs& a, int max_len, cudaStream_t s, dim3 grid) {
  if (a.o_dtype == GDN_BF16)
    recurrent_kernel<DK, TQ, __nv_bfloat16><<<grid, RC_THREADS, 0, s>>>(a, max_len);
  else
    recurrent_kernel<DK, TQ, float><<<grid, RC_THREADS, 0, s>>>(a, max_len);
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_q(const PrefillArgs& a, int max_len, cudaStream_t s, dim3 grid) {
  switch (a.qkv_dtype) {
    case GDN_F32: return launch_o<DK, float>(a, max_len, s, grid);
    case GDN_BF16: return launch_o<DK, __nv_bfloat16>(a, max_len, s, grid);
    case GDN_F16: return launch_o<DK, __half>(a, max_len, s, grid);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_recurrent(const PrefillArgs& a, int max_len, cudaStream_t s) {
  dim3 grid(a.d_v / RC_TILE, a.H_v, a.n_seqs);
  switch (a.d_k) {
    case 32: return launch_q<32>(a, max_len, s, grid);
    case 64: return launch_q<64>(a, max_len, s, grid);
    case 128: return launch_q<128>(a, max_len, s, grid);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdn
