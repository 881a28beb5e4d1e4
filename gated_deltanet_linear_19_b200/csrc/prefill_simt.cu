// Chunked gated delta rule in fp32 on the CUDA cores (the precise path: fp32 inputs,
// fp32 arithmetic end to end).
// Pages: qwen3next.cpp build_delta_net_chunking and the removed single-chunk path:
//   g_cum = cumsum(g) in the chunk; decay_ij = exp(g_cum_i - g_cum_j) for j <= i (masked
//   before exp); A = -(beta_i k_i.k_j decay_ij) for j < i; T = (I - A)^-1;
//   U = T (V*beta); W = T (K*beta*exp(g_cum)); P_ij = q_i.k_j decay_ij (j <= i);
//   v_new = U - W S; o = (Q*exp(g_cum)) S + P v_new; S = exp(g_last) S + (K*exp(g_last-g_cum))^T v_new.
// Differences from the pages' graph: T is never formed. (I - A)[W | U] = [K*beta*exp(g_cum) |
// V*beta] is solved by forward substitution in place, one thread per column, which needs no
// barrier between rows (each thread only reads rows it already finished) and costs about half
// of forming T and multiplying.
//
// Grid: (d_v / 32 column tiles, H_v, n_seqs); a CTA walks its sequence's chunks in order with
// its 128 x 32 state tile in shared memory. The S-independent part (A, P, the solve) is
// recomputed by each column tile; this kernel is the reference-precision path, the
// tensor-core kernel is the fast one.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int PS_THREADS = 256;
constexpr int PS_TILE = 32;
constexpr int CMAX = 64;

template <int DK>
struct SimtSmem {
  static constexpr int KP = DK + 4;             // padded row stride of K and Q
  static constexpr int WP = DK + PS_TILE + 4;   // [W | U] row stride
  static constexpr int VP = PS_TILE + 4;
  static size_t bytes(int C) {
    return sizeof(float) * ((size_t)C * KP * 2 + (size_t)C * WP + (size_t)C * C * 2 +
                            (size_t)C * VP + (size_t)DK * PS_TILE + 4 * (size_t)CMAX);
  }
};

template <int DK, typename TQ, typename TO>
__global__ void __launch_bounds__(PS_THREADS)
prefill_simt_kernel(const PrefillArgs p) {
  using SM = SimtSmem<DK>;
  constexpr int KP = SM::KP, WP = SM::WP, VP = SM::VP;
  const int C = p.chunk;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;                        // [C][KP]
  float* Qs = Ks + C * KP;               // [C][KP]
  float* WU = Qs + C * KP;               // [C][WP]  (W | U)
  float* Am = WU + C * WP;               // [C][C]
  float* Pm = Am + C * C;                // [C][C]
  float* Vn = Pm + C * C;                // [C][VP]  v_new
  float* Ss = Vn + C * VP;               // [DK][32] state tile
  float* gc = Ss + DK * PS_TILE;         // [CMAX] cumulative gate
  float* bt = gc + CMAX;                 // [CMAX] beta
  float* eg = bt + CMAX;                 // [CMAX] exp(g_cum)
  float* ed = eg + CMAX;                 // [CMAX] exp(g_last - g_cum)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int hk = khead_of(h, p.H_k, p.H_v, p.layout);
  const int d_v = p.d_v;

  const int64_t c0s = p.cu_seqlens[n], c1s = p.cu_seqlens[n + 1];
  if (c0s < 0 || c1s < c0s || c1s > p.T_total) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_EINVAL);
    return;
  }
  const int slot = p.slot_ids[n];
  if (slot < 0 || slot >= p.n_slots) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  // a slot repeated within the call: only its first sequence updates it
  if (block_slot_taken(p.slot_ids, n, slot)) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  const bool rst = p.reset != nullptr && p.reset[n] != 0;
  float* Sg = p.state + (((int64_t)slot * p.H_v + h) * DK) * d_v + tile * PS_TILE;

  for (int i = tid; i < DK * PS_TILE; i += PS_THREADS) {
    const int d = i / PS_TILE, j = i % PS_TILE;
    Ss[i] = rst ? 0.f : Sg[(int64_t)d * d_v + j];
  }

  const TQ* qg = static_cast<const TQ*>(p.q);
  const TQ* kg = static_cast<const TQ*>(p.k);
  const TQ* vg = static_cast<const TQ*>(p.v);
  TO* og = static_cast<TO*>(p.o);

  for (int64_t cs = c0s; cs < c1s; cs += C) {
    const int L = (int)((c1s - cs) < C ? (c1s - cs) : C);
    __syncthreads();  // previous chunk fully consumed
    // ---- load K, Q (zero rows beyond L), V tile, g, beta
    for (int i = tid; i < C * (DK / 4); i += PS_THREADS) {
      const int r = i / (DK / 4), c4 = (i % (DK / 4)) * 4;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), qv = kv;
      if (r < L) {
        const int64_t off = ((cs + r) * p.H_k + hk) * DK + c4;
        kv = ld4(kg + off);
        qv = ld4(qg + off);
      }
      *reinterpret_cast<float4*>(Ks + r * KP + c4) = kv;
      *reinterpret_cast<float4*>(Qs + r * KP + c4) = qv;
    }
    if (tid < CMAX) {
      float gv = 0.f, bv = 0.f;
      if (tid < L) {
        gv = fmaxf(p.g[(cs + tid) * p.H_v + h], kGateFloor);
        bv = p.beta[(cs + tid) * p.H_v + h];
      }
      gc[tid] = gv;
      bt[tid] = bv;
    }
    __syncthreads();
    // ---- g_cum (warp 0, two elements per lane, inclusive scan over CMAX)
    if (warp == 0) {
      float a0 = gc[2 * lane], a1 = gc[2 * lane + 1];
      float s = a0 + a1, incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const float excl = incl - s;
      gc[2 * lane] = excl + a0;
      gc[2 * lane + 1] = excl + a0 + a1;
    }
    __syncthreads();
    const float gl = gc[L - 1];
    if (tid < CMAX) {
      eg[tid] = expf(gc[tid]);
      ed[tid] = expf(gl - gc[tid]);
    }
    __syncthreads();
    // ---- right-hand sides: [K*beta*exp(g_cum) | V*beta]
    for (int i = tid; i < C * (DK + PS_TILE); i += PS_THREADS) {
      const int r = i / (DK + PS_TILE), c = i % (DK + PS_TILE);
      float val;
      if (c < DK) {
        val = Ks[r * KP + c] * bt[r] * eg[r];
      } else {
        val = 0.f;
        if (r < L) val = ld(vg + ((cs + r) * p.H_v + h) * d_v + tile * PS_TILE + (c - DK)) * bt[r];
      }
      WU[r * WP + c] = val;
    }
    // ---- A (strictly lower) and P (lower with diagonal); warp w owns rows w*C/8 ...
    {
      const int rpw = C / 8;
      for (int ii = 0; ii < rpw; ++ii) {
        const int i = warp * rpw + ii;
        for (int j = lane; j < C; j += 32) {
          float kk = 0.f, qk = 0.f;
          if (j <= i) {
            const float4* ki = reinterpret_cast<const float4*>(Ks + i * KP);
            const float4* qi = reinterpret_cast<const float4*>(Qs + i * KP);
            const float4* kj = reinterpret_cast<const float4*>(Ks + j * KP);
#pragma unroll 8
            for (int d4 = 0; d4 < DK / 4; ++d4) {
              const float4 a = ki[d4], q4 = qi[d4], c = kj[d4];
              kk = fmaf(a.x, c.x, kk); kk = fmaf(a.y, c.y, kk);
              kk = fmaf(a.z, c.z, kk); kk = fmaf(a.w, c.w, kk);
              qk = fmaf(q4.x, c.x, qk); qk = fmaf(q4.y, c.y, qk);
              qk = fmaf(q4.z, c.z, qk); qk = fmaf(q4.w, c.w, qk);
            }
          }
          float av = 0.f, pv = 0.f;
          if (j <= i) {
            const float dec = expf(gc[i] - gc[j]);  // only on the kept triangle
            pv = qk * dec;
            if (j < i) av = -bt[i] * kk * dec;
          }
          Am[i * C + j] = av;
          Pm[i * C + j] = pv;
        }
      }
    }
    __syncthreads();
    // ---- forward substitution: row i += sum_{j<i} A_ij row j, one thread per column
    if (tid < DK + PS_TILE) {
      const int c = tid;
      for (int i = 1; i < L; ++i) {
        float acc = WU[i * WP + c];
        for (int j = 0; j < i; ++j) acc = fmaf(Am[i * C + j], WU[j * WP + c], acc);
        WU[i * WP + c] = acc;
      }
    }
    __syncthreads();
    // ---- v_new = U - W S
    {
      const int jc = lane;
      for (int i = warp; i < C; i += PS_THREADS / 32) {
        float acc = 0.f;
        const float* wi = WU + i * WP;
#pragma unroll 8
        for (int d = 0; d < DK; ++d) acc = fmaf(wi[d], Ss[d * PS_TILE + jc], acc);
        Vn[i * VP + jc] = (i < L) ? (WU[i * WP + DK + jc] - acc) : 0.f;
      }
    }
    __syncthreads();
    // ---- o = (Q*exp(g_cum)) S + P v_new
    {
      const int jc = lane;
      for (int i = warp; i < L; i += PS_THREADS / 32) {
        float inter = 0.f, intra = 0.f;
        const float* qi = Qs + i * KP;
#pragma unroll 8
        for (int d = 0; d < DK; ++d) inter = fmaf(qi[d], Ss[d * PS_TILE + jc], inter);
        for (int m = 0; m <= i; ++m) intra = fmaf(Pm[i * C + m], Vn[m * VP + jc], intra);
        const float ov = fmaf(inter, eg[i], intra);
        st(og + ((cs + i) * p.H_v + h) * d_v + tile * PS_TILE + jc, ov);
      }
    }
    __syncthreads();
    // ---- S = exp(g_last) S + (K*exp(g_last - g_cum))^T v_new
    {
      const int jc = lane;
      const float el = expf(gl);
      for (int d = warp; d < DK; d += PS_THREADS / 32) {
        float acc = 0.f;
        for (int m = 0; m < L; ++m) acc = fmaf(Ks[m * KP + d] * ed[m], Vn[m * VP + jc], acc);
        Ss[d * PS_TILE + jc] = fmaf(Ss[d * PS_TILE + jc], el, acc);
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < DK * PS_TILE; i += PS_THREADS) {
    const int d = i / PS_TILE, j = i % PS_TILE;
    Sg[(int64_t)d * d_v + j] = Ss[i];
  }
}

template <int DK, typename TQ>
cudaError_t launch_o(const PrefillArgs& a, cudaStream_t s, dim3 grid, size_t smem) {
  if (a.o_dtype == GDN_BF16) {
    auto k = prefill_simt_kernel<DK, TQ, __nv_bfloat16>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, PS_THREADS, smem, s>>>(a);
  } else {
    auto k = prefill_simt_kernel<DK, TQ, float>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, PS_THREADS, smem, s>>>(a);
  }
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_q(const PrefillArgs& a, cudaStream_t s) {
  dim3 grid(a.d_v / PS_TILE, a.H_v, a.n_seqs);
  const size_t smem = SimtSmem<DK>::bytes(a.chunk);
  switch (a.qkv_dtype) {
    case GDN_F32: return launch_o<DK, float>(a, s, grid, smem);
    case GDN_BF16: return launch_o<DK, __nv_bfloat16>(a, s, grid, smem);
    case GDN_F16: return launch_o<DK, __half>(a, s, grid, smem);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s) {
  switch (a.d_k) {
    case 32: return launch_q<32>(a, s);
    case 64: return launch_q<64>(a, s);
    case 128: return launch_q<128>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdn
