// Chunked gated delta rule on the 5th-generation tensor cores (tcgen05, TMEM accumulators),
// for d_k = d_v = 128, chunk 64, fp16 q/k/v (the Qwen3-Next layer shape).
// Pages: qwen3next.cpp build_delta_net_chunking and the removed single-chunk path (the
// per-chunk math), chunk size 64 as QWEN3NEXT_CHUNK_SIZE in ik_llama.cpp.
//
// Two kernels:
//  1. tc_prep_kernel, one CTA per (chunk, value head), fully parallel. Everything that does
//     not depend on the recurrent state:
//       g_cum, decay_ij = exp(g_cum_i - g_cum_j) (masked before exp),
//       [K; Q] K^T as ONE M=128 MMA (rows 0-63: K K^T, rows 64-127: Q K^T),
//       L = beta_i (k_i.k_j) decay_ij (j < i), P = (q_i.k_j) decay_ij (j <= i),
//       T = (I + L)^-1 by a blocked 16x16 inversion on the CUDA cores,
//       W^T = (K*beta*exp(g_cum))^T T^T and U^T = (V*beta)^T T^T as M=128 MMAs.
//     The pages' attn = -(beta K K^T * decay) and T = (I - attn)^-1 are the same matrices.
//     W and P are written to the workspace already in the scan kernel's operand layout.
//  2. tc_scan_kernel, one CTA per (sequence, value head, 32-column d_v tile), sequential
//     over the sequence's chunks. Warps 0-3 own the fp32 state tile S[128 x 32] in registers
//     (thread i = row i = TMEM lane i) and run the chain
//       D1 = [W; Q*exp(g_cum)] S                      (M=128, N=32, K=128)
//       v_new = U - D1[0:64]
//       D2 = (K*exp(g_last - g_cum))^T v_new           (M=128, N=32, K=64)
//       D1[64:128] += P v_new                          (M=128, N=32, K=64; rows 0-63 unused)
//       S = exp(g_last) S + D2 ;  o = D1[64:128]
//     while warps 4-7 prefetch the next chunk (bulk copies of W and P, scaled Q and K,
//     the U tile) into the other of two shared-memory stages.
// Every wait is time-bounded; on a time-out the kernel records GDN_ETIMEOUT, stops issuing
// work, drains what it issued and frees its TMEM.
#include <mutex>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "umma.cuh"

namespace gdn {
namespace {

using namespace umma;

constexpr int C = 64;      // chunk
constexpr int D = 128;     // d_k = d_v
constexpr int TILE = 32;   // d_v columns per scan CTA

// workspace record per (chunk, value head)
constexpr int REC_W = 0;        // W [64 x 128] fp16, K-major canonical (LBO 128, SBO 2048)
constexpr int REC_U = 16384;    // U [64][128] fp16 row-major
constexpr int REC_P = 32768;    // P [64 x 64] fp16, K-major canonical (LBO 128, SBO 1024)
constexpr int REC_G = 40960;    // g_cum [64] fp32
constexpr int REC_BYTES = 41216;

__device__ __forceinline__ uint4 ld16(const __half* p) { return *reinterpret_cast<const uint4*>(p); }

__device__ __forceinline__ uint4 scale8(uint4 v, float s) {
  __half2* h = reinterpret_cast<__half2*>(&v);
  uint4 out;
  __half2* o = reinterpret_cast<__half2*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    o[i] = __floats2half2_rn(f.x * s, f.y * s);
  }
  return out;
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 out;
  __half2* o = reinterpret_cast<__half2*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return out;
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" : : "r"(id), "r"(n) : "memory");
}

// ======================================================================== prep kernel
constexpr int PREP_THREADS = 128;
constexpr int LDS = 65;  // fp32 row stride of L and T
// shared memory map (bytes)
constexpr int SM_AQK = 0;                 // 32768 [K; Q] K-major, later W / U staging
constexpr int SM_XW = 32768;              // 16384 (K*beta*exp(gc)) MN-major (M=d, K=token)
constexpr int SM_XU = 49152;              // 16384 (V*beta) MN-major
constexpr int SM_TB = 65536;              // 8192  T as K-major B (N = i, K = j)
constexpr int SM_LF = 73728;              // 64*65*4 = 16640
constexpr int SM_TF = SM_LF + 16640;      // 16640
constexpr int SM_XT = SM_TF + 16640;      // 3 * 256 * 4 = 3072
constexpr int SM_GC = SM_XT + 3072;       // 64 floats
constexpr int SM_BT = SM_GC + 256;
constexpr int SM_EG = SM_BT + 256;
constexpr int PREP_SMEM = SM_EG + 256;    // ~127 KB

// T = (I + L)^-1 for a strictly lower-triangular 64 x 64 L (fp32, row stride LDS).
// Diagonal 16 x 16 blocks by forward substitution (one warp per block, one lane per column),
// then off-diagonal blocks level by level: T_ab = -T_aa sum_{m=b}^{a-1} L_am T_mb.
__device__ void tri_inverse_64(const float* Lf, float* Tf, float* Xt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  {
    const int b = warp, c = lane;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m) acc = fmaf(Lf[(16 * b + i) * LDS + 16 * b + m], t[m], acc);
      t[i] = (i == c) ? 1.f : (i > c ? -acc : 0.f);
    }
    if (c < 16) {
#pragma unroll
      for (int i = 0; i < 16; ++i) Tf[(16 * b + i) * LDS + 16 * b + c] = t[i];
    }
  }
  __syncthreads();
  for (int lvl = 1; lvl < 4; ++lvl) {
    const int nb = 4 - lvl;
    for (int e = tid; e < nb * 256; e += PREP_THREADS) {
      const int b = e >> 8, i = (e >> 4) & 15, j = e & 15, a = b + lvl;
      float acc = 0.f;
      for (int m = 16 * b; m < 16 * a; ++m)
        acc = fmaf(Lf[(16 * a + i) * LDS + m], Tf[m * LDS + 16 * b + j], acc);
      Xt[e] = acc;
    }
    __syncthreads();
    for (int e = tid; e < nb * 256; e += PREP_THREADS) {
      const int b = e >> 8, i = (e >> 4) & 15, j = e & 15, a = b + lvl;
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m)
        acc = fmaf(Tf[(16 * a + i) * LDS + 16 * a + m], Xt[(b << 8) + m * 16 + j], acc);
      Tf[(16 * a + i) * LDS + 16 * b + j] = -acc;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(PREP_THREADS)
tc_prep_kernel(const PrefillArgs p, uint8_t* ws, int64_t max_chunks) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t bar[2];
  __shared__ uint32_t s_tbase;
  __shared__ int s_seq, s_seg, s_wsum[PREP_THREADS / 32];
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  if (tid == 0) s_abort = 0;

  int j = 0;
  const int n = block_locate_segment<PREP_THREADS>(p.cu_seqlens, p.n_seqs, p.T_total, C, 0,
                                                   blockIdx.x, &j, &s_seq, &s_seg, s_wsum,
                                                   p.status);
  if (n < 0 || (int64_t)blockIdx.x >= max_chunks) return;
  const int hk = h / (p.H_v / p.H_k);
  const int64_t c0 = (int64_t)p.cu_seqlens[n] + (int64_t)j * C;
  const int64_t rem = (int64_t)p.cu_seqlens[n + 1] - c0;
  const int L = rem < C ? (int)rem : C;
  uint8_t* rec = ws + ((int64_t)blockIdx.x * p.H_v + h) * REC_BYTES;

  uint8_t* Aqk = sm + SM_AQK;
  uint8_t* Xw = sm + SM_XW;
  uint8_t* Xu = sm + SM_XU;
  uint8_t* Tb = sm + SM_TB;
  float* Lf = reinterpret_cast<float*>(sm + SM_LF);
  float* Tf = reinterpret_cast<float*>(sm + SM_TF);
  float* Xt = reinterpret_cast<float*>(sm + SM_XT);
  float* gc = reinterpret_cast<float*>(sm + SM_GC);
  float* bt = reinterpret_cast<float*>(sm + SM_BT);
  float* eg = reinterpret_cast<float*>(sm + SM_EG);

  if (warp == 0) tmem_alloc(&s_tbase, 256);
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  if (tid < C) {
    gc[tid] = tid < L ? p.g[(c0 + tid) * p.H_v + h] : 0.f;
    bt[tid] = tid < L ? p.beta[(c0 + tid) * p.H_v + h] : 0.f;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = s_tbase;
  if (warp == 0) {  // inclusive cumulative sum of g over the chunk
    float a0 = gc[2 * lane], a1 = gc[2 * lane + 1];
    float s = a0 + a1, incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      float y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const float ex = incl - s;
    gc[2 * lane] = ex + a0;
    gc[2 * lane + 1] = ex + a0 + a1;
    eg[2 * lane] = expf(ex + a0);
    eg[2 * lane + 1] = expf(ex + a0 + a1);
  }
  __syncthreads();

  // ---- operands: [K; Q] (K-major), K*beta*exp(gc) and V*beta (MN-major, M = feature)
  const __half* qg = static_cast<const __half*>(p.q);
  const __half* kg = static_cast<const __half*>(p.k);
  const __half* vg = static_cast<const __half*>(p.v);
#pragma unroll 2
  for (int it = 0; it < 8; ++it) {
    const int combo = it * 4 + warp;          // 32 combos of (row group r8, dg quad)
    const int r = (combo >> 2) * 8 + (lane & 7);
    const int dg = (combo & 3) * 4 + (lane >> 3);
    uint4 kv = make_uint4(0, 0, 0, 0), qv = kv, vv = kv;
    if (r < L) {
      kv = ld16(kg + ((c0 + r) * p.H_k + hk) * D + dg * 8);
      qv = ld16(qg + ((c0 + r) * p.H_k + hk) * D + dg * 8);
      vv = ld16(vg + ((c0 + r) * p.H_v + h) * D + dg * 8);
    }
    *reinterpret_cast<uint4*>(Aqk + (r & 7) * 16 + (r >> 3) * 2048 + dg * 128) = kv;
    *reinterpret_cast<uint4*>(Aqk + (r & 7) * 16 + ((r + 64) >> 3) * 2048 + dg * 128) = qv;
    const uint32_t mo = dg * 1024 + (r >> 3) * 128 + (r & 7) * 16;
    *reinterpret_cast<uint4*>(Xw + mo) = scale8(kv, bt[r] * eg[r]);
    *reinterpret_cast<uint4*>(Xu + mo) = scale8(vv, bt[r]);
  }
  fence_proxy_async();
  fence_before_sync();
  __syncthreads();

  // ---- [K; Q] K^T -> TMEM columns 0..63
  if (tid == 0) {
    fence_after_sync();
    const uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint64_t ad = desc(smem_u32(Aqk) + ks * 256, 128, 2048);
      mma_f16(tb, ad, ad, id, ks > 0);  // B = rows 0-63 of the same buffer (K)
    }
    commit(&bar[0]);
  }
  if (!mbar_wait(&bar[0], 0, &s_abort)) {
    set_status(p.status, GDN_ETIMEOUT);
    s_abort = 1;
  }
  fence_after_sync();
  {
    uint32_t r0[32], r1[32];
    tmem_ld32(taddr(tb, warp * 32, 0), r0);
    tmem_ld32(taddr(tb, warp * 32, 32), r1);
    tmem_wait_ld();
    const int row = warp * 32 + lane;
    if (warp < 2) {  // L row i
      const int i = row;
      const float gi = gc[i], bi = bt[i];
#pragma unroll
      for (int jj = 0; jj < 64; ++jj) {
        const float kk = __uint_as_float(jj < 32 ? r0[jj] : r1[jj - 32]);
        Lf[i * LDS + jj] = (jj < i) ? bi * kk * expf(gi - gc[jj]) : 0.f;
      }
    } else {  // P row i -> workspace, K-major canonical (LBO 128, SBO 1024)
      const int i = row - 64;
      const float gi = gc[i];
      float pv[8];
#pragma unroll
      for (int jg = 0; jg < 8; ++jg) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int jj = jg * 8 + e;
          const float qk = __uint_as_float(jj < 32 ? r0[jj] : r1[jj - 32]);
          pv[e] = (jj <= i) ? qk * expf(gi - gc[jj]) : 0.f;
        }
        *reinterpret_cast<uint4*>(rec + REC_P + (i & 7) * 16 + (i >> 3) * 1024 + jg * 128) =
            pack8(pv);
      }
    }
  }
  __syncthreads();

  // ---- T = (I + L)^-1, then as the K-major B operand (N = i, K = j) in fp16
  tri_inverse_64(Lf, Tf, Xt);
  for (int e = tid; e < 64 * 8; e += PREP_THREADS) {
    const int i = e >> 3, jg = e & 7;
    float tv[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int jj = jg * 8 + x;
      tv[x] = jj <= i ? Tf[i * LDS + jj] : 0.f;
    }
    *reinterpret_cast<uint4*>(Tb + (i & 7) * 16 + (i >> 3) * 1024 + jg * 128) = pack8(tv);
  }
  fence_proxy_async();
  fence_before_sync();
  __syncthreads();

  // ---- W^T = Xw^T T^T -> cols 64..127 ; U^T = Xu^T T^T -> cols 128..191
  if (tid == 0 && !s_abort) {
    fence_after_sync();
    const uint32_t id = idesc_f16(128, 64, true, false);
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks) {
      const uint64_t bd = desc(smem_u32(Tb) + ks * 256, 128, 1024);
      mma_f16(tb + 64, desc(smem_u32(Xw) + ks * 256, 128, 1024), bd, id, ks > 0);
      mma_f16(tb + 128, desc(smem_u32(Xu) + ks * 256, 128, 1024), bd, id, ks > 0);
    }
    commit(&bar[1]);
  }
  if (!mbar_wait(&bar[1], 0, &s_abort)) {
    set_status(p.status, GDN_ETIMEOUT);
    s_abort = 1;
  }
  fence_after_sync();
  {
    // lane (feature) d holds W^T[d][i], U^T[d][i] for i = 0..63; stage W (K-major canonical
    // of the scan's [W; Q] operand) and U (row-major) in the Aqk buffer, then bulk-copy out.
    const int d = warp * 32 + lane;
    uint8_t* Wst = Aqk;
    uint8_t* Ust = Aqk + 16384;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t rw[32], ru[32];
      tmem_ld32(taddr(tb, warp * 32, 64 + 32 * half), rw);
      tmem_ld32(taddr(tb, warp * 32, 128 + 32 * half), ru);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int i = half * 32 + x;
        *reinterpret_cast<__half*>(Wst + (i & 7) * 16 + (i >> 3) * 2048 + (d >> 3) * 128 +
                                   (d & 7) * 2) = __float2half_rn(__uint_as_float(rw[x]));
        *reinterpret_cast<__half*>(Ust + i * 256 + d * 2) =
            __float2half_rn(__uint_as_float(ru[x]));
      }
    }
  }
  if (tid < C) reinterpret_cast<float*>(rec + REC_G)[tid] = gc[tid];
  fence_proxy_async();
  fence_before_sync();
  __syncthreads();
  if (tid == 0) {
    bulk_s2g(rec + REC_W, Aqk, 16384);
    bulk_s2g(rec + REC_U, Aqk + 16384, 16384);
    bulk_commit();
    bulk_wait_all();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_relinquish();
    tmem_dealloc(tb, 256);
  }
}

// ======================================================================== scan kernel
constexpr int SCAN_THREADS = 256;
// per-stage shared memory (bytes)
constexpr int ST_A1 = 0;        // 32768 [W ; Q*exp(gc)] K-major (LBO 128, SBO 2048)
constexpr int ST_AK = 32768;    // 16384 K*exp(gl-gc) MN-major (M = d, K = token; LBO 128, SBO 1024)
constexpr int ST_AP = 49152;    // 8192 P = rows 64..127 of a K-major operand whose rows 0..63
                                //      (the 8 KB before it, inside ST_AK) are never used
constexpr int ST_UT = 57344;    // 64 x 36 fp32 U tile = 9216
constexpr int ST_GC = 66560;    // 64 fp32
constexpr int ST_BYTES = 66816;
constexpr int UT_LD = 36;
constexpr int SM_BS = 2 * ST_BYTES;       // 8192 S as MN-major B (N = 32, K = 128; LBO 128, SBO 2048)
constexpr int SM_BV = SM_BS + 8192;       // 4096 v_new as MN-major B (N = 32, K = 64; LBO 128, SBO 1024)
constexpr int SCAN_SMEM = SM_BV + 4096;   // 145920

__global__ void __launch_bounds__(SCAN_THREADS, 1)
tc_scan_kernel(const PrefillArgs p, const uint8_t* ws, int64_t max_chunks) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t full[2], empty[2], mma_a, mma_b;
  __shared__ uint32_t s_tbase;
  __shared__ int64_t s_red[SCAN_THREADS / 32];
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int hk = h / (p.H_v / p.H_k);

  const int64_t cs0 = p.cu_seqlens[n], cs1 = p.cu_seqlens[n + 1];
  bool ok = cs0 >= 0 && cs1 >= cs0 && cs1 <= p.T_total;
  const int slot = p.slot_ids[n];
  if (slot < 0 || slot >= p.n_slots) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  if (!ok) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_EINVAL);
    return;
  }
  if (tid == 0 && h == 0 && tile == 0) {
    for (int m = 0; m < n; ++m)
      if (p.slot_ids[m] == slot) { set_status(p.status, GDN_ESLOT); break; }
  }
  const int64_t base = block_segment_base<SCAN_THREADS>(p.cu_seqlens, n, p.T_total, C, s_red);
  const int nck = (int)((cs1 - cs0 + C - 1) / C);
  if (base + nck > max_chunks) {
    if (tid == 0) set_status(p.status, GDN_EINVAL);
    return;
  }
  const bool rst = p.reset != nullptr && p.reset[n] != 0;
  float* Sg = p.state + (((int64_t)slot * p.H_v + h) * D) * p.d_v + tile * TILE;

  if (tid == 0) {
    s_abort = 0;
    mbar_init(&full[0], 128);
    mbar_init(&full[1], 128);
    mbar_init(&empty[0], 1);
    mbar_init(&empty[1], 1);
    mbar_init(&mma_a, 1);
    mbar_init(&mma_b, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tbase, 64);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = s_tbase;
  uint8_t* BS = sm + SM_BS;
  uint8_t* BV = sm + SM_BV;

  if (warp >= 4) {
    // ================= producer: stage chunk c into shared-memory stage c & 1
    const int pt = tid - 128, pw = pt >> 5;
    const __half* qg = static_cast<const __half*>(p.q);
    const __half* kg = static_cast<const __half*>(p.k);
    for (int c = 0; c < nck; ++c) {
      const int s = c & 1;
      uint8_t* st = sm + s * ST_BYTES;
      if (c >= 2 && !mbar_wait(&empty[s], ((c >> 1) - 1) & 1, &s_abort)) {
        set_status(p.status, GDN_ETIMEOUT);
        s_abort = 1;
      }
      const uint8_t* rec = ws + ((base + c) * p.H_v + h) * REC_BYTES;
      const int64_t c0 = cs0 + (int64_t)c * C;
      const int L = (cs1 - c0) < C ? (int)(cs1 - c0) : C;
      if (pt == 0 && !s_abort) {
        mbar_expect_tx(&full[s], 16384 + 8192);
        bulk_g2s(st + ST_A1, rec + REC_W, 16384, &full[s]);
        bulk_g2s(st + ST_AP, rec + REC_P, 8192, &full[s]);
      }
      float* gcs = reinterpret_cast<float*>(st + ST_GC);
      if (pt < C) gcs[pt] = reinterpret_cast<const float*>(rec + REC_G)[pt];
      named_bar(2, 128);
      const float gl = gcs[L - 1];
      // Q * exp(gc) -> A1 rows 64..127 (K-major); K * exp(gl - gc) -> AK (MN-major)
#pragma unroll 2
      for (int it = 0; it < 8; ++it) {
        const int combo = it * 4 + pw;
        const int r = (combo >> 2) * 8 + (lane & 7);
        const int dg = (combo & 3) * 4 + (lane >> 3);
        uint4 qv = make_uint4(0, 0, 0, 0), kv = qv;
        if (r < L) {
          qv = scale8(ld16(qg + ((c0 + r) * p.H_k + hk) * D + dg * 8), expf(gcs[r]));
          kv = scale8(ld16(kg + ((c0 + r) * p.H_k + hk) * D + dg * 8), expf(gl - gcs[r]));
        }
        *reinterpret_cast<uint4*>(st + ST_A1 + (r & 7) * 16 + ((r + 64) >> 3) * 2048 + dg * 128) = qv;
        *reinterpret_cast<uint4*>(st + ST_AK + dg * 1024 + (r >> 3) * 128 + (r & 7) * 16) = kv;
      }
      // U tile (fp32) : 64 rows x 32 columns
      {
        float* ut = reinterpret_cast<float*>(st + ST_UT);
        for (int e = pt; e < 64 * 4; e += 128) {
          const int r = e >> 2, part = e & 3;
          uint4 u = *reinterpret_cast<const uint4*>(rec + REC_U + r * 256 + tile * 64 + part * 16);
          const __half2* hu = reinterpret_cast<const __half2*>(&u);
          float4 a, b;
          float2 f0 = __half22float2(hu[0]), f1 = __half22float2(hu[1]);
          float2 f2 = __half22float2(hu[2]), f3 = __half22float2(hu[3]);
          a = make_float4(f0.x, f0.y, f1.x, f1.y);
          b = make_float4(f2.x, f2.y, f3.x, f3.y);
          *reinterpret_cast<float4*>(ut + r * UT_LD + part * 8) = a;
          *reinterpret_cast<float4*>(ut + r * UT_LD + part * 8 + 4) = b;
        }
      }
      fence_proxy_async();
      mbar_arrive(&full[s]);
    }
    // drain: make sure the last bulk copies have landed before the block can exit
    if (pt == 0) {
      for (int c = nck - 2 < 0 ? 0 : nck - 2; c < nck; ++c)
        mbar_wait(&full[c & 1], (c >> 1) & 1, nullptr, 200000000LL);
    }
  } else {
    // ================= consumer: state tile rows in registers, tcgen05 chain per chunk
    const int i = tid;  // S row = TMEM lane
    float srow[TILE];
    if (rst) {
#pragma unroll
      for (int x = 0; x < TILE; ++x) srow[x] = 0.f;
    } else {
#pragma unroll
      for (int x = 0; x < TILE; x += 4) {
        float4 v = *reinterpret_cast<const float4*>(Sg + (int64_t)i * p.d_v + x);
        srow[x] = v.x; srow[x + 1] = v.y; srow[x + 2] = v.z; srow[x + 3] = v.w;
      }
    }
    const uint32_t id_a = idesc_f16(128, TILE, false, true);
    const uint32_t id_k = idesc_f16(128, TILE, true, true);
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(p.o);
    float* of = static_cast<float*>(p.o);
    for (int c = 0; c < nck; ++c) {
      const int s = c & 1;
      uint8_t* st = sm + s * ST_BYTES;
      if (!mbar_wait(&full[s], (c >> 1) & 1, &s_abort)) {
        set_status(p.status, GDN_ETIMEOUT);
        s_abort = 1;
      }
      const int64_t c0 = cs0 + (int64_t)c * C;
      const int L = (cs1 - c0) < C ? (int)(cs1 - c0) : C;
      const float* gcs = reinterpret_cast<const float*>(st + ST_GC);
      const float el = expf(gcs[L - 1]);
      // (1) S -> fp16 MN-major B operand
#pragma unroll
      for (int jg = 0; jg < TILE / 8; ++jg)
        *reinterpret_cast<uint4*>(BS + jg * 2048 + (i >> 3) * 128 + (i & 7) * 16) =
            pack8(srow + jg * 8);
      fence_proxy_async();
      fence_before_sync();
      named_bar(1, 128);
      // (2) D1 = [W ; Q~] S
      if (tid == 0 && !s_abort) {
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_f16(tb, desc(smem_u32(st + ST_A1) + ks * 256, 128, 2048),
                  desc(smem_u32(BS) + ks * 256, 128, 2048), id_a, ks > 0);
        commit(&mma_a);
      }
      if (!mbar_wait(&mma_a, c & 1, &s_abort)) {
        set_status(p.status, GDN_ETIMEOUT);
        s_abort = 1;
      }
      fence_after_sync();
      // (3) v_new = U - D1[0:64] -> fp16 MN-major B operand
      if (warp < 2) {
        uint32_t r[32];
        tmem_ld32(taddr(tb, warp * 32, 0), r);
        tmem_wait_ld();
        const int t = i;
        const float* ut = reinterpret_cast<const float*>(st + ST_UT) + t * UT_LD;
        float vn[TILE];
#pragma unroll
        for (int x = 0; x < TILE; ++x) vn[x] = (t < L) ? ut[x] - __uint_as_float(r[x]) : 0.f;
#pragma unroll
        for (int jg = 0; jg < TILE / 8; ++jg)
          *reinterpret_cast<uint4*>(BV + jg * 1024 + (t >> 3) * 128 + (t & 7) * 16) =
              pack8(vn + jg * 8);
        fence_proxy_async();
      }
      fence_before_sync();
      named_bar(1, 128);
      // (4) D2 = K~^T v_new ; D1[64:128] += P v_new
      if (tid == 0 && !s_abort) {
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
          const uint64_t bd = desc(smem_u32(BV) + ks * 256, 128, 1024);
          mma_f16(tb + 32, desc(smem_u32(st + ST_AK) + ks * 256, 128, 1024), bd, id_k, ks > 0);
          mma_f16(tb, desc(smem_u32(st + ST_AP) - 8192 + ks * 256, 128, 1024), bd, id_a, 1);
        }
        commit(&mma_b);
      }
      if (!mbar_wait(&mma_b, c & 1, &s_abort)) {
        set_status(p.status, GDN_ETIMEOUT);
        s_abort = 1;
      }
      fence_after_sync();
      if (tid == 0) mbar_arrive(&empty[s]);
      // (5) S = exp(g_last) S + D2 ; o = D1[64:128]
      {
        uint32_t r[32];
        tmem_ld32(taddr(tb, warp * 32, 32), r);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < TILE; ++x) srow[x] = fmaf(el, srow[x], __uint_as_float(r[x]));
      }
      if (warp >= 2) {
        uint32_t r[32];
        tmem_ld32(taddr(tb, warp * 32, 0), r);
        tmem_wait_ld();
        const int t = i - 64;
        if (t < L && !s_abort) {
          const int64_t off = ((c0 + t) * p.H_v + h) * p.d_v + tile * TILE;
          if (p.o_dtype == GDN_BF16) {
#pragma unroll
            for (int x = 0; x < TILE; x += 4)
              st4(ob + off + x, make_float4(__uint_as_float(r[x]), __uint_as_float(r[x + 1]),
                                            __uint_as_float(r[x + 2]), __uint_as_float(r[x + 3])));
          } else {
#pragma unroll
            for (int x = 0; x < TILE; x += 4)
              st4(of + off + x, make_float4(__uint_as_float(r[x]), __uint_as_float(r[x + 1]),
                                            __uint_as_float(r[x + 2]), __uint_as_float(r[x + 3])));
          }
        }
      }
      fence_before_sync();
    }
    if (!s_abort) {
#pragma unroll
      for (int x = 0; x < TILE; x += 4)
        *reinterpret_cast<float4*>(Sg + (int64_t)i * p.d_v + x) =
            make_float4(srow[x], srow[x + 1], srow[x + 2], srow[x + 3]);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tmem_relinquish();
    tmem_dealloc(tb, 64);
  }
}

}  // namespace

bool prefill_tc_supported(int d_k, int d_v, int chunk, int qkv_dtype) {
  return d_k == D && d_v == D && chunk == C && qkv_dtype == GDN_F16;
}

size_t prefill_tc_workspace(int H_v, int d_k, int d_v, int64_t T_total, int n_seqs, int chunk) {
  (void)d_k; (void)d_v; (void)chunk;
  const int64_t max_chunks = (T_total + C - 1) / C + n_seqs;
  return (size_t)max_chunks * H_v * REC_BYTES;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
  if (!prefill_tc_supported(a.d_k, a.d_v, a.chunk, a.qkv_dtype)) return cudaErrorNotSupported;
  const int64_t max_chunks = (a.T_total + C - 1) / C + a.n_seqs;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  cudaError_t e = cudaFuncSetAttribute(tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       PREP_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(tc_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SCAN_SMEM);
  if (e != cudaSuccess) return e;
  if (max_chunks > 0) {
    dim3 g1((unsigned)max_chunks, a.H_v);
    tc_prep_kernel<<<g1, PREP_THREADS, PREP_SMEM, s>>>(a, ws, max_chunks);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dim3 g2(a.d_v / TILE, a.H_v, a.n_seqs);
  tc_scan_kernel<<<g2, SCAN_THREADS, SCAN_SMEM, s>>>(a, ws, max_chunks);
  return cudaGetLastError();
}


// ---------------------------------------------------------------- allocation-free variant
// Scratch for callers that cannot hand the library a workspace: it lives in one fixed-size
// array in device global memory that every GPU loading this library reserves until the
// process exits. All calls on a device share it, so calls that overlap on the GPU (two
// streams, or two threads) race on it. The prep kernel fully writes every record the scan
// kernel later reads, so nothing has to be cleared between calls.
constexpr size_t kNoAllocScratchBytes = 64ull << 20;  // 64 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

size_t prefill_tc_noalloc_capacity() { return kNoAllocScratchBytes; }

cudaError_t launch_prefill_tc_noalloc(const PrefillArgs& a, cudaStream_t s) {
  if (!prefill_tc_supported(a.d_k, a.d_v, a.chunk, a.qkv_dtype)) return cudaErrorNotSupported;
  if (prefill_tc_workspace(a.H_v, a.d_k, a.d_v, a.T_total, a.n_seqs, a.chunk) >
      kNoAllocScratchBytes)
    return cudaErrorInvalidValue;
  // The array's device address, looked up once per device with that device current (the
  // host-side name is only a stand-in and must never reach a kernel).
  constexpr int kMaxDev = 64;
  static void* addr[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return e;
      addr[dev] = p;
    }
    scratch = addr[dev];
  }
  PrefillArgs b = a;
  b.workspace = scratch;
  b.workspace_bytes = kNoAllocScratchBytes;
  return launch_prefill_tc(b, s);
}

}  // namespace gdn
