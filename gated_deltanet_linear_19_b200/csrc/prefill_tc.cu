// Chunked gated delta rule on the 5th-generation tensor cores (tcgen05, TMEM accumulators),
// for d_k = d_v = 128, chunk 64, fp16 q/k/v (the Qwen3-Next layer shape).
// Pages: qwen3next.cpp build_delta_net_chunking and the removed single-chunk path (the
// per-chunk math), chunk size 64 as QWEN3NEXT_CHUNK_SIZE in ik_llama.cpp.
//
// Two kernels:
//  1. tc_prep_kernel, one CTA per (chunk, key head) -- covering both value heads of the key
//     head when H_v = 2 H_k, else per (chunk, value head) -- fully parallel. Everything that
//     does not depend on the recurrent state:
//       [K; Q] K^T as ONE M=128 MMA (rows 0-63: K K^T, rows 64-127: Q K^T), once per key head,
//     and for each value head
//       g_cum, decay_ij = exp(g_cum_i - g_cum_j) (masked before exp),
//       L = beta_i (k_i.k_j) decay_ij (j < i), P = (q_i.k_j) decay_ij (j <= i),
//       T = (I + L)^-1 on the CUDA cores (blocked: 16 x 16 diagonal blocks by substitution,
//       then block products; the raw q, k, v rows arrive by TMA; shared memory is reused
//       stage by stage so that two CTAs fit on an SM),
//       W^T = (K*beta*exp(g_cum))^T T^T and U^T = (V*beta)^T T^T as M=128 MMAs,
//       Q~ = Q*exp(g_cum) and K~ = K*exp(g_last - g_cum).
//     The pages' attn = -(beta K K^T * decay) and T = (I - attn)^-1 are the same matrices.
//     Every field is written to the workspace record already in the scan kernel's operand
//     layout, so the scan only issues bulk copies. tc_prep_kernel<true> (the layer prefill)
//     computes its q, k, v rows and gates from raw x itself (the layer front: conv, SiLU,
//     L2 norm, q scale) instead of loading them; the scan then writes the new conv state.
//  2. tc_scan_kernel, one CTA per (sequence, value head, 32-column d_v tile), sequential
//     over the sequence's chunks. Warps 0-3 own the fp32 state tile S[128 x 32] in registers
//     (thread i = row i = TMEM lane i) and run the chain
//       D1 = [W; Q~] S                                 (M=128, N=32, K=128)
//       v_new = U - D1[0:64]
//       D2 = K~^T v_new                                (M=128, N=32, K=64)
//       D1[64:128] += P v_new                          (M=128, N=32, K=64; rows 0-63 unused)
//       S = exp(g_last) S + D2 ;  o = D1[64:128]
//     with each serial MMA split over two issuing threads, while a loader warp prefetches
//     the next chunks' record slices into NSTAGE shared-memory stages. (tc_scan_head_kernel
//     does the same for a whole head per CTA.) The sequences are taken longest first.
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

// workspace record per (chunk, value head); every field is one bulk copy for the scan
constexpr int REC_A1 = 0;       // [W ; Q~] [128 x 128] fp16, K-major canonical (LBO 128,
                                // SBO 2048): rows 0..63 W, rows 64..127 Q~ = Q*exp(g_cum)
constexpr int REC_AK = 32768;   // K~ = K*exp(g_last - g_cum) [64 x 128] fp16, MN-major
                                // canonical (M = d, K = token; LBO 128, SBO 1024)
constexpr int REC_P = 49152;    // P [64 x 64] fp16, K-major canonical (LBO 128, SBO 1024)
constexpr int REC_U = 57344;    // U as 4 column tiles of 32 columns (4 KB each), each an MN-major
                                // canonical operand (N = column, K = token; LBO 128, SBO 1024)
constexpr int REC_G = 73728;    // g_cum [64] fp32
constexpr int REC_BYTES = 73984;

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
// One block per (chunk, key head): the key-head work (the q, k rows -- in the layer prefill
// their front -- the [K; Q] operand and the [K; Q] K^T product) is done once for the NV value
// heads that read that key head (NV = H_v / H_k when that is 2, else 1 and one block per
// value head); then, value head after value head, the gate-dependent work (decay masks, L, P,
// T = (I + L)^-1, W, U) and the records.
constexpr int PREP_THREADS = 128;
// H_v = 2 H_k: one record block per (chunk, key head) covering both value heads, or one per
// (chunk, value head), which runs three blocks per SM instead of two but recomputes the key
// head's [K K^T ; Q K^T] (and, in the layer prefill, its front). Measured (B = 1, L2 flushed):
// the layer prefill is faster per key head (T = 2048 / 8192 / 16384: 123 / 405 / 791 against
// 126 / 418 / 807 us; varlen 2.23 against 2.32 ms, 4 x 65536 10.7 against 11.1 ms; only
// T = 4096 is 3 us slower), the q / k / v prefill per value head once the per-value-head grid
// fills two waves (T = 2048 / 4096 / 8192 / 16384: 125 / 224 / 422 / 814 against
// 127 / 234 / 431 / 842 us; T = 1024: 78 against 74 us).
constexpr int kPrepPerValueHeadMinWaves = 2;
// shared memory map (bytes). R0 is reused as the kernel proceeds:
//   raw k | raw q rows -> [K; Q] K-major operand -> L (fp32, stride 65) | T (fp32, stride 68)
//   -> T as the fp16 B operand (over L) -> W | U staging for the bulk store.
constexpr int LS = 65;                    // L row stride (conflict-free row and column access)
constexpr int TS = 68;                    // T row stride (16-byte rows for float4 reads)
constexpr int SM_R0 = 0;                  // 34048 = 64*65*4 + 64*68*4 (>= 32768 for [K; Q])
constexpr int SM_XU0 = 34048;             // 16384 raw v rows of value head 0 -> (V*beta) MN-major
constexpr int SM_XW0 = SM_XU0 + 16384;    // 16384 (K*beta*exp(gc)) MN-major, value head 0
constexpr int SM_XU1 = SM_XW0 + 16384;    // the same for value head 1
constexpr int SM_XW1 = SM_XU1 + 16384;
constexpr int SM_X = SM_XW1 + 16384;      // 32 x 36 fp32 = 4608: block products of the inverse
// then the gates (prep_g_off): per value head g_cum, beta, exp(g_cum), exp(g_last - g_cum),
// 64 fp32 each (1024 bytes); 106240 bytes in all, two blocks per SM.
// A block of one value head (NV = 1) has no second XU / XW pair: the inverse's scratch and
// the gates move down to where XU1 would be (72448 bytes: three blocks per SM), its fused
// front's x tiles start at R0 and are converted in place, and its tensor memory is 128
// columns ([K K^T ; Q K^T] in 0..63, then U^T over them and W^T in 64..127).
constexpr int prep_x_off(int nv) { return nv == 2 ? SM_X : SM_XU1; }
constexpr int prep_g_off(int nv) { return prep_x_off(nv) + 4608; }
constexpr int prep_smem(int nv) { return prep_g_off(nv) + nv * 1024; }
constexpr uint32_t prep_tmem_cols(int nv) { return nv == 2 ? 256 : 128; }
constexpr uint32_t prep_w_col(int nv) { return nv == 2 ? 128 : 64; }
constexpr uint32_t prep_u_col(int nv) { return nv == 2 ? 192 : 0; }
constexpr int prep_min_blocks(int nv) { return nv == 2 ? 2 : 3; }

// T = (I + L)^-1 for a strictly lower-triangular 64 x 64 L (fp32, row stride LS), written to
// Tm (row stride TS), in two block levels:
//   1. the four 16 x 16 diagonal blocks by forward substitution (warp b, lane = column);
//   2. within each 32 x 32 half, T_10 = -T_11 (L_10 T_00) with 16 x 16 blocks;
//   3. T_10 = -T_11 (L_10 T_00) again with the 32 x 32 halves.
// (For a block lower-triangular matrix the inverse's off-diagonal block is -T_11 L_10 T_00.)
// The block products are register-blocked (each thread a 1 x 4 or 2 x 4 strip of outputs).
__device__ void tri_inverse_blocked(const float* Lf, float* Tm, float* X) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // 1. diagonal 16 x 16 blocks; zero the upper 16 x 16 blocks of each 32 x 32 half
  {
    const int b = warp, c = lane & 15;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m) {
        if (m & 1) acc1 = fmaf(Lf[(16 * b + i) * LS + 16 * b + m], t[m], acc1);
        else acc0 = fmaf(Lf[(16 * b + i) * LS + 16 * b + m], t[m], acc0);
      }
      t[i] = (i == c) ? 1.f : (i > c ? -(acc0 + acc1) : 0.f);
    }
    if (lane < 16) {
#pragma unroll
      for (int i = 0; i < 16; ++i) Tm[(16 * b + i) * TS + 16 * b + c] = t[i];
    } else if ((b & 1) == 0) {
      // block (b, b + 1) above the diagonal inside the 32 x 32 half
#pragma unroll
      for (int i = 0; i < 16; ++i) Tm[(16 * b + i) * TS + 16 * (b + 1) + c] = 0.f;
    }
  }
  __syncthreads();
  // 2. T_{2P+1, 2P} = -T_{2P+1, 2P+1} (L_{2P+1, 2P} T_{2P, 2P}) for P = 0, 1
  const int P = tid >> 6, i2 = (tid & 63) >> 2, j2 = (tid & 3) * 4;
  const int r0 = 32 * P, r1 = 32 * P + 16;  // row/column offsets of blocks 2P and 2P+1
  {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int k = 0; k < 16; ++k) {
      const float l = Lf[(r1 + i2) * LS + r0 + k];
      const float4 tv = *reinterpret_cast<const float4*>(Tm + (r0 + k) * TS + r0 + j2);
      acc.x = fmaf(l, tv.x, acc.x); acc.y = fmaf(l, tv.y, acc.y);
      acc.z = fmaf(l, tv.z, acc.z); acc.w = fmaf(l, tv.w, acc.w);
    }
    *reinterpret_cast<float4*>(X + P * 16 * 20 + i2 * 20 + j2) = acc;
  }
  __syncthreads();
  {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int k = 0; k < 16; ++k) {
      const float tl = Tm[(r1 + i2) * TS + r1 + k];
      const float4 xv = *reinterpret_cast<const float4*>(X + P * 16 * 20 + k * 20 + j2);
      acc.x = fmaf(tl, xv.x, acc.x); acc.y = fmaf(tl, xv.y, acc.y);
      acc.z = fmaf(tl, xv.z, acc.z); acc.w = fmaf(tl, xv.w, acc.w);
    }
    *reinterpret_cast<float4*>(Tm + (r1 + i2) * TS + r0 + j2) =
        make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
  }
  __syncthreads();
  // 3. T[32:64][0:32] = -T[32:64][32:64] (L[32:64][0:32] T[0:32][0:32]); thread = 2 rows x 4 cols
  const int rp = tid >> 3, cq = (tid & 7) * 4;
  {
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const float l0 = Lf[(32 + 2 * rp) * LS + k], l1 = Lf[(33 + 2 * rp) * LS + k];
      const float4 tv = *reinterpret_cast<const float4*>(Tm + k * TS + cq);
      a0.x = fmaf(l0, tv.x, a0.x); a0.y = fmaf(l0, tv.y, a0.y);
      a0.z = fmaf(l0, tv.z, a0.z); a0.w = fmaf(l0, tv.w, a0.w);
      a1.x = fmaf(l1, tv.x, a1.x); a1.y = fmaf(l1, tv.y, a1.y);
      a1.z = fmaf(l1, tv.z, a1.z); a1.w = fmaf(l1, tv.w, a1.w);
    }
    *reinterpret_cast<float4*>(X + (2 * rp) * 36 + cq) = a0;
    *reinterpret_cast<float4*>(X + (2 * rp + 1) * 36 + cq) = a1;
  }
  __syncthreads();
  {
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const float t0 = Tm[(32 + 2 * rp) * TS + 32 + k], t1 = Tm[(33 + 2 * rp) * TS + 32 + k];
      const float4 xv = *reinterpret_cast<const float4*>(X + k * 36 + cq);
      a0.x = fmaf(t0, xv.x, a0.x); a0.y = fmaf(t0, xv.y, a0.y);
      a0.z = fmaf(t0, xv.z, a0.z); a0.w = fmaf(t0, xv.w, a0.w);
      a1.x = fmaf(t1, xv.x, a1.x); a1.y = fmaf(t1, xv.y, a1.y);
      a1.z = fmaf(t1, xv.z, a1.z); a1.w = fmaf(t1, xv.w, a1.w);
    }
    *reinterpret_cast<float4*>(Tm + (32 + 2 * rp) * TS + cq) = make_float4(-a0.x, -a0.y, -a0.z, -a0.w);
    *reinterpret_cast<float4*>(Tm + (33 + 2 * rp) * TS + cq) = make_float4(-a1.x, -a1.y, -a1.z, -a1.w);
  }
  __syncthreads();
}

// SiLU for the fp16 q / k / v operands: y sigmoid(y) = h + h tanh(h) with h = y / 2, from the
// PTX approximate tanh (one special-function instruction instead of an exponential and a
// reciprocal; its error, a few 1e-4 of |y|, is below the fp16 rounding of the result)
__device__ __forceinline__ float silu16(float y) {
  const float h = 0.5f * y;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

__device__ __forceinline__ void unpack8_bf16(uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// x tile of the layer prefill: 67 rows (3 conv-window rows before the chunk, then its 64)
// x 128 channels bf16, as one TMA box
constexpr int XT_ROWS = C + 3;
constexpr int XT_BYTES = XT_ROWS * 256;  // 17152

// 8 fp16 values times a common fp16 scale (packed multiplies)
__device__ __forceinline__ uint4 hscale8(uint4 v, __half2 s) {
  __half2* h = reinterpret_cast<__half2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __hmul2(h[i], s);
  return v;
}

// Layer prefill front for one 128-channel group of the chunk: x tile (bf16, 67 rows) ->
// conv + SiLU (+ L2 norm and scale for q / k) -> 64 fp16 rows, row-major [64][128] at dst
// (the same evaluation as the front kernel's). The 3 window rows before a sequence's first
// token come from its conv state (or zero on reset). Thread: 8 channels (cg) of 8 rows.
__device__ void front_group(const PrefillArgs& p, uint8_t* tile, uint8_t* dst, int ch0,
                            bool norm, float scale, bool first, bool rst,
                            const __nv_bfloat16* cst, int cdim, bool in_place = false) {
  const int tid = threadIdx.x;
  if (first) {
    if (tid < 48) {
      const int row = tid >> 4, cg = tid & 15;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (!rst) v = *reinterpret_cast<const uint4*>(cst + (int64_t)row * cdim + ch0 + cg * 8);
      *reinterpret_cast<uint4*>(tile + row * 256 + cg * 16) = v;
    }
    __syncthreads();
  }
  const int cg = tid & 15, rb = tid >> 4;
  float w[8][4];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float4 w4 = *reinterpret_cast<const float4*>(p.conv_w + (int64_t)(ch0 + cg * 8 + e) * 4);
    w[e][0] = w4.x; w[e][1] = w4.y; w[e][2] = w4.z; w[e][3] = w4.w;
  }
  float xa[8], xb[8], xc[8], y[8][8], ss[8];
  const uint8_t* tp = tile + (rb * 8) * 256 + cg * 16;
  unpack8_bf16(*reinterpret_cast<const uint4*>(tp), xa);
  unpack8_bf16(*reinterpret_cast<const uint4*>(tp + 256), xb);
  unpack8_bf16(*reinterpret_cast<const uint4*>(tp + 512), xc);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float xd[8];
    unpack8_bf16(*reinterpret_cast<const uint4*>(tp + (i + 3) * 256), xd);
    ss[i] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float acc = w[e][0] * xa[e];
      acc = fmaf(w[e][1], xb[e], acc);
      acc = fmaf(w[e][2], xc[e], acc);
      acc = fmaf(w[e][3], xd[e], acc);
      y[i][e] = silu16(acc);
      ss[i] = fmaf(y[i][e], y[i][e], ss[i]);
      xa[e] = xb[e]; xb[e] = xc[e]; xc[e] = xd[e];
    }
  }
  // dst overlapping the tile: every thread has read its rows before any is overwritten
  if (in_place) __syncthreads();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float mul = 1.f;
    if (norm) {
      float t = ss[i];
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      mul = scale * rsqrtf(t + p.eps);
    }
    float f[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = y[i][e] * mul;
    *reinterpret_cast<uint4*>(dst + (rb * 8 + i) * 256 + cg * 16) = pack8(f);
  }
}

// 16-byte chunk (row r, 8-element group dg) handled by this thread in iteration it (0..7).
// Each 8-lane quarter of a warp takes one diagonal of an 8-row x 8-group block: 8 different
// rows and 8 different groups, so both the row-major reads (bank group = dg mod 8) and the
// canonical-layout accesses (bank group = r mod 8) are conflict-free.
__device__ __forceinline__ void chunk_of(int it, int& r, int& dg) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int P = (it * 4 + warp) * 4 + (lane >> 3), j = lane & 7;
  r = (P >> 4) * 8 + j;
  dg = ((P >> 3) & 1) * 8 + ((j + P) & 7);
}

// FUSED: the layer prefill; the block computes its chunk's q, k (its key head) and v (its
// value heads) rows and the gates from x itself (conv + SiLU + L2 norm + q scale, as the front
// kernel does) into the same raw row layout the TMA loads fill otherwise.
template <bool FUSED, int NV>
__global__ void __launch_bounds__(PREP_THREADS, prep_min_blocks(NV))
tc_prep_kernel(const PrefillArgs p, uint8_t* ws, int64_t max_chunks,
               const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_x) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t bar[4];
  __shared__ uint32_t s_tbase;
  __shared__ int s_seq, s_seg, s_wsum[PREP_THREADS / 32];
  __shared__ int s_abort;
  // after a wait that gave up: the asynchronous work still to drain before the block may exit
  // (the TMA loads on bar[2], the MMA committed to bar[0], the MMA of value head s_pend1 on
  // bar[1]); the drain waits with the default limit
  __shared__ int s_pend2, s_pend0, s_pend1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the scan kernel may be scheduled now (it reads the records only after its
  // griddepcontrol.wait, which returns once this grid has completed)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) { s_abort = 0; s_pend2 = 0; s_pend0 = 0; s_pend1 = -1; }
  // every wait of this kernel gives up after this many cycles (GDN_ETIMEOUT)
  const long long wlim = p.wait_cycles > 0 ? p.wait_cycles : 2000000000LL;

  int j = 0;
  const int n = block_locate_segment<PREP_THREADS>(p.cu_seqlens, p.n_seqs, p.T_total, C, 0,
                                                   blockIdx.x, &j, &s_seq, &s_seg, s_wsum,
                                                   p.status);
  if (n < 0 || (int64_t)blockIdx.x >= max_chunks) return;
  // short sequences go to the token-by-token kernel of the same call: no record needed
  if (p.short_max > 0 && (int64_t)p.cu_seqlens[n + 1] - p.cu_seqlens[n] <= p.short_max) return;
  // key head and its value heads: NV == 2 -> blockIdx.y is the key head; NV == 1 -> the value
  // head
  int hk, hv[2];
  if constexpr (NV == 2) {
    hk = blockIdx.y;
    const bool tiled = (p.layout & GDN_GQA_TILED) != 0;
    hv[0] = tiled ? hk : 2 * hk;
    hv[1] = tiled ? hk + p.H_k : 2 * hk + 1;
  } else {
    hv[0] = hv[1] = blockIdx.y;
    hk = khead_of(hv[0], p.H_k, p.H_v, p.layout);
  }
  const int64_t c0 = (int64_t)p.cu_seqlens[n] + (int64_t)j * C;
  const int64_t rem = (int64_t)p.cu_seqlens[n + 1] - c0;
  const int L = rem < C ? (int)rem : C;

  uint8_t* R0 = sm + SM_R0;
  float* Lf = reinterpret_cast<float*>(R0);                   // L [64][LS]
  float* Tm = reinterpret_cast<float*>(R0 + 64 * LS * 4);     // T [64][TS]
  constexpr int kX = prep_x_off(NV), kG = prep_g_off(NV);
  float* Xp = reinterpret_cast<float*>(sm + kX);              // inverse block products
  uint8_t* Tb = R0;  // T as the fp16 B operand of the W / U MMAs, over L after the inverse
  auto XU = [&](int w) { return sm + (w ? SM_XU1 : SM_XU0); };
  auto XW = [&](int w) { return sm + (w ? SM_XW1 : SM_XW0); };
  auto gcp = [&](int w) { return reinterpret_cast<float*>(sm + kG + w * 1024); };
  auto btp = [&](int w) { return reinterpret_cast<float*>(sm + kG + w * 1024 + 256); };
  auto egp = [&](int w) { return reinterpret_cast<float*>(sm + kG + w * 1024 + 512); };
  auto ekp = [&](int w) { return reinterpret_cast<float*>(sm + kG + w * 1024 + 768); };
  // fused front: the x tiles (k, q, then the value heads' v), one after another from here
  uint8_t* const xt = sm + (NV == 2 ? SM_XU0 : SM_R0);
  // the chunk's gates, loaded now so that their latency overlaps the setup below
  float g_in[2] = {0.f, 0.f}, b_in[2] = {0.f, 0.f};
  if (tid < L) {
#pragma unroll
    for (int w = 0; w < NV; ++w) {
      const int h = hv[w];
      if constexpr (FUSED) {
        const float z = gate_alpha(p.fa, c0 + tid, h, p.H_k, p.H_v, p.layout) + p.dt_bias[h];
        g_in[w] = -expf(p.A_log[h]) * softplusf_(z);
        b_in[w] = sigmoidf_(gate_beta_logit(p.fa, p.fb, c0 + tid, h, p.H_k, p.H_v, p.layout));
      } else {
        g_in[w] = p.g[(c0 + tid) * p.H_v + h];
        b_in[w] = p.beta[(c0 + tid) * p.H_v + h];
      }
    }
  }
  const int cdim = (2 * p.H_k + p.H_v) * D;  // conv channels (q | k | v)
  const int ch_q = hk * D, ch_k = p.H_k * D + hk * D;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], 1);
    mbar_init(&bar[3], 1);
    fence_mbar_init();
    if constexpr (FUSED) {
      // x tiles (rows c0 - 3 .. c0 + 63; rows before row 0 read as zero) of the k, q and v
      // channels, one after another from xt on (NV = 2: from SM_XU0, the last reaching into
      // SM_X; NV = 1: from R0, the last reaching into XW0), all in flight
      mbar_arrive_expect_tx(&bar[2], (2 + NV) * XT_BYTES);
      tma_load_2d(xt, &tm_x, ch_k, (int)c0 - 3, &bar[2]);
      tma_load_2d(xt + XT_BYTES, &tm_x, ch_q, (int)c0 - 3, &bar[2]);
      for (int w = 0; w < NV; ++w)
        tma_load_2d(xt + (2 + w) * XT_BYTES, &tm_x, 2 * p.H_k * D + hv[w] * D, (int)c0 - 3,
                    &bar[2]);
    } else {
      // the chunk's raw rows of k, q (key head) and v (value heads): one TMA box [64 x 128]
      mbar_arrive_expect_tx(&bar[2], (2 + NV) * 16384);
      tma_load_3d(R0, &tm_k, 0, hk, (int)c0, &bar[2]);
      tma_load_3d(R0 + 16384, &tm_q, 0, hk, (int)c0, &bar[2]);
      for (int w = 0; w < NV; ++w) tma_load_3d(XU(w), &tm_v, 0, hv[w], (int)c0, &bar[2]);
    }
  }
  if (warp == 0) {
    tmem_alloc(&s_tbase, prep_tmem_cols(NV));
    // give up the right to allocate at once: another block is only placed on this SM once
    // the resident blocks have done so
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = s_tbase;
  if (tid < C) {
#pragma unroll
    for (int w = 0; w < NV; ++w) {
      gcp(w)[tid] = fmaxf(g_in[w], kGateFloor);  // see kGateFloor
      btp(w)[tid] = b_in[w];
    }
  }
  __syncthreads();
  if (warp < NV) {  // inclusive cumulative sum of g over the chunk, one warp per value head
    float* gc = gcp(warp);
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
    egp(warp)[2 * lane] = expf(ex + a0);
    egp(warp)[2 * lane + 1] = expf(ex + a0 + a1);
    // g_last = g_cum of the last token (rows past L add g = 0, so it is also g_cum[63])
    const float gl = __shfl_sync(0xffffffffu, incl, 31);
    ekp(warp)[2 * lane] = expf(gl - (ex + a0));
    ekp(warp)[2 * lane + 1] = expf(gl - (ex + a0 + a1));
  }
  if (!mbar_wait(&bar[2], 0, &s_abort, wlim)) {
    set_status(p.status, GDN_ETIMEOUT);
    s_abort = 1;
    s_pend2 = 1;
  }
  __syncthreads();
  if constexpr (FUSED) {
    const bool first = j == 0, rst = p.reset != nullptr && p.reset[n] != 0;
    const int slot = p.slot_ids[n];
    const __nv_bfloat16* cst =
        static_cast<const __nv_bfloat16*>(p.conv_state) + (int64_t)slot * 3 * cdim;
    // k tile -> raw k rows in R0[0, 16K), q tile -> R0[16K, 32K), v tile w -> raw v rows in
    // XU(w). NV = 2: each destination only overlaps tiles that are completely read by then.
    // NV = 1: each destination overlaps its own tile (converted in place: all reads of the
    // tile come before the first write) and tiles already read.
    constexpr bool kInPlace = NV == 1;
    front_group(p, xt, R0, ch_k, true, 1.f, first, rst, cst, cdim, kInPlace);
    __syncthreads();
    front_group(p, xt + XT_BYTES, R0 + 16384, ch_q, true, p.q_scale, first, rst, cst, cdim,
                kInPlace);
    __syncthreads();
    for (int w = 0; w < NV; ++w) {
      front_group(p, xt + (2 + w) * XT_BYTES, XU(w), 2 * p.H_k * D + hv[w] * D, false, 1.f,
                  first, rst, cst, cdim, kInPlace);
      __syncthreads();
    }
  }

  // ---- raw k | q rows -> [K; Q] K-major (in place, rows past L zero)
  {
    uint4 rk[8], rq[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      int r, dg;
      chunk_of(it, r, dg);
      rk[it] = *reinterpret_cast<const uint4*>(R0 + r * 256 + dg * 16);
      rq[it] = *reinterpret_cast<const uint4*>(R0 + 16384 + r * 256 + dg * 16);
    }
    __syncthreads();
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      int r, dg;
      chunk_of(it, r, dg);
      *reinterpret_cast<uint4*>(R0 + (r & 7) * 16 + (r >> 3) * 2048 + dg * 128) =
          r < L ? rk[it] : z;
      *reinterpret_cast<uint4*>(R0 + (r & 7) * 16 + ((r + 64) >> 3) * 2048 + dg * 128) =
          r < L ? rq[it] : z;
    }
  }
  fence_proxy_async();
  fence_before_sync();
  __syncthreads();
  // ---- [K; Q] K^T -> TMEM columns 0..63 (read by every value head)
  __shared__ int s_mma0;
  if (tid == 0) s_mma0 = 0;
  if (tid == 0 && !s_abort) {
    s_mma0 = 1;
    fence_after_sync();
    const uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint64_t ad = desc(smem_u32(R0) + ks * 256, 128, 2048);
      mma_f16(tb, ad, ad, id, ks > 0);  // B = rows 0-63 of the same operand (K)
    }
    commit(&bar[0]);
  }
  // ---- per value head, beside that MMA: V*beta MN-major (in place), K*beta*exp(gc)
  // MN-major, and the records' Q~ = Q exp(gc) and K~ = K exp(g_last - gc); read from the
  // [K; Q] operand (the MMA reads it too), scaled with packed fp16 multiplies
  for (int w = 0; w < NV; ++w) {
    const float* bt = btp(w);
    const float* eg = egp(w);
    const float* ek = ekp(w);
    uint8_t* rec = ws + ((int64_t)blockIdx.x * p.H_v + hv[w]) * REC_BYTES;
    uint8_t* xu = XU(w);
    uint8_t* xw = XW(w);
    uint4 rv[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      int r, dg;
      chunk_of(it, r, dg);
      rv[it] = *reinterpret_cast<const uint4*>(xu + r * 256 + dg * 16);
    }
    __syncthreads();
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      int r, dg;
      chunk_of(it, r, dg);
      const uint4 kv = *reinterpret_cast<const uint4*>(R0 + (r & 7) * 16 + (r >> 3) * 2048 + dg * 128);
      const bool in = r < L;
      *reinterpret_cast<uint4*>(xu + dg * 1024 + (r >> 3) * 128 + (r & 7) * 16) =
          in ? hscale8(rv[it], __float2half2_rn(bt[r])) : z;
      *reinterpret_cast<uint4*>(xw + dg * 1024 + (r >> 3) * 128 + (r & 7) * 16) =
          in ? hscale8(kv, __float2half2_rn(bt[r] * eg[r])) : z;
    }
    // the scan's operands Q~ = Q exp(gc) (rows 64.. of [W ; Q~]) and K~ = K exp(g_last - gc),
    // straight to the record: consecutive threads take consecutive 16-byte chunks of the
    // record, so every warp stores 512 contiguous bytes
#pragma unroll 4
    for (int it = 0; it < 8; ++it) {
      const int c = it * PREP_THREADS + tid;  // chunk of the 16 KB field
      // Q~: the same K-major canonical layout as the Q half of [K; Q]
      const int rq = (c >> 7) * 8 + (c & 7);
      const uint4 qv = *reinterpret_cast<const uint4*>(R0 + 16384 + c * 16);
      *reinterpret_cast<uint4*>(rec + REC_A1 + 16384 + c * 16) =
          rq < L ? hscale8(qv, __float2half2_rn(eg[rq])) : z;
      // K~: MN-major (M = d, K = token); chunk c holds token t's 8 features of group c / 64
      const int t = ((c >> 3) & 7) * 8 + (c & 7), dgr = c >> 6;
      const uint4 kv = *reinterpret_cast<const uint4*>(R0 + (t & 7) * 16 + (t >> 3) * 2048 + dgr * 128);
      *reinterpret_cast<uint4*>(rec + REC_AK + c * 16) =
          t < L ? hscale8(kv, __float2half2_rn(ek[t])) : z;
    }
  }
  fence_proxy_async();
  if (!mbar_wait(&bar[0], 0, &s_abort, wlim)) {
    set_status(p.status, GDN_ETIMEOUT);
    s_abort = 1;
    s_pend0 = 1;  // drained only if the MMA was issued (see the end)
  }
  fence_after_sync();
  __syncthreads();  // [K; Q] is no longer read: R0 is free for L, T and the staging

  __shared__ int s_mma1;
  for (int w = 0; w < NV; ++w) {
    const float* gc = gcp(w);
    const float* bt = btp(w);
    uint8_t* rec = ws + ((int64_t)blockIdx.x * p.H_v + hv[w]) * REC_BYTES;
    // ---- decay masks, L and P from [K K^T ; Q K^T] (TMEM columns 0..63)
    {
      const int row = warp * 32 + lane;
      const int i = row & 63;
      const float gi = gc[i], bi = bt[i];
      // rows 0-31 (warps 0 and 2) have no entries at columns >= 32: their L part is never
      // read and their P part is stored as zeros
      const int jpmax = (warp & 1) ? 4 : 2;
#pragma unroll 1
      for (int jp = 0; jp < jpmax; ++jp) {  // 16 columns of [K K^T ; Q K^T] at a time
        uint32_t r[16];
        tmem_ld16(taddr(tb, warp * 32, jp * 16), r);
        tmem_wait_ld();
#pragma unroll
        for (int hg = 0; hg < 2; ++hg) {
          const int jg = jp * 2 + hg;
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int jj = jg * 8 + e;
            const float dec = jj <= i ? __expf(gi - gc[jj]) : 0.f;  // masked before exp
            v[e] = __uint_as_float(r[hg * 8 + e]) * dec;
          }
          if (warp < 2) {  // L row i (strictly lower), beta_i on the left
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int jj = jg * 8 + e;
              Lf[i * LS + jj] = jj < i ? bi * v[e] : 0.f;
            }
          } else {         // P row i -> record, K-major canonical (LBO 128, SBO 1024)
            *reinterpret_cast<uint4*>(rec + REC_P + (i & 7) * 16 + (i >> 3) * 1024 + jg * 128) =
                pack8(v);
          }
        }
      }
      if (warp == 2) {
#pragma unroll
        for (int jg = 4; jg < 8; ++jg)
          *reinterpret_cast<uint4*>(rec + REC_P + (i & 7) * 16 + (i >> 3) * 1024 + jg * 128) =
              make_uint4(0, 0, 0, 0);
      }
    }
    fence_before_sync();
    __syncthreads();

    // ---- T = (I + L)^-1 (blocked), then T as the fp16 K-major B operand (N = i, K = j)
    tri_inverse_blocked(Lf, Tm, Xp);
#pragma unroll 1
    for (int e = tid; e < 64 * 8; e += PREP_THREADS) {
      const int i = e & 63, jg = e >> 6;  // 8 lanes = 8 rows: conflict-free 16-byte stores
      float tv[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) tv[x] = (jg * 8 + x <= i) ? Tm[i * TS + jg * 8 + x] : 0.f;
      *reinterpret_cast<uint4*>(Tb + (i & 7) * 16 + (i >> 3) * 1024 + jg * 128) = pack8(tv);
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();

    // ---- W^T = Xw^T T^T -> cols wc..wc+63 ; U^T = Xu^T T^T -> cols uc..uc+63 (NV = 1: U^T
    // over [K K^T ; Q K^T], whose last reader, the masks, finished before T was formed)
    if (tid == 0) s_mma1 = -1;
    if (tid == 0 && !s_abort) {
      s_mma1 = w;
      fence_after_sync();
      const uint32_t id = idesc_f16(128, 64, true, false);
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        const uint64_t bd = desc(smem_u32(Tb) + ks * 256, 128, 1024);
        mma_f16(tb + prep_w_col(NV), desc(smem_u32(XW(w)) + ks * 256, 128, 1024), bd, id,
                ks > 0);
        mma_f16(tb + prep_u_col(NV), desc(smem_u32(XU(w)) + ks * 256, 128, 1024), bd, id,
                ks > 0);
      }
      commit(&bar[1]);
    }
    __syncthreads();  // s_mma1 below
    if (!mbar_wait(&bar[1], w & 1, &s_abort, wlim)) {
      set_status(p.status, GDN_ETIMEOUT);
      if (s_mma1 == w) s_pend1 = w;  // that MMA is still to be drained
      s_abort = 1;
    }
    fence_after_sync();
    {
      // lane (feature) d holds W^T[d][i], U^T[d][i] for i = 0..63; stage W (K-major canonical
      // of the scan's [W; Q] operand) and U (4 MN-major column tiles) in the value head's
      // XW / XU operand buffers (the MMA that read them has completed), then bulk-copy out
      // while the next value head already uses R0. Lanes d and d + 1 (d even) swap half of
      // their values so that each writes 32-bit words holding columns d, d + 1 of one row i:
      // the even lane rows 8 ig + 0..3, the odd lane rows 8 ig + 4..7 (half the shared-memory
      // stores of one value per lane).
      const int d = warp * 32 + lane;
      const int dp = d & ~1;  // column pair
      const bool odd = (lane & 1) != 0;
      uint8_t* Wst = XW(w);
      uint8_t* Ust = XU(w);
#pragma unroll 1
      for (int ig = 0; ig < 8; ++ig) {
        uint32_t rw[8], ru[8];
        tmem_ld8(taddr(tb, warp * 32, prep_w_col(NV) + ig * 8), rw);
        tmem_ld8(taddr(tb, warp * 32, prep_u_col(NV) + ig * 8), ru);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // the partner needs, of this lane's rows, 8 ig + k (odd lane) or 8 ig + 4 + k (even)
          const float sw = __uint_as_float(odd ? rw[k] : rw[4 + k]);
          const float su = __uint_as_float(odd ? ru[k] : ru[4 + k]);
          const float pw = __shfl_xor_sync(0xffffffffu, sw, 1);
          const float pu = __shfl_xor_sync(0xffffffffu, su, 1);
          const float ow = __uint_as_float(odd ? rw[4 + k] : rw[k]);
          const float ou = __uint_as_float(odd ? ru[4 + k] : ru[k]);
          const int i = ig * 8 + (odd ? 4 + k : k);
          // low half = even column
          const __half2 hw = odd ? __floats2half2_rn(pw, ow) : __floats2half2_rn(ow, pw);
          const __half2 hu = odd ? __floats2half2_rn(pu, ou) : __floats2half2_rn(ou, pu);
          *reinterpret_cast<__half2*>(Wst + (i & 7) * 16 + (i >> 3) * 2048 + (dp >> 3) * 128 +
                                      (dp & 7) * 2) = hw;
          *reinterpret_cast<__half2*>(Ust + (dp >> 5) * 4096 + ((dp & 31) >> 3) * 1024 +
                                      (i >> 3) * 128 + (i & 7) * 16 + (dp & 7) * 2) = hu;
        }
      }
    }
    if (tid < C) reinterpret_cast<float*>(rec + REC_G)[tid] = gc[tid];
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      bulk_s2g(rec + REC_A1, XW(w), 16384);
      bulk_s2g(rec + REC_U, XU(w), 16384);
      bulk_commit();
    }
  }
  // the record stores must have read their shared-memory sources before the block ends
  if (tid == 0) bulk_wait_read_all();
  // a wait gave up: let every copy and MMA this block issued finish before its shared memory
  // and tensor memory are released (these waits use the default limit)
  if (tid == 0 && s_abort) {
    if (s_pend2) mbar_wait(&bar[2], 0, nullptr);
    if (s_pend0 && s_mma0) mbar_wait(&bar[0], 0, nullptr);
    if (s_pend1 >= 0) mbar_wait(&bar[1], s_pend1 & 1, nullptr);
    bulk_wait_all();
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, prep_tmem_cols(NV));
}

// Layer prefill: the new conv state of sequence n (the last 3 rows of [old state; x]) for the
// channels of v-head h, and of its k-head's q and k channels when h is the k-head's first
// v-head. Called by one warp of the (tile 0, h, n) scan block after griddepcontrol.wait, so the
// prep grid, which reads the old state, has completed. Each lane reads all three source rows of
// a channel group before writing the three new rows: a new row r comes from old row len + r.
__device__ void write_conv_state(const PrefillArgs& p, int n, int h, int64_t cs0, int64_t cs1,
                                 int slot, bool rst, int lane) {
  const int cdim = (2 * p.H_k + p.H_v) * D;
  const int hk = khead_of(h, p.H_k, p.H_v, p.layout);
  const int ngroups = first_vhead_of_khead(h, p.H_k, p.H_v, p.layout) ? 3 : 1;
  const int64_t len = cs1 - cs0;
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
  __nv_bfloat16* st = static_cast<__nv_bfloat16*>(p.conv_state) + (int64_t)slot * 3 * cdim;
  for (int e = lane; e < ngroups * 16; e += 32) {
    const int grp = e >> 4, cg = e & 15;
    const int ch0 = grp == 0 ? 2 * p.H_k * D + h * D : (grp == 1 ? hk * D : p.H_k * D + hk * D);
    const int ch = ch0 + cg * 8;
    uint4 v[3];
#pragma unroll
    for (int row = 0; row < 3; ++row) {
      const int64_t ei = len + row;  // row of [old state; x]
      if (ei < 3)
        v[row] = rst ? make_uint4(0, 0, 0, 0)
                     : *reinterpret_cast<const uint4*>(st + ei * cdim + ch);
      else
        v[row] = *reinterpret_cast<const uint4*>(x + (cs0 + ei - 3) * cdim + ch);
    }
#pragma unroll
    for (int row = 0; row < 3; ++row)
      *reinterpret_cast<uint4*>(st + (int64_t)row * cdim + ch) = v[row];
  }
}

// ======================================================================== scan kernel
// Warps 0-3 own the state tile (thread i = row i = TMEM lane i) and run the serial chain.
// One thread issues a tcgen05.mma only about every 100 cycles whatever its size, and two
// threads issue about twice as fast, so every MMA is split in two halves of its K range,
// issued by two threads into separate accumulators that the readers add: half hf of
// D1 = [W ; Q~] S covers d in [64 hf, 64 hf + 64) (threads 0 and 32), half hf of
// D2 = K~^T v_new covers tokens [32 hf, 32 hf + 32) (threads 0 and 32), half hf of the
// output term P v_new covers the same tokens and is added into D1 half hf by warps 5 and 8,
// off the chain.
// Warp 4: loader (bulk copies of a chunk's record slice up to NSTAGE chunks ahead).
// Warps 6, 7 (TMEM lanes 64-127): read each chunk's output rows and store them, off the chain.
// D1 is double-buffered by chunk parity; mbarriers that are waited on by another role than
// the chain are per buffer too, so that no waiter can miss a phase.
constexpr int SCAN_THREADS = 288;
constexpr long long kWaitCycles = 2000000000LL;  // about 1 s: a wait this long is an error
constexpr int NSTAGE = 3;
// per-stage shared memory (bytes): one bulk copy per record field
constexpr int ST_A1 = 0;        // 32768 [W ; Q~] K-major (LBO 128, SBO 2048)
constexpr int ST_AK = 32768;    // 16384 K~ MN-major (M = d, K = token; LBO 128, SBO 1024)
constexpr int ST_AP = 49152;    // 8192 P = rows 64..127 of a K-major operand whose rows 0..63
                                //      (the 8 KB before it, inside ST_AK) are never used
constexpr int ST_RU = 57344;    // 4096 the U tile, MN-major canonical (N = column, K = token)
constexpr int ST_GC = ST_RU + 4096;        // 64 fp32 g_cum
constexpr int ST_BYTES = ST_GC + 256;      // 61696 (a multiple of 128)
constexpr int SM_BS = NSTAGE * ST_BYTES;   // 8192 S as MN-major B (N = 32, K = 128; LBO 128, SBO 2048)
constexpr int SM_BV = SM_BS + 8192;        // 2 x 4096 v_new as MN-major B (N = 32, K = 64; LBO 128,
                                           //   SBO 1024), double-buffered by chunk parity
constexpr int SCAN_SMEM = SM_BV + 8192;    // 201472
// TMEM columns: D1 halves a and b, each double-buffered by chunk parity; D2 halves a and b
constexpr uint32_t TM_D1A = 0, TM_D1B = 64, TM_D2A = 128, TM_D2B = 160;
constexpr uint32_t SCAN_TMEM_COLS = 256;

// Longest first: the sequence whose length cu[m + 1] - cu[m] is the r-th largest of the
// call's (equal lengths in index order; a strict total order, so ranks 0 .. n_seqs - 1 map
// one to one onto the sequences). A grid whose block index r picks its sequence this way
// starts the longest serial chains first and lets the shorter ones fill in behind them
// (longest-processing-time-first list scheduling), since blocks are dispatched in index
// order. Calls of more than kLongestFirstMax sequences keep the identity: the ranking puts a
// dependent round trip to global memory and two barriers in front of every block, and in a
// 64-sequence batch of 60 single tokens and 4 prompts (2,048 scan blocks, most of which exit
// at once, one at a time per SM) that cost more than the order saved. Block-wide: every
// thread must call it.
constexpr int kLongestFirstMax = 16;
__device__ __forceinline__ int block_longest_first(const int32_t* cu, int n_seqs, int r) {
  if (n_seqs <= 1 || n_seqs > kLongestFirstMax) return r;
  __shared__ int s_len[kLongestFirstMax];
  __shared__ int s_pick;
  for (int m = threadIdx.x; m < n_seqs; m += blockDim.x) s_len[m] = cu[m + 1] - cu[m];
  __syncthreads();
  for (int m = threadIdx.x; m < n_seqs; m += blockDim.x) {
    const int lm = s_len[m];
    int rank = 0;
    for (int j = 0; j < n_seqs; ++j) {
      const int lj = s_len[j];
      rank += (lj > lm || (lj == lm && j < m)) ? 1 : 0;
    }
    if (rank == r) s_pick = m;
  }
  __syncthreads();
  return s_pick;
}

__global__ void __launch_bounds__(SCAN_THREADS, 1)
tc_scan_kernel(const PrefillArgs p, const uint8_t* ws, int64_t max_chunks) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t loaded[NSTAGE], empty[NSTAGE], mma_a[2], mma_b[2], mma_bo[2], mma_c[2];
  __shared__ uint64_t o_done[2];
  __shared__ uint32_t s_tbase;
  __shared__ int64_t s_red[SCAN_THREADS / 32];
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x, h = blockIdx.y;
  const int n = block_longest_first(p.cu_seqlens, p.n_seqs, blockIdx.z);

  const int64_t cs0 = p.cu_seqlens[n], cs1 = p.cu_seqlens[n + 1];
  const bool ok = cs0 >= 0 && cs1 >= cs0 && cs1 <= p.T_total;
  const int slot = p.slot_ids[n];
  if (slot < 0 || slot >= p.n_slots) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  if (!ok) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_EINVAL);
    return;
  }
  // short sequences belong to the token-by-token kernel of the same call
  if (p.short_max > 0 && cs1 - cs0 <= p.short_max) return;
  // a slot repeated within the call: only its first sequence updates it (and, in the layer
  // prefill, rolls its conv state); every block of a later one skips it
  if (block_slot_taken(p.slot_ids, n, slot)) {
    if (tid == 0 && h == 0 && tile == 0) set_status(p.status, GDN_ESLOT);
    return;
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
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&loaded[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mma_a[b], 1);   // per MMA half
      mbar_init(&mma_b[b], 1);   // per MMA half
      mbar_init(&mma_bo[b], 2);  // per buffer: both halves of the chunk's D2 MMA are done
      mbar_init(&mma_c[b], 2);   // per D1 buffer: both halves of the chunk's output MMA are done
      mbar_init(&o_done[b], 2);  // per D1 buffer: both output warps have read it
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s_tbase, SCAN_TMEM_COLS);
    tmem_relinquish();  // lets the next block be placed on this SM (see the prep kernel)
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = s_tbase;
  uint8_t* BS = sm + SM_BS;
  uint8_t* BV = sm + SM_BV;
  auto fail = [&]() {
    set_status(p.status, GDN_ETIMEOUT);
    s_abort = 1;
  };

  if (warp == 4) {
    if (p.fused && tile == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      write_conv_state(p, n, h, cs0, cs1, slot, rst, lane);
    }
    // ================= loader: bulk copies of chunk c into stage c % NSTAGE
    if (lane == 0) {
      // the records come from the prep kernel, which may still be running when this grid
      // starts (programmatic dependent launch): wait for it to complete
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int c = 0; c < nck; ++c) {
        const int s = c % NSTAGE;
        uint8_t* st = sm + s * ST_BYTES;
        if (c >= NSTAGE &&
            !mbar_wait(&empty[s], ((c / NSTAGE) - 1) & 1, &s_abort, kWaitCycles, 256))
          fail();
        if (s_abort) break;
        const uint8_t* rec = ws + ((base + c) * p.H_v + h) * REC_BYTES;
        mbar_arrive_expect_tx(&loaded[s], 32768 + 16384 + 8192 + 4096 + 256);
        bulk_g2s(st + ST_A1, rec + REC_A1, 32768, &loaded[s]);
        bulk_g2s(st + ST_AK, rec + REC_AK, 16384, &loaded[s]);
        bulk_g2s(st + ST_AP, rec + REC_P, 8192, &loaded[s]);
        bulk_g2s(st + ST_RU, rec + REC_U + tile * 4096, 4096, &loaded[s]);
        bulk_g2s(st + ST_GC, rec + REC_G, 256, &loaded[s]);
      }
      // drain: copies still in flight must land before the block may exit
      for (int c = nck > NSTAGE ? nck - NSTAGE : 0; c < nck; ++c)
        mbar_wait(&loaded[c % NSTAGE], (c / NSTAGE) & 1, nullptr, 200000000LL);
    }
  } else if (warp == 5 || warp == 8) {
    // ================= output MMA halves: D1 half hf rows 64-127 += P v_new over tokens
    // [32 hf, 32 hf + 32), after chunk c's serial MMAs (the operand rows 0-63 are the unused
    // bytes before P)
    if (lane == 0) {
      const int hf = warp == 5 ? 0 : 1;
      const uint32_t id_a = idesc_f16(128, TILE, false, true);
      for (int c = 0; c < nck; ++c) {
        uint8_t* st = sm + (c % NSTAGE) * ST_BYTES;
        if (!mbar_wait(&mma_bo[c & 1], (c >> 1) & 1, &s_abort, kWaitCycles, 64)) fail();
        fence_after_sync();
        if (s_abort) break;
        const uint64_t ap = desc(smem_u32(st + ST_AP) - 8192 + hf * 512, 128, 1024);
        const uint64_t bv = desc(smem_u32(BV) + (c & 1) * 4096 + hf * 512, 128, 1024);
        const uint32_t d1 = (hf ? TM_D1B : TM_D1A) + (c & 1) * 32;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) mma_f16(tb + d1, ap + 16 * ks, bv + 16 * ks, id_a, 1);
        commit(&mma_c[c & 1]);
      }
    }
  } else if (warp == 6 || warp == 7) {
    // ================= output rows of chunk c = D1a + D1b of buffer (c & 1), TMEM lanes 64-127
    const int t = (warp - 4) * 32 + lane - 64;  // token row within the chunk
    for (int c = 0; c < nck; ++c) {
      const uint32_t b = c & 1;
      if (!mbar_wait(&mma_c[b], (c >> 1) & 1, &s_abort, kWaitCycles, 128)) fail();
      fence_after_sync();
      if (s_abort) break;
      // every MMA of chunk c is done: its stage can be refilled
      if (tid == 192) mbar_arrive(&empty[c % NSTAGE]);
      uint32_t ra[32], rb[32];
      tmem_ld32(taddr(tb, (warp - 4) * 32, TM_D1A + b * 32), ra);
      tmem_ld32(taddr(tb, (warp - 4) * 32, TM_D1B + b * 32), rb);
      tmem_wait_ld();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_done[b]);  // the buffer may be overwritten
      const int64_t c0 = cs0 + (int64_t)c * C;
      const int L = (cs1 - c0) < C ? (int)(cs1 - c0) : C;
      if (t < L) {
        const int64_t off = ((c0 + t) * p.H_v + h) * p.d_v + tile * TILE;
        float ov[TILE];
#pragma unroll
        for (int x = 0; x < TILE; ++x) ov[x] = __uint_as_float(ra[x]) + __uint_as_float(rb[x]);
        if (p.o_dtype == GDN_BF16) {
          uint4* ob = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + off);
#pragma unroll
          for (int x = 0; x < TILE; x += 8) {
            uint4 u;
            __nv_bfloat162* hb = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) hb[e] = __floats2bfloat162_rn(ov[x + 2 * e], ov[x + 2 * e + 1]);
            ob[x / 8] = u;
          }
        } else {
          float* of = static_cast<float*>(p.o) + off;
#pragma unroll
          for (int x = 0; x < TILE; x += 4)
            st4(of + x, make_float4(ov[x], ov[x + 1], ov[x + 2], ov[x + 3]));
        }
      }
    }
  } else if (warp < 4) {
    // ================= chain: state tile rows in registers
    const int i = tid;    // S row = TMEM lane
    const int hf = warp;  // MMA half issued by threads 0 and 32
    const bool issuer = lane == 0 && warp < 2;
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
    for (int c = 0; c < nck; ++c) {
      const int s = c % NSTAGE;
      uint8_t* st = sm + s * ST_BYTES;
      const uint32_t b = c & 1;
      if (!mbar_wait(&loaded[s], (c / NSTAGE) & 1, &s_abort)) fail();
      const int64_t c0 = cs0 + (int64_t)c * C;
      const int L = (cs1 - c0) < C ? (int)(cs1 - c0) : C;
      const float el = expf(reinterpret_cast<const float*>(st + ST_GC)[L - 1]);
      // (1) S -> fp16 MN-major B operand
#pragma unroll
      for (int jg = 0; jg < TILE / 8; ++jg)
        *reinterpret_cast<uint4*>(BS + jg * 2048 + (i >> 3) * 128 + (i & 7) * 16) =
            pack8(srow + jg * 8);
      fence_proxy_async();
      fence_before_sync();
      named_bar(1, 128);
      // (2) D1 half hf = [W ; Q~][:, 64 hf : 64 hf + 64] S[64 hf : 64 hf + 64, :], into
      // buffer b (the issuer has seen the output warps release it after chunk c - 2)
      if (issuer) {
        fence_after_sync();
        if (!s_abort) {
          // a K step of 16 moves both operands by 256 bytes = 16 in the address field
          const uint64_t a0 = desc(smem_u32(st + ST_A1) + hf * 1024, 128, 2048);
          const uint64_t b0 = desc(smem_u32(BS) + hf * 1024, 128, 2048);
          const uint32_t d1 = (hf ? TM_D1B : TM_D1A) + b * 32;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16(tb + d1, a0 + 16 * ks, b0 + 16 * ks, id_a, ks > 0);
          commit(&mma_a[hf]);
        }
      }
      // the issuing lane's warp-mates wait here rather than poll beside it
      __syncwarp();
      if (!mbar_wait(&mma_a[0], c & 1, &s_abort) || !mbar_wait(&mma_a[1], c & 1, &s_abort))
        fail();
      fence_after_sync();
      // (3) v_new = U - D1[0:64] -> fp16 MN-major B operand buffer b (warps 0, 1: TMEM lanes
      // 0-63). The output MMA of chunk c - 2, the last reader of that buffer, is complete:
      // the output warps released D1 buffer b only after it, and MMA-A of chunk c was issued
      // only after that release.
      if (warp < 2) {
        uint32_t ra[32], rb[32];
        tmem_ld32(taddr(tb, warp * 32, TM_D1A + b * 32), ra);
        tmem_ld32(taddr(tb, warp * 32, TM_D1B + b * 32), rb);
        tmem_wait_ld();
        const int t = i;
        // U row t: 8 columns per 16-byte chunk, column group q4 at q4 * 1024
        const uint8_t* up = st + ST_RU + (t >> 3) * 128 + (t & 7) * 16;
        float vn[TILE];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 u = *reinterpret_cast<const uint4*>(up + q4 * 1024);
          const __half2* hu = reinterpret_cast<const __half2*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(hu[e]);
            const int x = q4 * 8 + e * 2;
            vn[x] = (t < L) ? f.x - __uint_as_float(ra[x]) - __uint_as_float(rb[x]) : 0.f;
            vn[x + 1] =
                (t < L) ? f.y - __uint_as_float(ra[x + 1]) - __uint_as_float(rb[x + 1]) : 0.f;
          }
        }
#pragma unroll
        for (int jg = 0; jg < TILE / 8; ++jg)
          *reinterpret_cast<uint4*>(BV + b * 4096 + jg * 1024 + (t >> 3) * 128 + (t & 7) * 16) =
              pack8(vn + jg * 8);
        fence_proxy_async();
      }
      fence_before_sync();
      named_bar(1, 128);
      // (4) D2 half hf = K~^T v_new over tokens [32 hf, 32 hf + 32)
      if (issuer) {
        fence_after_sync();
        if (!s_abort) {
          const uint64_t ak = desc(smem_u32(st + ST_AK) + hf * 512, 128, 1024);
          const uint64_t bv = desc(smem_u32(BV) + b * 4096 + hf * 512, 128, 1024);
          const uint32_t d2 = hf ? TM_D2B : TM_D2A;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
            mma_f16(tb + d2, ak + 16 * ks, bv + 16 * ks, id_k, ks > 0);
          commit(&mma_b[hf]);
          commit(&mma_bo[b]);
        }
        // D1 buffer of chunk c + 1 is free once the output warps have read chunk c - 1 from
        // it; checked here, in the shadow of this chunk's MMA-B
        if (c >= 1 && c + 1 < nck &&
            !mbar_wait(&o_done[(c + 1) & 1], (((c + 1) >> 1) - 1) & 1, &s_abort))
          fail();
      }
      __syncwarp();
      if (!mbar_wait(&mma_b[0], c & 1, &s_abort) || !mbar_wait(&mma_b[1], c & 1, &s_abort))
        fail();
      fence_after_sync();
      // (5) S = exp(g_last) S + D2
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(taddr(tb, warp * 32, TM_D2A), ra);
        tmem_ld32(taddr(tb, warp * 32, TM_D2B), rb);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < TILE; ++x)
          srow[x] = fmaf(el, srow[x], __uint_as_float(ra[x]) + __uint_as_float(rb[x]));
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
  if (warp == 0) tmem_dealloc(tb, SCAN_TMEM_COLS);
}

// ======================================================================== whole-head scan
// One CTA per (sequence, value head): the whole 128 x 128 state, so every tensor-core
// instruction of the chain covers all 128 columns (N = 128) -- four times the work of the
// 32-column tile kernel's per instruction at about the same issue cost -- and the records are
// read once per head instead of once per column tile.
// Warps 0-7 hold the fp32 state: thread = row r = 32 (w % 4) + lane (= TMEM lane), columns
// 64 (w / 4) .. +64. Chain per chunk, every MMA split over two issuing threads (warps 0 and
// 4, lane 0) by halves of its K range into separate accumulators that the readers add:
//   D1 = [W ; Q~] S            (M=128, N=128, K=128)     v_new = U - D1[0:64]
//   D2 = K~^T v_new            (M=128, N=128, K=64)      S = exp(g_last) S + D2
// Off the chain: warps 10 and 11 (TMEM lanes 64-127) first add P v_new into D1 rows 64-127
// (lane 0 of each issues one half of its token range), then read and store o; warp 8
// bulk-copies the records into HS_NSTAGE stages; warp 9 has no role (it only keeps the output
// warps in the TMEM lane quadrants 2 and 3). D1 is single-buffered: its next MMA waits until
// the output warps have read it.
constexpr int HS_THREADS = 384;  // 12 warps
constexpr int HS_NSTAGE = 2;
constexpr int HS_A1 = 0;         // 32768 [W ; Q~] K-major (LBO 128, SBO 2048)
constexpr int HS_AK = 32768;     // 16384 K~ MN-major (M = d, K = token; LBO 128, SBO 1024)
constexpr int HS_AP = 49152;     // 8192 P = rows 64..127 of a K-major operand (rows 0..63 are
                                 //      the 8 KB before it, never used)
constexpr int HS_RU = 57344;     // 16384 U as 4 column tiles, each MN-major canonical
constexpr int HS_GC = HS_RU + 16384;         // 64 fp32 g_cum
constexpr int HS_ST = HS_GC + 256;           // 74240 per stage (a multiple of 128)
constexpr int HS_BS = HS_NSTAGE * HS_ST;     // 32768 S as MN-major B (N = 128, K = 128; LBO 128,
                                             //   SBO 2048)
constexpr int HS_BV = HS_BS + 32768;         // 16384 v_new as MN-major B (N = 128, K = 64; LBO
                                             //   128, SBO 1024)
constexpr int HS_SMEM = HS_BV + 16384;       // 197632
// TMEM columns: the two K halves of D1 and of D2, 128 columns each
constexpr uint32_t HS_D1A = 0, HS_D1B = 128, HS_D2A = 256, HS_D2B = 384;
constexpr uint32_t HS_TMEM_COLS = 512;

__global__ void __launch_bounds__(HS_THREADS, 1)
tc_scan_head_kernel(const PrefillArgs p, const uint8_t* ws, int64_t max_chunks) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t loaded[HS_NSTAGE], empty[HS_NSTAGE], mma_a[2], mma_b[2];
  __shared__ uint64_t mma_bo, mma_c, o_done;
  __shared__ uint32_t s_tbase;
  __shared__ int64_t s_red[HS_THREADS / 32];
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const int n = block_longest_first(p.cu_seqlens, p.n_seqs, blockIdx.z);

  const int64_t cs0 = p.cu_seqlens[n], cs1 = p.cu_seqlens[n + 1];
  const bool ok = cs0 >= 0 && cs1 >= cs0 && cs1 <= p.T_total;
  const int slot = p.slot_ids[n];
  if (slot < 0 || slot >= p.n_slots) {
    if (tid == 0 && h == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  if (!ok) {
    if (tid == 0 && h == 0) set_status(p.status, GDN_EINVAL);
    return;
  }
  // short sequences belong to the token-by-token kernel of the same call
  if (p.short_max > 0 && cs1 - cs0 <= p.short_max) return;
  // a slot repeated within the call: only its first sequence updates it (and, in the layer
  // prefill, rolls its conv state); every block of a later one skips it
  if (block_slot_taken(p.slot_ids, n, slot)) {
    if (tid == 0 && h == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  const int64_t base = block_segment_base<HS_THREADS>(p.cu_seqlens, n, p.T_total, C, s_red);
  const int nck = (int)((cs1 - cs0 + C - 1) / C);
  if (base + nck > max_chunks) {
    if (tid == 0) set_status(p.status, GDN_EINVAL);
    return;
  }
  const bool rst = p.reset != nullptr && p.reset[n] != 0;
  float* Sg = p.state + (((int64_t)slot * p.H_v + h) * D) * p.d_v;

  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < HS_NSTAGE; ++s) {
      mbar_init(&loaded[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mma_a[b], 1);
      mbar_init(&mma_b[b], 1);
    }
    mbar_init(&mma_bo, 2);  // both halves of the chunk's D2 MMA are issued (v_new is ready)
    mbar_init(&mma_c, 2);   // both halves of the chunk's output MMA are done
    mbar_init(&o_done, 2);  // both output warps have read D1
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s_tbase, HS_TMEM_COLS);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = s_tbase;
  uint8_t* BS = sm + HS_BS;
  uint8_t* BV = sm + HS_BV;
  auto fail = [&]() {
    set_status(p.status, GDN_ETIMEOUT);
    s_abort = 1;
  };

  if (warp == 8) {
    if (p.fused) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      write_conv_state(p, n, h, cs0, cs1, slot, rst, lane);
    }
    // ================= loader: bulk copies of chunk c into stage c % HS_NSTAGE
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int issued = 0;
      for (int c = 0; c < nck; ++c) {
        const int s = c % HS_NSTAGE;
        uint8_t* st = sm + s * HS_ST;
        if (c >= HS_NSTAGE &&
            !mbar_wait(&empty[s], ((c / HS_NSTAGE) - 1) & 1, &s_abort, kWaitCycles, 256))
          fail();
        if (s_abort) break;
        const uint8_t* rec = ws + ((base + c) * p.H_v + h) * REC_BYTES;
        mbar_arrive_expect_tx(&loaded[s], 32768 + 16384 + 8192 + 16384 + 256);
        bulk_g2s(st + HS_A1, rec + REC_A1, 32768, &loaded[s]);
        bulk_g2s(st + HS_AK, rec + REC_AK, 16384, &loaded[s]);
        bulk_g2s(st + HS_AP, rec + REC_P, 8192, &loaded[s]);
        bulk_g2s(st + HS_RU, rec + REC_U, 16384, &loaded[s]);
        bulk_g2s(st + HS_GC, rec + REC_G, 256, &loaded[s]);
        issued = c + 1;
      }
      // drain: copies still in flight must land before the block may exit
      for (int c = issued > HS_NSTAGE ? issued - HS_NSTAGE : 0; c < issued; ++c)
        mbar_wait(&loaded[c % HS_NSTAGE], (c / HS_NSTAGE) & 1, nullptr, 200000000LL);
    }
  } else if (warp == 10 || warp == 11) {
    // ================= output: D1 half hf rows 64-127 += P v_new over tokens [32 hf, 32 hf
    // + 32) once chunk c's v_new is in place (the chain has read D1 rows 0-63), then o rows
    // of chunk c = D1a + D1b rows 64-127 (TMEM lanes 64-127)
    const int hf = warp - 10;
    const int t = hf * 32 + lane;  // token row within the chunk
    const uint32_t id_a = idesc_f16(128, 128, false, true);
    for (int c = 0; c < nck; ++c) {
      if (lane == 0) {
        uint8_t* st = sm + (c % HS_NSTAGE) * HS_ST;
        if (!mbar_wait(&mma_bo, c & 1, &s_abort, kWaitCycles, 64)) fail();
        fence_after_sync();
        if (!s_abort) {
          const uint64_t ap = desc(smem_u32(st + HS_AP) - 8192 + hf * 512, 128, 1024);
          const uint64_t bv = desc(smem_u32(BV) + hf * 512, 128, 1024);
          const uint32_t d1 = hf ? HS_D1B : HS_D1A;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) mma_f16(tb + d1, ap + 16 * ks, bv + 16 * ks, id_a, 1);
          commit(&mma_c);
        }
      }
      __syncwarp();
      if (!mbar_wait(&mma_c, c & 1, &s_abort, kWaitCycles, 128)) fail();
      fence_after_sync();
      if (s_abort) break;
      // every MMA of chunk c is done: its stage can be refilled
      if (tid == 320) mbar_arrive(&empty[c % HS_NSTAGE]);
      const int64_t c0 = cs0 + (int64_t)c * C;
      const int L = (cs1 - c0) < C ? (int)(cs1 - c0) : C;
      const int64_t off = ((c0 + t) * p.H_v + h) * p.d_v;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {  // 32 columns at a time
        uint32_t ra[32], rb[32];
        tmem_ld32(taddr(tb, (warp - 8) * 32, HS_D1A + q * 32), ra);
        tmem_ld32(taddr(tb, (warp - 8) * 32, HS_D1B + q * 32), rb);
        tmem_wait_ld();
        if (t < L) {
          float ov[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) ov[x] = __uint_as_float(ra[x]) + __uint_as_float(rb[x]);
          if (p.o_dtype == GDN_BF16) {
            uint4* ob = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + off + q * 32);
#pragma unroll
            for (int x = 0; x < 32; x += 8) {
              uint4 u;
              __nv_bfloat162* hb = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                hb[e] = __floats2bfloat162_rn(ov[x + 2 * e], ov[x + 2 * e + 1]);
              ob[x / 8] = u;
            }
          } else {
            float* of = static_cast<float*>(p.o) + off + q * 32;
#pragma unroll
            for (int x = 0; x < 32; x += 4)
              st4(of + x, make_float4(ov[x], ov[x + 1], ov[x + 2], ov[x + 3]));
          }
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_done);  // D1 may be overwritten
    }
  } else if (warp < 8) {
    // ================= chain: state rows in registers, 64 columns per thread
    const int q4 = warp & 3, ch = warp >> 2;
    const int i = q4 * 32 + lane;   // S row = TMEM lane
    const int col0 = ch * 64;       // this thread's column half
    const bool issuer = lane == 0 && q4 == 0;  // warps 0 and 4: K half ch
    const int hf = ch;
    float srow[64];
    if (rst) {
#pragma unroll
      for (int x = 0; x < 64; ++x) srow[x] = 0.f;
    } else {
#pragma unroll
      for (int x = 0; x < 64; x += 4) {
        float4 v = *reinterpret_cast<const float4*>(Sg + (int64_t)i * p.d_v + col0 + x);
        srow[x] = v.x; srow[x + 1] = v.y; srow[x + 2] = v.z; srow[x + 3] = v.w;
      }
    }
    const uint32_t id_a = idesc_f16(128, 128, false, true);
    const uint32_t id_k = idesc_f16(128, 128, true, true);
    for (int c = 0; c < nck; ++c) {
      const int s = c % HS_NSTAGE;
      uint8_t* st = sm + s * HS_ST;
      if (!mbar_wait(&loaded[s], (c / HS_NSTAGE) & 1, &s_abort)) fail();
      const int64_t c0 = cs0 + (int64_t)c * C;
      const int L = (cs1 - c0) < C ? (int)(cs1 - c0) : C;
      const float el = expf(reinterpret_cast<const float*>(st + HS_GC)[L - 1]);
      // (1) S -> fp16 MN-major B operand: row i, columns col0 .. col0 + 63 (8 column groups)
#pragma unroll
      for (int jg = 0; jg < 8; ++jg)
        *reinterpret_cast<uint4*>(BS + (col0 / 8 + jg) * 2048 + (i >> 3) * 128 + (i & 7) * 16) =
            pack8(srow + jg * 8);
      fence_proxy_async();
      fence_before_sync();
      named_bar(1, 256);
      // (2) D1 half hf = [W ; Q~][:, 64 hf : 64 hf + 64] S[64 hf : 64 hf + 64, :], once the
      // output warps have read chunk c - 1's D1
      if (issuer) {
        if (c >= 1 && !mbar_wait(&o_done, (c - 1) & 1, &s_abort)) fail();
        fence_after_sync();
        if (!s_abort) {
          const uint64_t a0 = desc(smem_u32(st + HS_A1) + hf * 1024, 128, 2048);
          const uint64_t b0 = desc(smem_u32(BS) + hf * 1024, 128, 2048);
          const uint32_t d1 = hf ? HS_D1B : HS_D1A;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16(tb + d1, a0 + 16 * ks, b0 + 16 * ks, id_a, ks > 0);
          commit(&mma_a[hf]);
        }
      }
      __syncwarp();
      if (!mbar_wait(&mma_a[0], c & 1, &s_abort) || !mbar_wait(&mma_a[1], c & 1, &s_abort))
        fail();
      fence_after_sync();
      // (3) v_new = U - D1[0:64] for this thread's 64 columns -> fp16 MN-major B operand
      // (warps 0, 1, 4, 5: TMEM lanes 0-63). The previous output MMA, the last reader of
      // BV, completed before the output warps released D1, and D1 was issued after that.
      if (q4 < 2) {
        const int t = i;
#pragma unroll 1
        for (int hq = 0; hq < 4; ++hq) {  // 16 columns at a time
          const int cb = col0 + hq * 16;
          uint32_t ra[16], rb[16];
          tmem_ld16(taddr(tb, q4 * 32, HS_D1A + cb), ra);
          tmem_ld16(taddr(tb, q4 * 32, HS_D1B + cb), rb);
          tmem_wait_ld();
          // U row t, columns cb .. cb + 15: column tile cb / 32 (4 KB each), its column groups
          // (cb % 32) / 8 and the next (1 KB apart)
          const uint8_t* up =
              st + HS_RU + (cb / 32) * 4096 + ((cb % 32) / 8) * 1024 + (t >> 3) * 128 + (t & 7) * 16;
          float vn[16];
#pragma unroll
          for (int g2 = 0; g2 < 2; ++g2) {
            const uint4 u = *reinterpret_cast<const uint4*>(up + g2 * 1024);
            const __half2* hu = reinterpret_cast<const __half2*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(hu[e]);
              const int x = g2 * 8 + e * 2;
              vn[x] = (t < L) ? f.x - __uint_as_float(ra[x]) - __uint_as_float(rb[x]) : 0.f;
              vn[x + 1] =
                  (t < L) ? f.y - __uint_as_float(ra[x + 1]) - __uint_as_float(rb[x + 1]) : 0.f;
            }
          }
#pragma unroll
          for (int jg = 0; jg < 2; ++jg)
            *reinterpret_cast<uint4*>(BV + (cb / 8 + jg) * 1024 + (t >> 3) * 128 + (t & 7) * 16) =
                pack8(vn + jg * 8);
        }
        fence_proxy_async();
      }
      fence_before_sync();
      named_bar(1, 256);
      // (4) D2 half hf = K~^T v_new over tokens [32 hf, 32 hf + 32)
      if (issuer) {
        fence_after_sync();
        if (!s_abort) {
          const uint64_t ak = desc(smem_u32(st + HS_AK) + hf * 512, 128, 1024);
          const uint64_t bv = desc(smem_u32(BV) + hf * 512, 128, 1024);
          const uint32_t d2 = hf ? HS_D2B : HS_D2A;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
            mma_f16(tb + d2, ak + 16 * ks, bv + 16 * ks, id_k, ks > 0);
          commit(&mma_b[hf]);
          commit(&mma_bo);
        }
      }
      __syncwarp();
      if (!mbar_wait(&mma_b[0], c & 1, &s_abort) || !mbar_wait(&mma_b[1], c & 1, &s_abort))
        fail();
      fence_after_sync();
      // (5) S = exp(g_last) S + D2, 16 columns at a time
#pragma unroll
      for (int hq = 0; hq < 4; ++hq) {
        uint32_t ra[16], rb[16];
        tmem_ld16(taddr(tb, q4 * 32, HS_D2A + col0 + hq * 16), ra);
        tmem_ld16(taddr(tb, q4 * 32, HS_D2B + col0 + hq * 16), rb);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x)
          srow[hq * 16 + x] =
              fmaf(el, srow[hq * 16 + x], __uint_as_float(ra[x]) + __uint_as_float(rb[x]));
      }
      fence_before_sync();
    }
    if (!s_abort) {
#pragma unroll
      for (int x = 0; x < 64; x += 4)
        *reinterpret_cast<float4*>(Sg + (int64_t)i * p.d_v + col0 + x) =
            make_float4(srow[x], srow[x + 1], srow[x + 2], srow[x + 3]);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, HS_TMEM_COLS);
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

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// fp16 [T][H][128] viewed as a 3-D tensor (128, H, T); box = one head's 64 consecutive tokens.
cudaError_t make_head_map(CUtensorMap* m, const void* base, int H, int64_t T) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)(T > 0 ? T : 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  const cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)C};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
// bf16 x [T][conv_dim] as a 2-D tensor (conv_dim, T); box = 128 channels x (64 + 3) rows.
cudaError_t make_x_map(CUtensorMap* m, const void* base, int cdim, int64_t T) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cdim, (cuuint64_t)(T > 0 ? T : 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)cdim * 2};
  const cuuint32_t box[2] = {(cuuint32_t)D, (cuuint32_t)XT_ROWS};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
  if (!prefill_tc_supported(a.d_k, a.d_v, a.chunk, a.qkv_dtype)) return cudaErrorNotSupported;
  const int64_t max_chunks = (a.T_total + C - 1) / C + a.n_seqs;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  alignas(64) CUtensorMap tm_q{}, tm_k{}, tm_v{}, tm_x{};
  if (a.T_total > 0) {
    cudaError_t em = cudaSuccess;
    if (a.fused) {
      em = make_x_map(&tm_x, a.x, (2 * a.H_k + a.H_v) * D, a.T_total);
    } else {
      em = make_head_map(&tm_q, a.q, a.H_k, a.T_total);
      if (em == cudaSuccess) em = make_head_map(&tm_k, a.k, a.H_k, a.T_total);
      if (em == cudaSuccess) em = make_head_map(&tm_v, a.v, a.H_v, a.T_total);
    }
    if (em != cudaSuccess) return em;
  }
  int dev = 0, sms = 0;
  {
    cudaError_t ea = cudaGetDevice(&dev);
    if (ea == cudaSuccess) ea = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (ea != cudaSuccess) return ea;
  }
  // one prep block per (chunk, key head) when each key head has two value heads, except for
  // the q / k / v prefill of a grid of value-head blocks that fills kPrepPerValueHeadMinWaves
  // waves at three blocks per SM
  const bool pair = a.H_v == 2 * a.H_k &&
                    (a.fused || max_chunks * a.H_v <
                                    (int64_t)kPrepPerValueHeadMinWaves * prep_min_blocks(1) * sms);
  auto prep = a.fused ? (pair ? tc_prep_kernel<true, 2> : tc_prep_kernel<true, 1>)
                      : (pair ? tc_prep_kernel<false, 2> : tc_prep_kernel<false, 1>);
  const int prep_bytes = prep_smem(pair ? 2 : 1);
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       prep_bytes);
  if (e != cudaSuccess) return e;
  // the whole unified L1 / shared array as shared memory, so two prep blocks fit per SM
  e = cudaFuncSetAttribute(prep, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  bool head = (a.flags & GDN_PREFILL_TC_HEAD_SCAN) != 0;
  if (!head && !(a.flags & GDN_PREFILL_TC_TILE_SCAN)) {
    // the whole-head scan (a chunk step about 2.5 times longer, a quarter of the CTAs, one
    // CTA per SM either way) wins once the tile scan needs more than two waves
    head = (int64_t)(a.d_v / TILE) * a.n_seqs * a.H_v > 2LL * sms;
  }
  e = head ? cudaFuncSetAttribute(tc_scan_head_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, HS_SMEM)
           : cudaFuncSetAttribute(tc_scan_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, SCAN_SMEM);
  if (e != cudaSuccess) return e;
  if (max_chunks > 0) {
    dim3 g1((unsigned)max_chunks, pair ? a.H_k : a.H_v);
    prep<<<g1, PREP_THREADS, prep_bytes, s>>>(a, ws, max_chunks, tm_q, tm_k, tm_v, tm_x);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // programmatic dependent launch: the scan's prologue (barriers, TMEM, state loads) overlaps
  // the tail of the prep grid; its loader waits for the prep grid before reading records
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(head ? 1 : a.d_v / TILE, a.H_v, a.n_seqs);
  cfg.blockDim = dim3(head ? HS_THREADS : SCAN_THREADS);
  cfg.dynamicSmemBytes = head ? HS_SMEM : SCAN_SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (head)
    return cudaLaunchKernelEx(&cfg, tc_scan_head_kernel, a, static_cast<const uint8_t*>(ws),
                              max_chunks);
  return cudaLaunchKernelEx(&cfg, tc_scan_kernel, a, static_cast<const uint8_t*>(ws), max_chunks);
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

namespace {
// Unique id of the current CUDA context (driver entry points looked up through the runtime,
// so the library needs no link-time dependency on the driver library).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
cudaError_t current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  if (!get_current || !get_id) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
  if (get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  return cudaSuccess;
}
}  // namespace

cudaError_t launch_prefill_tc_noalloc(const PrefillArgs& a, cudaStream_t s) {
  if (!prefill_tc_supported(a.d_k, a.d_v, a.chunk, a.qkv_dtype)) return cudaErrorNotSupported;
  if (prefill_tc_workspace(a.H_v, a.d_k, a.d_v, a.T_total, a.n_seqs, a.chunk) >
      kNoAllocScratchBytes)
    return cudaErrorInvalidValue;
  // The array's device address, looked up with the device current (the host-side name is
  // only a stand-in and must never reach a kernel). It is cached per device together with the
  // id of the context it was looked up in: a context torn down and created again (for example
  // after cudaDeviceReset) loads the module anew, so a new context id means a new lookup.
  constexpr int kMaxDev = 64;
  static void* addr[kMaxDev] = {};
  static unsigned long long ctx_id[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    unsigned long long id = 0;
    // no current context yet (the runtime creates it lazily): the lookup below creates it
    const bool have_ctx = current_context_id(&id) == cudaSuccess;
    if (!have_ctx || !addr[dev] || ctx_id[dev] != id) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return e;
      e = current_context_id(&id);
      if (e != cudaSuccess) return e;
      addr[dev] = p;
      ctx_id[dev] = id;
    }
    scratch = addr[dev];
  }
  PrefillArgs b = a;
  b.workspace = scratch;
  b.workspace_bytes = kNoAllocScratchBytes;
  return launch_prefill_tc(b, s);
}

}  // namespace gdn
