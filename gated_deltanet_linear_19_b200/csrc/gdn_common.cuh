// Shared device helpers for the gated delta-rule kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>

#include "../../include/gdn.h"

namespace gdn {

// ------------------------------------------------------------------ element I/O
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
  }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float load(const __half* p) { return __half2float(*p); }
  static __device__ __forceinline__ void store(__half* p, float v) { *p = __float2half_rn(v); }
};

template <typename T>
__device__ __forceinline__ float ld(const T* p) { return Elem<T>::load(p); }
template <typename T>
__device__ __forceinline__ void st(T* p, float v) { Elem<T>::store(p, v); }

// Load 4 consecutive elements (16-byte aligned for float, 8-byte for 16-bit types).
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ float4 ld4(const __half* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  __half2 a = *reinterpret_cast<__half2*>(&u.x);
  __half2 b = *reinterpret_cast<__half2*>(&u.y);
  float2 fa = __half22float2(a), fb = __half22float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void st4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void st4(__half* p, float4 v) {
  __half2 a = __floats2half2_rn(v.x, v.y);
  __half2 b = __floats2half2_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// Streaming (evict-first) 16-byte global load/store for data touched once per call.
__device__ __forceinline__ float4 ld4_stream(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st4_stream(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}

// Asks L2 to fetch [p, p + bytes) (bytes a multiple of 16, p 16-byte aligned); no data
// reaches the SM and nothing waits for it.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// L2 prefetch one wave ahead, for grids of (column tile, value head, sequence) blocks over fp32
// states [slot][H_v][DK][d_v]: thread 0 asks L2 for one contiguous row band of the state of the
// block `dist` places after this one in launch order (x fastest). The gridDim.x blocks of one
// (sequence, head) are adjacent, so together they cover that head's state whatever the column
// split (gridDim.x divides DK for every supported shape).
template <int DK>
__device__ __forceinline__ void prefetch_state_ahead(const float* state, const int32_t* slot_ids,
                                                     int n_slots, int H_v, int d_v, int dist) {
  if (dist <= 0 || threadIdx.x != 0) return;
  const int64_t gx = gridDim.x, gxy = gx * gridDim.y;
  const int64_t lin = blockIdx.x + gx * blockIdx.y + gxy * blockIdx.z + dist;
  if (lin >= gxy * gridDim.z) return;
  const int bf = (int)(lin / gxy), hf = (int)((lin % gxy) / gx), tf = (int)(lin % gx);
  const int sf = slot_ids[bf];
  const int rows = DK / (int)gx;
  if (sf >= 0 && sf < n_slots)
    prefetch_l2(state + (((int64_t)sf * H_v + hf) * DK + (int64_t)tf * rows) * d_v,
                (uint32_t)(rows * d_v * 4));
}

// Blocks of `kern` (`threads` threads, no dynamic shared memory) resident on the whole GPU at
// once (cached per device; 0 if unknown): the prefetch distance of one wave.
template <typename Kern>
int resident_blocks(Kern kern, int threads) {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int r = cache[dev].load(std::memory_order_relaxed);
  if (r == 0) {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 0;
    r = per_sm * sms;
    cache[dev].store(r, std::memory_order_relaxed);
  }
  return r;
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): each lane is one IEEE fp32 operation rounded to
// nearest, so a lane gives exactly the scalar fmaf / multiply; one instruction does two.
__device__ __forceinline__ uint64_t pack_f2(float2 v) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
  return r;
}
__device__ __forceinline__ float2 unpack_f2(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pack_f2(a)), "l"(pack_f2(b)), "l"(pack_f2(c)));
  return unpack_f2(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack_f2(a)), "l"(pack_f2(b)));
  return unpack_f2(d);
}

// ------------------------------------------------------------------ status word
// Records the first device-side error of a call sequence; read by gdn_device_status.
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }
// z * sigmoid(z) with the accurate exponential and an IEEE division
__device__ __forceinline__ float silu_exact(float z) { return z / (1.0f + expf(-z)); }
// Floor applied to a token's gate g inside the chunked kernels' cumulative sums. A chunk's
// decays are exp(g_cum_i - g_cum_j), differences of fp32 running sums: a gate of -1e4 would
// leave those sums so large that their differences lose about 1 % to rounding. Clamped at
// -40, a token still leaves at most exp(-40) = 4e-18 of what came before (the exact value is
// smaller, and both vanish next to the fp32 rounding of the result), and a 64-token sum stays
// within 2560, where its differences are exact to about 2e-4 relative.
constexpr float kGateFloor = -40.0f;

// softplus(x) = max(x,0) + log1p(exp(-|x|)), exact for all x (no threshold switch)
__device__ __forceinline__ float softplusf_(float x) {
  return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

// Key head read by value head h: grouped (h / (H_v / H_k)) or, with GDN_GQA_TILED, tiled
// (h % H_k).
__device__ __forceinline__ int khead_of(int h, int H_k, int H_v, int layout) {
  return (layout & GDN_GQA_TILED) ? h % H_k : h / (H_v / H_k);
}
// The first value head that reads key head hk (the one that owns hk's channels where a
// single writer is needed).
__device__ __forceinline__ bool first_vhead_of_khead(int h, int H_k, int H_v, int layout) {
  return (layout & GDN_GQA_TILED) ? h < H_k : h % (H_v / H_k) == 0;
}
// Gate inputs of token t, value head h: alpha (a) and the beta logit (b), from separate
// [T][H_v] arrays or, with GDN_GATES_MIXED_BA, from the fused [T][H_k][2 r] array passed as
// `a` (per key head first the r beta logits, then the r alphas of value heads hk r + j).
__device__ __forceinline__ float gate_alpha(const float* a, int64_t t, int h, int H_k, int H_v,
                                            int layout) {
  if (layout & GDN_GATES_MIXED_BA) {
    const int r = H_v / H_k;
    return a[(t * H_k + h / r) * 2 * r + r + h % r];
  }
  return a[t * H_v + h];
}
__device__ __forceinline__ float gate_beta_logit(const float* a, const float* b, int64_t t, int h,
                                                 int H_k, int H_v, int layout) {
  if (layout & GDN_GATES_MIXED_BA) {
    const int r = H_v / H_k;
    return a[(t * H_k + h / r) * 2 * r + h % r];
  }
  return b[t * H_v + h];
}

// Slot ids repeated within one call: the first occurrence wins. True when some earlier entry
// m < n of `ids` equals `slot`; every block working for entry n calls this (block-wide, all
// threads, 1-D blocks) and skips the entry when it returns true, so no two sequences of one
// call ever update the same pool row. Costs n loads spread over the block's threads.
__device__ __forceinline__ bool block_slot_taken(const int32_t* ids, int n, int slot) {
  int hit = 0;
  for (int m = threadIdx.x; m < n; m += blockDim.x) hit |= (ids[m] == slot) ? 1 : 0;
  return __syncthreads_or(hit) != 0;
}

// Find the sequence n with cu[n] <= t < cu[n+1] (cu non-decreasing); -1 if none.
__device__ __forceinline__ int find_seq(const int32_t* cu, int n_seqs, int64_t t) {
  int lo = 0, hi = n_seqs - 1, ans = -1;
  while (lo <= hi) {
    int mid = (lo + hi) >> 1;
    if ((int64_t)cu[mid] <= t) { ans = mid; lo = mid + 1; } else { hi = mid - 1; }
  }
  return ans;
}


// Start of sequence n in the packed token stream; cu == nullptr means one token per
// sequence (cu[n] = n).
__device__ __forceinline__ int64_t cu_at(const int32_t* cu, int64_t n) {
  return cu ? (int64_t)cu[n] : n;
}

// Map a flat segment id to (sequence, segment index within the sequence) for packed
// sequences, where sequence n owns max(min_count, ceil(len_n / seg)) consecutive segment
// ids in sequence order (cu == nullptr: one token per sequence, min_count <= 1). Block-wide:
// every thread must call it; s_wsum needs one int per warp. Returns the sequence (or -1 when
// `target` is past the last segment) and writes the segment index to *seg_out. Sequences with inconsistent cu_seqlens own no segment; block
// (0, 0, 0) records GDN_EINVAL for them.
template <int NT>
__device__ int block_locate_segment(const int32_t* cu, int n_seqs, int64_t T_total, int seg,
                                    int min_count, int64_t target, int* seg_out,
                                    int* s_seq, int* s_seg, int* s_wsum, int32_t* status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;
  const bool first_block = blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
  if (cu == nullptr) {
    // no cu_seqlens: one token per sequence, so (with min_count <= 1) sequence n owns
    // exactly segment n
    if (target >= n_seqs) return -1;
    *seg_out = 0;
    return (int)target;
  }
  if (n_seqs == 1) {
    // one sequence: every thread decides alone, with the same checks and results as below
    const int64_t c0 = cu[0], c1 = cu[1];
    if (first_block && tid == 0 && (c0 != 0 || c1 != T_total)) set_status(status, GDN_EINVAL);
    if (c0 < 0 || c1 < c0 || c1 > T_total) {
      if (first_block && tid == 0) set_status(status, GDN_EINVAL);
      return -1;
    }
    int64_t cnt = (c1 - c0 + seg - 1) / seg;
    if (cnt < min_count) cnt = min_count;
    if (target >= cnt) return -1;
    *seg_out = (int)target;
    return 0;
  }
  if (tid == 0) { *s_seq = -1; *s_seg = 0; }
  __syncthreads();
  int64_t run = 0;
  for (int base = 0; base < n_seqs; base += NT) {
    const int n = base + tid;
    int cnt = 0;
    if (n < n_seqs) {
      const int64_t c0 = cu[n], c1 = cu[n + 1];
      if (c0 < 0 || c1 < c0 || c1 > T_total) {
        if (first_block) set_status(status, GDN_EINVAL);
      } else {
        cnt = (int)((c1 - c0 + seg - 1) / seg);
        if (cnt < min_count) cnt = min_count;
      }
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int wbase = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      if (w < warp) wbase += s_wsum[w];
      tot += s_wsum[w];
    }
    incl += wbase;
    const int64_t lo = run + incl - cnt, hi = run + incl;
    if (cnt > 0 && target >= lo && target < hi) { *s_seq = n; *s_seg = (int)(target - lo); }
    run += tot;
    __syncthreads();
    if (*s_seq >= 0 || run > target) break;
  }
  if (first_block && tid == 0) {
    if (cu[0] != 0 || (int64_t)cu[n_seqs] != T_total) set_status(status, GDN_EINVAL);
  }
  const int n = *s_seq;
  *seg_out = *s_seg;
  return n;
}

// Block-wide sum over sequences m < n of ceil(len_m / seg) (the first segment id of n).
// Counts the same way as block_locate_segment with min_count 0 (invalid sequences own none).
template <int NT>
__device__ int64_t block_segment_base(const int32_t* cu, int n, int64_t T_total, int seg,
                                      int64_t* s_red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t acc = 0;
  for (int m = tid; m < n; m += NT) {
    const int64_t c0 = cu[m], c1 = cu[m + 1];
    if (c0 >= 0 && c1 > c0 && c1 <= T_total) acc += (c1 - c0 + seg - 1) / seg;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) s_red[warp] = acc;
  __syncthreads();
  int64_t tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) tot += s_red[w];
  __syncthreads();
  return tot;
}

}  // namespace gdn
