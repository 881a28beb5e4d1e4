// Front of the gated delta-rule layer: causal depthwise conv1d over [conv_state; x] with the
// rolling conv state, SiLU, q|k|v split, L2 norm of q and k, q scale, and the gates
// g = -exp(A_log) * softplus(a + dt_bias), beta = sigmoid(b).
// Pages: ik_llama.cpp src/llama-delta-net.cpp, build_layer_attn_linear_core (ggml_ssm_conv,
// ggml_silu on the whole conv output, ggml_l2_norm, conv-state write-back);
// qwen3next.cpp build_layer_attn_linear (gate) and build_delta_net_* (sigmoid, 1/sqrt scale).
//
// Work decomposition: each sequence is cut into segments of FRONT_SEG tokens that start at
// the sequence's first token; blockIdx.x enumerates all segments of all sequences and
// blockIdx.y a block of FRONT_WARPS channel groups (one 128-channel head = one group for
// Qwen3-Next shapes). A warp owns one group for the whole segment, keeps the conv window in
// registers and reduces the L2 norm with shuffles. Only the first segment of a sequence reads
// the old conv state, so the same threads that read it also write the new one: no other
// block touches those bytes, and the update is race-free in one launch.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int FRONT_WARPS = 4;
constexpr int MAXCPL = 4;       // channels per lane (head dim 128 / 32 lanes)

// SiLU; with 16-bit q/k/v outputs an approximate form below the output rounding, the fp32
// outputs keep the accurate library functions.
template <typename TQ>
__device__ __forceinline__ float silu(float y) {
  if constexpr (sizeof(TQ) == 2) {
    // y sigmoid(y) = h + h tanh(h), h = y / 2, from the PTX approximate tanh (one
    // special-function instruction instead of an exponential and a reciprocal; its error, a
    // few 1e-4 of |y|, is below the 16-bit rounding of the result), the same form as the
    // record kernel's fused front
    const float h = 0.5f * y;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
  } else {
    return y * sigmoidf_(y);
  }
}

// SEG = tokens per segment (>= d_conv - 1): 16 for long sequences, 4 for decode-like batches
// of very short sequences (fewer registers, more blocks in flight).
template <typename TX, typename TS, typename TQ, int FRONT_SEG>
__global__ void __launch_bounds__(FRONT_WARPS * 32)
front_kernel(const FrontArgs p) {
  __shared__ int s_seq, s_seg;
  __shared__ int s_wsum[FRONT_WARPS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // Let a programmatically dependent kernel (the decode step) launch now: it only reads this
  // kernel's outputs after its own griddepcontrol.wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- map blockIdx.x to (sequence, segment); every sequence owns at least one segment so
  // that an empty sequence still writes (or resets) its conv state
  int seg = 0;
  const int n = block_locate_segment<FRONT_WARPS * 32>(p.cu_seqlens, p.n_seqs, p.T_total,
                                                       FRONT_SEG, 1, blockIdx.x, &seg, &s_seq,
                                                       &s_seg, s_wsum, p.status);
  if (n < 0) return;
  const int64_t tseq0 = cu_at(p.cu_seqlens, n);
  const int64_t len = cu_at(p.cu_seqlens, n + 1) - tseq0;
  const int64_t p0 = (int64_t)seg * FRONT_SEG;                 // first position in segment
  const int64_t p1 = p0 + FRONT_SEG < len ? p0 + FRONT_SEG : len;
  const int R = p.d_conv > 0 ? p.d_conv - 1 : 0;               // conv state rows

  int slot = 0;
  const bool rst = p.reset != nullptr && p.reset[n] != 0;
  if (R > 0) {
    slot = p.slot_ids[n];
    if (slot < 0 || slot >= p.n_slots) {
      if (tid == 0 && blockIdx.y == 0 && seg == 0) set_status(p.status, GDN_ESLOT);
      return;
    }
    // a slot repeated within the call: only its first sequence reads and rolls the conv
    // state; every block of a later one skips it and writes nothing
    if (block_slot_taken(p.slot_ids, n, slot)) {
      if (tid == 0 && blockIdx.y == 0 && seg == 0) set_status(p.status, GDN_ESLOT);
      return;
    }
  }

  // ---- gates for the segment's tokens (one channel block does them)
  if (blockIdx.y == 0) {
    const int nt = (int)(p1 - p0);
    for (int idx = tid; idx < nt * p.H_v; idx += blockDim.x) {
      const int64_t t = tseq0 + p0 + idx / p.H_v;
      const int h = idx % p.H_v;
      const float z = gate_alpha(p.a, t, h, p.H_k, p.H_v, p.layout) + p.dt_bias[h];
      p.g[t * p.H_v + h] = -expf(p.A_log[h]) * softplusf_(z);
      p.beta[t * p.H_v + h] = sigmoidf_(gate_beta_logit(p.a, p.b, t, h, p.H_k, p.H_v, p.layout));
    }
  }

  // ---- conv + SiLU + L2 norm for this warp's channel group
  const int G = 2 * p.H_k + p.H_v;
  const int gi = blockIdx.y * FRONT_WARPS + warp;
  if (gi >= G) return;
  const int64_t conv_dim = 2LL * p.H_k * p.d_k + (int64_t)p.H_v * p.d_v;
  int d, kind;  // kind 0 = q, 1 = k, 2 = v
  int64_t chan0;
  if (gi < p.H_k) { kind = 0; d = p.d_k; chan0 = (int64_t)gi * p.d_k; }
  else if (gi < 2 * p.H_k) { kind = 1; d = p.d_k; chan0 = (int64_t)gi * p.d_k; }
  else { kind = 2; d = p.d_v; chan0 = 2LL * p.H_k * p.d_k + (int64_t)(gi - 2 * p.H_k) * p.d_v; }
  const int cpl = d >> 5;
  const int64_t c0 = chan0 + (int64_t)lane * cpl;

  const TX* x = static_cast<const TX*>(p.x);
  TS* cst = static_cast<TS*>(p.conv_state);
  TS* my_state = cst ? cst + (int64_t)slot * R * conv_dim : nullptr;

  // Taps are right-aligned: wa[j][3] multiplies the current token, wa[j][2] the newest
  // window row, ... ; window slot 2 is the newest row, slot 3-R the oldest; unused slots have
  // zero weight.
  float wa[MAXCPL][4];
  float win[3][MAXCPL];
  float old_state[3][MAXCPL];
#pragma unroll
  for (int j = 0; j < MAXCPL; ++j) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tap = p.d_conv - 4 + i;
      wa[j][i] = (j < cpl && tap >= 0) ? p.conv_w[(c0 + j) * p.d_conv + tap] : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < 3; ++r) { win[r][j] = 0.0f; old_state[r][j] = 0.0f; }
  }
  // window slots hold x_ext rows [p0, p0 + R) with x_ext = [state rows; x rows]
#pragma unroll
  for (int sl = 0; sl < 3; ++sl) {
    const int r = sl - (3 - R);  // window row (0 = oldest)
    if (r >= 0) {
      const int64_t e = p0 + r;  // x_ext index
#pragma unroll
      for (int j = 0; j < MAXCPL; ++j) {
        if (j < cpl) {
          float val;
          if (e < R) {
            val = rst ? 0.0f : ld(my_state + e * conv_dim + c0 + j);
          } else {
            val = ld(x + (tseq0 + e - R) * conv_dim + c0 + j);
          }
          win[sl][j] = val;
        }
      }
    }
  }
  if (seg == 0) {
    // x_ext rows 0..R-1 are the old state (or zeros on reset); kept for the write-back
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
      for (int j = 0; j < MAXCPL; ++j)
        if (r < R && j < cpl) old_state[r][j] = rst ? 0.0f : ld(my_state + (int64_t)r * conv_dim + c0 + j);
  }

  TQ* out;
  int64_t out_stride, out_off;
  if (kind == 0) { out = static_cast<TQ*>(p.q); out_stride = (int64_t)p.H_k * p.d_k; out_off = (int64_t)gi * p.d_k; }
  else if (kind == 1) { out = static_cast<TQ*>(p.k); out_stride = (int64_t)p.H_k * p.d_k; out_off = (int64_t)(gi - p.H_k) * p.d_k; }
  else { out = static_cast<TQ*>(p.v); out_stride = (int64_t)p.H_v * p.d_v; out_off = (int64_t)(gi - 2 * p.H_k) * p.d_v; }
  const float scale = kind == 0 ? p.q_scale : 1.0f;

  // all of the segment's x values first (independent loads in flight), then the recurrence
  // over the conv window
  float xs[FRONT_SEG][MAXCPL];
#pragma unroll
  for (int tt = 0; tt < FRONT_SEG; ++tt) {
    const int64_t pos = p0 + tt;
    const int64_t t = tseq0 + (pos < p1 ? pos : p0);
    if (cpl == 4) {
      const float4 v4 = ld4(x + t * conv_dim + c0);
      xs[tt][0] = v4.x; xs[tt][1] = v4.y; xs[tt][2] = v4.z; xs[tt][3] = v4.w;
    } else {
#pragma unroll
      for (int j = 0; j < MAXCPL; ++j) xs[tt][j] = j < cpl ? ld(x + t * conv_dim + c0 + j) : 0.0f;
    }
  }
#pragma unroll
  for (int tt = 0; tt < FRONT_SEG; ++tt) {
    const int64_t pos = p0 + tt;
    if (pos >= p1) break;
    const int64_t t = tseq0 + pos;
    float u[MAXCPL];
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < MAXCPL; ++j) {
      const float xv = xs[tt][j];
      if (p.d_conv > 0) {
        float y = wa[j][0] * win[0][j];
        y = fmaf(wa[j][1], win[1][j], y);
        y = fmaf(wa[j][2], win[2][j], y);
        y = fmaf(wa[j][3], xv, y);
        u[j] = silu<TQ>(y);
      } else {
        u[j] = xv;
      }
      if (j < cpl) ss = fmaf(u[j], u[j], ss);
      win[0][j] = win[1][j];
      win[1][j] = win[2][j];
      win[2][j] = xv;
    }
    float mul = scale;
    if (kind != 2) {
      ss = warp_sum(ss);
      mul = scale / sqrtf(ss + p.eps);
    }
    TQ* dst = out + t * out_stride + out_off + (int64_t)lane * cpl;
    if (cpl == 4) {
      st4(dst, make_float4(u[0] * mul, u[1] * mul, u[2] * mul, u[3] * mul));
    } else {
#pragma unroll
      for (int j = 0; j < MAXCPL; ++j) if (j < cpl) st(dst + j, u[j] * mul);
    }
  }

  // ---- new conv state = last R rows of x_ext (written by the segment that read the old one)
  if (seg == 0 && R > 0) {
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      if (r < R) {
        const int64_t e = len + r;  // x_ext index
#pragma unroll
        for (int j = 0; j < MAXCPL; ++j) {
          if (j < cpl) {
            float val;
            if (e < R) {
              val = e == 0 ? old_state[0][j] : (e == 1 ? old_state[1][j] : old_state[2][j]);
            } else {
              val = ld(x + (tseq0 + e - R) * conv_dim + c0 + j);
            }
            st(my_state + (int64_t)r * conv_dim + c0 + j, val);
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Variant for d_k == d_v == D: each lane owns 4 consecutive channels (8-byte loads of 16-bit
// x), a head's D channels are D / 4 consecutive lanes reduced with xor shuffles, and a block
// of FRONT_WARPS warps covers FRONT_WARPS * 128 channels of one segment. All SEG x rows of
// the segment are loaded, still packed, before any arithmetic, so every thread has SEG + R
// independent loads in flight; the conv window then slides through registers. The gates of
// a segment's tokens are spread over the channel blocks (block y takes heads y, y + gridDim.y,
// ...). Same segments and the same race-free conv-state update as front_kernel.
template <typename T> struct Pack4;
template <> struct Pack4<__nv_bfloat16> {
  using R = uint2;
  static __device__ __forceinline__ R load(const __nv_bfloat16* p) {
    R r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                 : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
  }
  static __device__ __forceinline__ R zero() { return make_uint2(0u, 0u); }
  static __device__ __forceinline__ void unpack(R r, float* f) {
    // a bf16 is the upper half of the fp32 with the same bits
    f[0] = __uint_as_float(r.x << 16); f[1] = __uint_as_float(r.x & 0xffff0000u);
    f[2] = __uint_as_float(r.y << 16); f[3] = __uint_as_float(r.y & 0xffff0000u);
  }
};
template <> struct Pack4<float> {
  using R = float4;
  static __device__ __forceinline__ R load(const float* p) {
    R r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
  }
  static __device__ __forceinline__ R zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  static __device__ __forceinline__ void unpack(R r, float* f) {
    f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
  }
};

// 16-bit x: at most 85 registers for long segments so that 6 blocks fit per SM (measured
// faster than 5), at most 64 for decode-like segments so that a 64-sequence step fits in
// one wave of 8 blocks per SM
template <typename TX, typename TS, typename TQ, int SEG, int D>
__global__ void __launch_bounds__(FRONT_WARPS * 32, sizeof(TX) == 2 ? (SEG == 4 ? 8 : 6) : 1)
front4_kernel(const FrontArgs p) {
  constexpr int LPH = D / 4;  // lanes per head
  __shared__ int s_seq, s_seg;
  __shared__ int s_wsum[FRONT_WARPS];
  const int tid = threadIdx.x;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  int seg = 0;
  const int n = block_locate_segment<FRONT_WARPS * 32>(p.cu_seqlens, p.n_seqs, p.T_total, SEG, 1,
                                                       blockIdx.x, &seg, &s_seq, &s_seg, s_wsum,
                                                       p.status);
  if (n < 0) return;
  const int64_t tseq0 = cu_at(p.cu_seqlens, n);
  const int64_t len = cu_at(p.cu_seqlens, n + 1) - tseq0;
  // short-sequence mode: longer sequences belong to other kernels of the same call
  if (p.max_len > 0 && len > p.max_len) return;
  // row of the sequence's first token in q, k, v, g, beta
  const int64_t orow0 = p.max_len > 0 ? (int64_t)n * p.max_len : tseq0;
  const int64_t p0 = (int64_t)seg * SEG;
  const int np = (int)((p0 + SEG < len ? p0 + SEG : len) - p0);  // tokens in this segment
  const int R = p.d_conv > 0 ? p.d_conv - 1 : 0;
  int slot = 0;
  const bool rst = p.reset != nullptr && p.reset[n] != 0;
  if (R > 0) {
    slot = p.slot_ids[n];
    if (slot < 0 || slot >= p.n_slots) {
      if (tid == 0 && blockIdx.y == 0 && seg == 0) set_status(p.status, GDN_ESLOT);
      return;
    }
    // a slot repeated within the call: only its first sequence reads and rolls the conv
    // state; every block of a later one skips it and writes nothing
    if (block_slot_taken(p.slot_ids, n, slot)) {
      if (tid == 0 && blockIdx.y == 0 && seg == 0) set_status(p.status, GDN_ESLOT);
      return;
    }
  }
  const int64_t conv_dim = (int64_t)(2 * p.H_k + p.H_v) * D;
  const int64_t c0 = (int64_t)blockIdx.y * (FRONT_WARPS * 128) + (int64_t)tid * 4;
  const bool active = c0 < conv_dim;
  const TX* x = static_cast<const TX*>(p.x);
  const TX* xp = x + (tseq0 + p0) * conv_dim + c0;

  // ---- x rows of the segment, packed
  typename Pack4<TX>::R xr[SEG];
#pragma unroll
  for (int u = 0; u < SEG; ++u)
    xr[u] = (active && u < np) ? Pack4<TX>::load(xp + (int64_t)u * conv_dim) : Pack4<TX>::zero();

  // ---- gates of the segment's tokens for heads y, y + gridDim.y, ...
  {
    const int gy = gridDim.y, hy = blockIdx.y;
    const int nh = hy < p.H_v ? (p.H_v - hy + gy - 1) / gy : 0;
    for (int idx = tid; idx < np * nh; idx += blockDim.x) {
      const int64_t t = tseq0 + p0 + idx / nh;
      const int64_t tr = orow0 + p0 + idx / nh;  // output row
      const int h = hy + (idx % nh) * gy;
      const float z = gate_alpha(p.a, t, h, p.H_k, p.H_v, p.layout) + p.dt_bias[h];
      p.g[tr * p.H_v + h] = -expf(p.A_log[h]) * softplusf_(z);
      p.beta[tr * p.H_v + h] = sigmoidf_(gate_beta_logit(p.a, p.b, t, h, p.H_k, p.H_v, p.layout));
    }
  }

  // region of this lane's channels: 0 = q, 1 = k, 2 = v (a head never straddles lane groups)
  const int64_t qk_end = (int64_t)p.H_k * D;
  const int kind = c0 < qk_end ? 0 : (c0 < 2 * qk_end ? 1 : 2);
  TS* my_state = R > 0 ? static_cast<TS*>(p.conv_state) + (int64_t)slot * R * conv_dim : nullptr;

  // taps are right-aligned: wa[j][3] multiplies the current token, wa[j][2] the newest window
  // row; window slot 2 is the newest row, slot 3 - R the oldest; unused slots weigh zero
  float wa[4][4], win[3][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (active && p.d_conv == 4) {
      const float4 w4 = *reinterpret_cast<const float4*>(p.conv_w + (c0 + j) * 4);
      wa[j][0] = w4.x; wa[j][1] = w4.y; wa[j][2] = w4.z; wa[j][3] = w4.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tap = p.d_conv - 4 + i;
        wa[j][i] = (active && tap >= 0) ? p.conv_w[(c0 + j) * p.d_conv + tap] : 0.0f;
      }
    }
#pragma unroll
    for (int r = 0; r < 3; ++r) win[r][j] = 0.0f;
  }
  if (active) {
    // window slots hold x_ext rows [p0, p0 + R) with x_ext = [state rows; x rows]
#pragma unroll
    for (int sl = 0; sl < 3; ++sl) {
      const int r = sl - (3 - R);
      if (r >= 0) {
        const int64_t e = p0 + r;
        if (e < R) {
          if (!rst) {
            const float4 v = ld4(my_state + e * conv_dim + c0);
            win[sl][0] = v.x; win[sl][1] = v.y; win[sl][2] = v.z; win[sl][3] = v.w;
          }
        } else {
          Pack4<TX>::unpack(Pack4<TX>::load(x + (tseq0 + e - R) * conv_dim + c0), win[sl]);
        }
      }
    }
  }
  TQ* out;
  int64_t out_stride, out_off;
  if (kind == 0) { out = static_cast<TQ*>(p.q); out_stride = qk_end; out_off = c0; }
  else if (kind == 1) { out = static_cast<TQ*>(p.k); out_stride = qk_end; out_off = c0 - qk_end; }
  else { out = static_cast<TQ*>(p.v); out_stride = (int64_t)p.H_v * D; out_off = c0 - 2 * qk_end; }
  const float scale = kind == 0 ? p.q_scale : 1.0f;
  TQ* op = out + (orow0 + p0) * out_stride + out_off;

  // long segments: tokens in groups of G = 4, a head's sums of squares reduced for the 4
  // tokens together; short (decode) segments, which mostly hold one token: G = 1
  constexpr int G = SEG >= 16 ? 4 : 1;
  static_assert(SEG % G == 0, "segments hold whole token groups");
  const int lane = tid & 31;
#pragma unroll
  for (int u0 = 0; u0 < SEG; u0 += G) {
    if (u0 >= np) break;
    float y[G][4], ss[G];
#pragma unroll
    for (int t = 0; t < G; ++t) {
      float xs[4];
      Pack4<TX>::unpack(xr[u0 + t], xs);
      ss[t] = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float acc = wa[j][0] * win[0][j];  // d_conv >= 1 here (launch_front)
        acc = fmaf(wa[j][1], win[1][j], acc);
        acc = fmaf(wa[j][2], win[2][j], acc);
        acc = fmaf(wa[j][3], xs[j], acc);
        y[t][j] = silu<TQ>(acc);
        ss[t] = fmaf(y[t][j], y[t][j], ss[t]);
        win[0][j] = win[1][j];
        win[1][j] = win[2][j];
        win[2][j] = xs[j];
      }
    }
    float mul[G];
#pragma unroll
    for (int t = 0; t < G; ++t) mul[t] = 1.0f;
    if constexpr (LPH == 32 && G == 1) {
      // a warp is one head: v heads skip the norm
      if (kind != 2) {
        float tot = ss[0];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        if constexpr (sizeof(TQ) == 2) mul[0] = scale * rsqrtf(tot + p.eps);
        else mul[0] = scale / sqrtf(tot + p.eps);
      }
    } else if constexpr (LPH == 32) {
      // a warp is one head: v heads skip the norm; q, k heads reduce the 4 sums with 6
      // shuffles (after the xor-16 and xor-8 exchanges lane l holds token 2 (l>>4 & 1) +
      // (l>>3 & 1), summed over 4 lanes; three more levels finish it), then broadcast
      if (kind != 2) {
        const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0;
        const float sa = __shfl_xor_sync(0xffffffffu, b4 ? ss[0] : ss[2], 16);
        const float sb = __shfl_xor_sync(0xffffffffu, b4 ? ss[1] : ss[3], 16);
        const float t0 = (b4 ? ss[2] : ss[0]) + sa, t1 = (b4 ? ss[3] : ss[1]) + sb;
        float tot = (b3 ? t1 : t0) + __shfl_xor_sync(0xffffffffu, b3 ? t0 : t1, 8);
        tot += __shfl_xor_sync(0xffffffffu, tot, 4);
        tot += __shfl_xor_sync(0xffffffffu, tot, 2);
        tot += __shfl_xor_sync(0xffffffffu, tot, 1);
        float inv;
        if constexpr (sizeof(TQ) == 2) inv = scale * rsqrtf(tot + p.eps);
        else inv = scale / sqrtf(tot + p.eps);
#pragma unroll
        for (int t = 0; t < 4; ++t) mul[t] = __shfl_sync(0xffffffffu, inv, t * 8);
      }
    } else {
      // a head is LPH < 32 lanes, and one warp may hold heads of different kinds: every lane
      // takes part in the shuffles
#pragma unroll
      for (int t = 0; t < G; ++t) {
        float tot = ss[t];
#pragma unroll
        for (int o = 1; o < LPH; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        if (kind != 2) {
          if constexpr (sizeof(TQ) == 2) mul[t] = scale * rsqrtf(tot + p.eps);
          else mul[t] = scale / sqrtf(tot + p.eps);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < G; ++t) {
      if (active && u0 + t < np)
        st4(op + (int64_t)(u0 + t) * out_stride,
            make_float4(y[t][0] * mul[t], y[t][1] * mul[t], y[t][2] * mul[t], y[t][3] * mul[t]));
    }
  }

  // new conv state = last R rows of x_ext, written by the segment that read the old rows
  if (seg == 0 && R > 0 && active) {
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      if (r < R) {
        const int64_t e = len + r;
        float4 f;
        if (e < R) {  // still an old-state row (sequences shorter than R)
          f = rst ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(my_state + e * conv_dim + c0);
        } else {
          float t4[4];
          Pack4<TX>::unpack(Pack4<TX>::load(x + (tseq0 + e - R) * conv_dim + c0), t4);
          f = make_float4(t4[0], t4[1], t4[2], t4[3]);
        }
        // new row r comes from old row len + r >= r, and rows are rewritten in increasing
        // order, so every old row is read before it is overwritten
        st4(my_state + (int64_t)r * conv_dim + c0, f);
      }
    }
  }
}

template <typename TX, typename TS, int SEG>
cudaError_t launch_t2(const FrontArgs& a, cudaStream_t s, dim3 grid, dim3 block) {
  switch (a.qkv_dtype) {
    case GDN_F32: front_kernel<TX, TS, float, SEG><<<grid, block, 0, s>>>(a); break;
    case GDN_BF16: front_kernel<TX, TS, __nv_bfloat16, SEG><<<grid, block, 0, s>>>(a); break;
    case GDN_F16: front_kernel<TX, TS, __half, SEG><<<grid, block, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename TX, int SEG>
cudaError_t launch_t1(const FrontArgs& a, cudaStream_t s, dim3 grid, dim3 block) {
  if (a.conv_state_dtype == GDN_BF16) return launch_t2<TX, __nv_bfloat16, SEG>(a, s, grid, block);
  return launch_t2<TX, float, SEG>(a, s, grid, block);
}

template <int SEG>
cudaError_t launch_seg(const FrontArgs& a, cudaStream_t s) {
  const int G = 2 * a.H_k + a.H_v;
  const int64_t segs = (a.T_total + SEG - 1) / SEG + a.n_seqs;
  dim3 grid((unsigned)segs, (unsigned)((G + FRONT_WARPS - 1) / FRONT_WARPS));
  dim3 block(FRONT_WARPS * 32);
  if (a.x_dtype == GDN_BF16) return launch_t1<__nv_bfloat16, SEG>(a, s, grid, block);
  return launch_t1<float, SEG>(a, s, grid, block);
}

}  // namespace

template <typename TX, typename TS, int SEG, int D>
cudaError_t launch8_q(const FrontArgs& a, cudaStream_t s) {
  const int64_t conv_dim = (int64_t)(2 * a.H_k + a.H_v) * D;
  const int64_t segs = (a.T_total + SEG - 1) / SEG + a.n_seqs;
  dim3 grid((unsigned)segs, (unsigned)((conv_dim + FRONT_WARPS * 128 - 1) / (FRONT_WARPS * 128)));
  dim3 block(FRONT_WARPS * 32);
  switch (a.qkv_dtype) {
    case GDN_F32: front4_kernel<TX, TS, float, SEG, D><<<grid, block, 0, s>>>(a); break;
    case GDN_BF16: front4_kernel<TX, TS, __nv_bfloat16, SEG, D><<<grid, block, 0, s>>>(a); break;
    case GDN_F16: front4_kernel<TX, TS, __half, SEG, D><<<grid, block, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <int SEG, int D>
cudaError_t launch8(const FrontArgs& a, cudaStream_t s) {
  if (a.x_dtype == GDN_BF16) {
    if (a.conv_state_dtype == GDN_BF16) return launch8_q<__nv_bfloat16, __nv_bfloat16, SEG, D>(a, s);
    return launch8_q<__nv_bfloat16, float, SEG, D>(a, s);
  }
  if (a.conv_state_dtype == GDN_BF16) return launch8_q<float, __nv_bfloat16, SEG, D>(a, s);
  return launch8_q<float, float, SEG, D>(a, s);
}

template <int SEG>
cudaError_t launch8_d(const FrontArgs& a, cudaStream_t s) {
  switch (a.d_k) {
    case 32: return launch8<SEG, 32>(a, s);
    case 64: return launch8<SEG, 64>(a, s);
    case 128: return launch8<SEG, 128>(a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_front(const FrontArgs& a, cudaStream_t s) {
  if (a.max_len > 0 && !(a.d_k == a.d_v && a.d_conv > 0)) return cudaErrorNotSupported;
  // decode-like batches (about one token per sequence) use short segments
  const bool short_seqs = a.T_total < 8 * (int64_t)a.n_seqs;
  // front4_kernel assumes a convolution (d_conv >= 1); without one the general kernel runs
  if (a.d_k == a.d_v && a.d_conv > 0) return short_seqs ? launch8_d<4>(a, s) : launch8_d<16>(a, s);
  return short_seqs ? launch_seg<4>(a, s) : launch_seg<16>(a, s);
}

}  // namespace gdn
