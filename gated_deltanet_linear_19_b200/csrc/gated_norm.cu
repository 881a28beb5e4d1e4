// Output gate of the layer: out = o / sqrt(mean(o^2) + eps) * norm_w * SiLU(z), the RMS norm
// taken over each (token, value head) row of d_v values, norm_w shared by all value heads.
// Pages: ik_llama.cpp src/llama-delta-net.cpp, build_layer_attn_linear_core
// (llm_build_norm with ssm_norm and LLM_NORM_RMS, then ggml_fused_mul_unary(z, ., SILU)).
//
// One warp per row: lane l holds d_v / 32 consecutive values; the sum of squares is reduced
// with xor shuffles. Memory-bound (o and z read once, out written once); may run in place.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int GN_WARPS = 8;

template <typename T> __device__ __forceinline__ void load_n(const T* p, float* f, int n) {
  for (int i = 0; i < n; ++i) f[i] = ld(p + i);
}

template <int VPL, typename TO, typename TZ, typename TR>
__global__ void __launch_bounds__(GN_WARPS * 32) gated_norm_kernel(const GateArgs p) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * GN_WARPS + (threadIdx.x >> 5);
  if (row >= p.rows) return;
  const int c0 = lane * VPL;
  float o[VPL], z[VPL];
  load_n(static_cast<const TO*>(p.o) + row * p.d_v + c0, o, VPL);
  load_n(static_cast<const TZ*>(p.z) + row * p.d_v + c0, z, VPL);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) ss = fmaf(o[i], o[i], ss);
  ss = warp_sum(ss);
  const float inv = 1.0f / sqrtf(ss / (float)p.d_v + p.eps);
  TR* out = static_cast<TR*>(p.out) + row * p.d_v + c0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) st(out + i, o[i] * inv * p.norm_w[c0 + i] * silu_exact(z[i]));
}

template <int VPL, typename TO, typename TZ>
cudaError_t launch_r(const GateArgs& a, cudaStream_t s) {
  const unsigned blocks = (unsigned)((a.rows + GN_WARPS - 1) / GN_WARPS);
  if (a.out_dtype == GDN_BF16)
    gated_norm_kernel<VPL, TO, TZ, __nv_bfloat16><<<blocks, GN_WARPS * 32, 0, s>>>(a);
  else
    gated_norm_kernel<VPL, TO, TZ, float><<<blocks, GN_WARPS * 32, 0, s>>>(a);
  return cudaGetLastError();
}

template <int VPL, typename TO>
cudaError_t launch_z(const GateArgs& a, cudaStream_t s) {
  if (a.z_dtype == GDN_BF16) return launch_r<VPL, TO, __nv_bfloat16>(a, s);
  return launch_r<VPL, TO, float>(a, s);
}

template <int VPL>
cudaError_t launch_v(const GateArgs& a, cudaStream_t s) {
  if (a.o_dtype == GDN_BF16) return launch_z<VPL, __nv_bfloat16>(a, s);
  return launch_z<VPL, float>(a, s);
}

}  // namespace

cudaError_t launch_gated_norm(const GateArgs& a, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  switch (a.d_v) {
    case 32: return launch_v<1>(a, s);
    case 64: return launch_v<2>(a, s);
    case 128: return launch_v<4>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdn
