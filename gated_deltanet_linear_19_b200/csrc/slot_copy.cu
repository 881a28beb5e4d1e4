// Recurrent-state slot copy: state[dst[i]] = state[src[i]], conv_state[dst[i]] =
// conv_state[src[i]], bit-exact (the counterpart of the recurrent-state copy map s_copy of
// llama.cpp PR #16095, llm_graph_input_rs::set_input).
// Grid: (blocks per slot, n pairs). 16-byte vector copies; every block checks its own pair's
// slot ids and skips the pair if its dst repeats an earlier pair's dst or is used as a source.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int SC_THREADS = 256;
constexpr int SC_BLOCKS_PER_SLOT = 32;

__global__ void __launch_bounds__(SC_THREADS) slot_copy_kernel(const SlotCopyArgs p) {
  const int i = blockIdx.y;
  const int src = p.src[i], dst = p.dst[i];
  if (src < 0 || src >= p.n_slots || dst < 0 || dst >= p.n_slots) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  // pair i is skipped when its dst was already taken by an earlier pair (the first occurrence
  // wins) or is also read as a source by any pair (the copy would race with that read);
  // every block of the pair decides the same way
  int bad = 0;
  for (int j = threadIdx.x; j < p.n; j += blockDim.x)
    bad |= ((j < i && p.dst[j] == dst) || p.src[j] == dst) ? 1 : 0;
  if (__syncthreads_or(bad)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, GDN_ESLOT);
    return;
  }
  const int64_t tid = (int64_t)blockIdx.x * SC_THREADS + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * SC_THREADS;
  if (p.state) {
    const float4* s = reinterpret_cast<const float4*>(p.state + (int64_t)src * p.state_elems);
    float4* d = reinterpret_cast<float4*>(p.state + (int64_t)dst * p.state_elems);
    const int64_t n4 = p.state_elems / 4;
    for (int64_t e = tid; e < n4; e += stride) d[e] = s[e];
    for (int64_t e = n4 * 4 + tid; e < p.state_elems; e += stride)
      p.state[(int64_t)dst * p.state_elems + e] = p.state[(int64_t)src * p.state_elems + e];
  }
  if (p.conv_state) {
    const uint8_t* s = static_cast<const uint8_t*>(p.conv_state) + (int64_t)src * p.conv_bytes;
    uint8_t* d = static_cast<uint8_t*>(p.conv_state) + (int64_t)dst * p.conv_bytes;
    if ((p.conv_bytes & 15) == 0) {
      const int64_t n16 = p.conv_bytes / 16;
      for (int64_t e = tid; e < n16; e += stride)
        reinterpret_cast<uint4*>(d)[e] = reinterpret_cast<const uint4*>(s)[e];
    } else {
      for (int64_t e = tid; e < p.conv_bytes; e += stride) d[e] = s[e];
    }
  }
}

}  // namespace

cudaError_t launch_slot_copy(const SlotCopyArgs& a, cudaStream_t s) {
  dim3 grid(SC_BLOCKS_PER_SLOT, a.n);
  slot_copy_kernel<<<grid, SC_THREADS, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace gdn
