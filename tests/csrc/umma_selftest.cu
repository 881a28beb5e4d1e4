// Test-only kernel: one M=128 tcgen05 kind::f16 GEMM D = A * B with A, B staged in shared
// memory in the no-swizzle canonical layouts of umma.cuh (K-major or MN-major, with either
// the K groups or the M/N groups as the outer stride), D read back with tcgen05.ld.
// Checks the descriptor conventions the prefill kernels rely on.
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../gated_deltanet_linear_19_b200/csrc/umma.cuh"

using namespace gdn::umma;

// byte offset of element (mn, k) in a canonical layout
__device__ __forceinline__ uint32_t off(int mn, int k, bool mn_major, uint32_t lbo, uint32_t sbo) {
  if (!mn_major) return (mn % 8) * 16 + (k % 8) * 2 + (mn / 8) * sbo + (k / 8) * lbo;
  return (mn % 8) * 2 + (k % 8) * 16 + (mn / 8) * sbo + (k / 8) * lbo;
}

__global__ void __launch_bounds__(128) gemm_kernel(const __half* A, const __half* B, float* D,
                                                   int N, int K, int a_mn, int b_mn, int outer_k,
                                                   int* err) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int M = 128;
  uint8_t* As = sm;
  uint8_t* Bs = sm + M * K * 2;
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int tid = threadIdx.x, warp = tid >> 5;
  // strides: outer_k -> K groups outermost
  const uint32_t a_lbo = outer_k ? (M / 8) * 128 : 128, a_sbo = outer_k ? 128 : (K / 8) * 128;
  const uint32_t b_lbo = outer_k ? (N / 8) * 128 : 128, b_sbo = outer_k ? 128 : (K / 8) * 128;
  for (int i = tid; i < M * K; i += 128) {
    int m = i / K, k = i % K;
    *reinterpret_cast<__half*>(As + off(m, k, a_mn, a_lbo, a_sbo)) = A[i];
  }
  for (int i = tid; i < K * N; i += 128) {
    int k = i / N, n = i % N;
    *reinterpret_cast<__half*>(Bs + off(n, k, b_mn, b_lbo, b_sbo)) = B[i];
  }
  fence_proxy_async();
  if (warp == 0) tmem_alloc(&tbase, 256);
  if (tid == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tbase;
  if (tid == 0) {
    const uint32_t id = idesc_f16(M, N, a_mn, b_mn);
    for (int ks = 0; ks < K / 16; ++ks) {
      uint64_t ad = desc(smem_u32(As) + ks * 2 * a_lbo, a_lbo, a_sbo);
      uint64_t bd = desc(smem_u32(Bs) + ks * 2 * b_lbo, b_lbo, b_sbo);
      mma_f16(tb, ad, bd, id, ks > 0);
    }
    commit(&bar);
  }
  if (!mbar_wait(&bar, 0, nullptr)) { if (tid == 0) atomicExch(err, 1); }
  fence_after_sync();
  for (int c = 0; c < N; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr(tb, warp * 32, c), r);
    tmem_wait_ld();
    const int row = warp * 32 + (tid & 31);
    for (int j = 0; j < 32 && c + j < N; ++j) D[row * N + c + j] = __uint_as_float(r[j]);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) { tmem_relinquish(); tmem_dealloc(tb, 256); }
}

extern "C" int umma_selftest(const void* A, const void* B, void* D, int N, int K, int a_mn,
                             int b_mn, int outer_k, int* err) {
  size_t smem = 128 * K * 2 + K * N * 2;
  cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  gemm_kernel<<<1, 128, smem>>>((const __half*)A, (const __half*)B, (float*)D, N, K, a_mn, b_mn,
                                outer_k, err);
  cudaError_t e = cudaDeviceSynchronize();
  return (int)e;
}

// ---------------------------------------------------------------- A in tensor memory
// D = A * B with A held in TMEM: row m in lane m, K elements packed two per 32-bit column
// (even k in the low half), so a K step of 16 is 8 columns. B in shared memory as above.
// (tmem_wait_st and mma_f16_tmem_a come from umma.cuh.)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      :
      : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__global__ void __launch_bounds__(128) gemm_tmem_a_kernel(const __half* A, const __half* B,
                                                          float* D, int N, int K, int b_mn,
                                                          int* err) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int M = 128;
  uint8_t* Bs = sm;
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t b_lbo = 128, b_sbo = (K / 8) * 128;
  for (int i = tid; i < K * N; i += 128) {
    int k = i / N, n = i % N;
    *reinterpret_cast<__half*>(Bs + off(n, k, b_mn, b_lbo, b_sbo)) = B[i];
  }
  fence_proxy_async();
  if (warp == 0) tmem_alloc(&tbase, 256);
  if (tid == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tbase;
  constexpr uint32_t A_COL = 128;
  // row m = tid: 32 K values per tcgen05.st of 16 columns
  for (int kc = 0; kc < K / 32; ++kc) {
    uint32_t r[16];
    for (int j = 0; j < 16; ++j) {
      const __half2 h = __halves2half2(A[tid * K + kc * 32 + 2 * j], A[tid * K + kc * 32 + 2 * j + 1]);
      r[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    tmem_st16(taddr(tb, warp * 32, A_COL + kc * 16), r);
  }
  tmem_wait_st();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (tid == 0) {
    const uint32_t id = idesc_f16(M, N, false, b_mn);
    for (int ks = 0; ks < K / 16; ++ks) {
      uint64_t bd = desc(smem_u32(Bs) + ks * 2 * b_lbo, b_lbo, b_sbo);
      mma_f16_tmem_a(tb, tb + A_COL + ks * 8, bd, id, ks > 0);
    }
    commit(&bar);
  }
  if (!mbar_wait(&bar, 0, nullptr)) { if (tid == 0) atomicExch(err, 1); }
  fence_after_sync();
  for (int c = 0; c < N; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr(tb, warp * 32, c), r);
    tmem_wait_ld();
    const int row = warp * 32 + (tid & 31);
    for (int j = 0; j < 32 && c + j < N; ++j) D[row * N + c + j] = __uint_as_float(r[j]);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) { tmem_relinquish(); tmem_dealloc(tb, 256); }
}

extern "C" int umma_selftest_tmem_a(const void* A, const void* B, void* D, int N, int K, int b_mn,
                                    int* err) {
  if (N > 128 || K > 128 || K % 32 != 0 || N % 32 != 0) return -1;
  size_t smem = K * N * 2;
  cudaFuncSetAttribute(gemm_tmem_a_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  gemm_tmem_a_kernel<<<1, 128, smem>>>((const __half*)A, (const __half*)B, (float*)D, N, K, b_mn,
                                       err);
  cudaError_t e = cudaDeviceSynchronize();
  return (int)e;
}

// ---------------------------------------------------------------- bounded waits
// A wait that runs out. One MMA (zero operands) is issued and committed to barrier `done`;
// every thread then waits on barrier `never`, which nothing completes, with a limit of `limit`
// cycles (or, with `abort_first`, with the default limit but the abort flag already raised).
// The wait must give up and return false; the kernel records -5 (GDN_ETIMEOUT) in *status,
// then drains what it issued (waits for `done` under the default limit), records whether the
// drain completed in *drained, and frees its TMEM before it exits.
__global__ void __launch_bounds__(128) timeout_kernel(int* status, long long limit,
                                                      int abort_first, int* drained) {
  __shared__ __align__(128) uint8_t ops[128 * 16 * 2 + 32 * 16 * 2];
  __shared__ uint64_t done, never;
  __shared__ uint32_t tbase;
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < (int)sizeof(ops) / 4; i += 128) reinterpret_cast<uint32_t*>(ops)[i] = 0u;
  fence_proxy_async();
  if (warp == 0) tmem_alloc(&tbase, 32);
  if (tid == 0) {
    s_abort = abort_first ? 1 : 0;
    mbar_init(&done, 1);
    mbar_init(&never, 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tbase;
  if (tid == 0) {
    // M = 128, N = 32, K = 16, both operands K-major (LBO 128, SBO 256)
    const uint64_t ad = desc(smem_u32(ops), 128, 256);
    const uint64_t bd = desc(smem_u32(ops + 128 * 16 * 2), 128, 256);
    mma_f16(tb, ad, bd, idesc_f16(128, 32, false, false), 0);
    commit(&done);
  }
  __syncwarp();
  const bool ok = abort_first ? mbar_wait(&never, 0, &s_abort)
                              : mbar_wait(&never, 0, nullptr, limit);
  if (!ok && tid == 0) atomicCAS(status, 0, -5);
  const bool d = mbar_wait(&done, 0, nullptr);
  if (tid == 0) *drained = d ? 1 : 0;
  fence_before_sync();
  __syncthreads();
  if (warp == 0) { tmem_relinquish(); tmem_dealloc(tb, 32); }
}

extern "C" int umma_selftest_timeout(int* status, long long limit, int abort_first,
                                     int* drained) {
  timeout_kernel<<<1, 128>>>(status, limit, abort_first, drained);
  return (int)cudaDeviceSynchronize();
}

// ---------------------------------------------------------------- 128-byte swizzled operands
// The layouts a TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes (16-bit elements): a swizzle
// atom is 8 rows x 128 bytes (64 elements), 1024-byte aligned, and the 16-byte chunk j of row
// r of an atom sits at chunk position j ^ r.
//   K-major  (rows = M or N, K contiguous): atoms of 8 rows stacked along M/N every 1024 bytes
//            (SBO); the next 64 elements of K in another atom column `katom` bytes further.
//            A K step of 16 inside an atom moves the start address by 32 bytes.
//   MN-major (rows = K, M/N contiguous): atoms of 8 K-rows stacked along K every 1024 bytes
//            (SBO); the next 64 elements of M/N `lbo` bytes further (LBO).
__device__ __forceinline__ uint32_t off_sw128(int mn, int k, bool mn_major, uint32_t katom,
                                              uint32_t lbo) {
  if (!mn_major) {
    const uint32_t r = mn, c = k;
    return (c / 64) * katom + (r / 8) * 1024 + (r % 8) * 128 + ((((c % 64) / 8) ^ (r % 8)) * 16) +
           (c % 8) * 2;
  }
  const uint32_t r = k, c = mn;
  return (c / 64) * lbo + (r / 8) * 1024 + (r % 8) * 128 + ((((c % 64) / 8) ^ (r % 8)) * 16) +
         (c % 8) * 2;
}

__global__ void __launch_bounds__(128) gemm_sw128_kernel(const __half* A, const __half* B, float* D,
                                                         int N, int K, int a_mn, int b_mn, int* err) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  // 1024-byte aligned base (the launch asks for 1 KB of slack)
  uint8_t* sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
  const int M = 128;
  uint8_t* As = sm;
  uint8_t* Bs = sm + M * K * 2;
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int tid = threadIdx.x, warp = tid >> 5;
  // A: K-major -> atom columns of M/8 atoms; MN-major -> 64-element M blocks of K/8 atoms
  const uint32_t a_katom = (M / 8) * 1024, a_lbo = (K / 8) * 1024;
  const uint32_t b_katom = (N / 8) * 1024, b_lbo = (K / 8) * 1024;
  for (int i = tid; i < M * K; i += 128) {
    int m = i / K, k = i % K;
    *reinterpret_cast<__half*>(As + off_sw128(m, k, a_mn, a_katom, a_lbo)) = A[i];
  }
  for (int i = tid; i < K * N; i += 128) {
    int k = i / N, n = i % N;
    *reinterpret_cast<__half*>(Bs + off_sw128(n, k, b_mn, b_katom, b_lbo)) = B[i];
  }
  fence_proxy_async();
  if (warp == 0) tmem_alloc(&tbase, 256);
  if (tid == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tbase;
  if (tid == 0) {
    const uint32_t id = idesc_f16(M, N, a_mn, b_mn);
    for (int ks = 0; ks < K / 16; ++ks) {
      // K-major: atom column ks / 4, 32 bytes per K step inside it; MN-major: 2 K-row groups
      const uint32_t ao = a_mn ? ks * 2 * 1024 : (ks / 4) * a_katom + (ks % 4) * 32;
      const uint32_t bo = b_mn ? ks * 2 * 1024 : (ks / 4) * b_katom + (ks % 4) * 32;
      const uint64_t ad = desc_sw128(smem_u32(As) + ao, a_mn ? a_lbo : 16, 1024);
      const uint64_t bd = desc_sw128(smem_u32(Bs) + bo, b_mn ? b_lbo : 16, 1024);
      mma_f16(tb, ad, bd, id, ks > 0);
    }
    commit(&bar);
  }
  if (!mbar_wait(&bar, 0, nullptr)) { if (tid == 0) atomicExch(err, 1); }
  fence_after_sync();
  for (int c = 0; c < N; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr(tb, warp * 32, c), r);
    tmem_wait_ld();
    const int row = warp * 32 + (tid & 31);
    for (int j = 0; j < 32 && c + j < N; ++j) D[row * N + c + j] = __uint_as_float(r[j]);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) { tmem_relinquish(); tmem_dealloc(tb, 256); }
}

extern "C" int umma_selftest_sw128(const void* A, const void* B, void* D, int N, int K, int a_mn,
                                   int b_mn, int* err) {
  if (K % 64 != 0 || K > 128 || N > 256 || N % 16 != 0) return -1;
  if (b_mn && N % 64 != 0) return -1;
  size_t smem = 128 * K * 2 + K * N * 2 + 1024;
  cudaFuncSetAttribute(gemm_sw128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  gemm_sw128_kernel<<<1, 128, smem>>>((const __half*)A, (const __half*)B, (float*)D, N, K, a_mn,
                                      b_mn, err);
  return (int)cudaDeviceSynchronize();
}
