// probes.cu -- measurement probes behind two test hooks of gauss_testing.h:
// the MUFU ex2 rate of an SM (the denominator of the roofline that the
// benchmark reports for the exponential-bound kernels) and the cost of
// back-to-back tcgen05.mma kind::f16 instructions issued by one thread (which
// bounds the tensor-core kernels' MMA-issuing thread).  They exist so that the
// figures the design rests on can be re-measured from this repository; no
// kernel of the computation uses them.
#include "internal.h"
#include "ptx.cuh"

namespace gs {
namespace {

constexpr int kEx2Threads = 1024;
constexpr int kEx2Chains = 8;
// dynamic shared memory that keeps every probe CTA alone on its SM
constexpr int kProbeSmem = 120 * 1024;

// Each thread runs kEx2Chains independent chains v <- 2^(-v/2) (one FMUL and
// one MUFU ex2 a step; the values settle near 0.77, far from subnormals), with
// 32 warps a CTA to cover the MUFU latency.  Thread 0 reads the SM clock around
// the CTA's loop (between two CTA barriers): cycles[block].  sink[thread] keeps
// the chains live.
__global__ void __launch_bounds__(kEx2Threads, 1)
    ex2_probe_kernel(long long* cycles, float* sink, int iters) {
  float v[kEx2Chains];
#pragma unroll
  for (int c = 0; c < kEx2Chains; ++c) v[c] = 0.25f * static_cast<float>(c + 1) + 1e-4f * threadIdx.x;
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < kEx2Chains; ++c) v[c] = ex2(-0.5f * v[c]);
  }
  __syncthreads();
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kEx2Chains; ++c) s += v[c];
  sink[static_cast<int64_t>(blockIdx.x) * kEx2Threads + threadIdx.x] = s;
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// One thread issues n_mma MMAs D[TMEM] (+)= A B^T of M = 128, N = n_cols, K = 16
// (kind::f16, both operands zero in shared memory, one accumulator), commits
// them to an mbarrier and waits for it (bounded: 2 s); cycles[block] = the SM
// cycles from the first issue to the completion, or -1 (and *status |= 1) if
// the wait ran out.  Shared memory: A 128 rows x 128 B, B 256 rows x 128 B
// (128-byte-swizzled K-major atoms, as the kernels' operands), the mbarrier and
// the TMEM address slot.
__global__ void __launch_bounds__(128, 1)
    mma_probe_kernel(long long* cycles, int* status, int n_mma, int n_cols) {
  extern __shared__ uint8_t probe_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(probe_smem) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int kA = 128 * 128, kB = 256 * 128;
  uint8_t* sA = base;
  uint8_t* sB = base + kA;
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + kA + kB);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  for (int q = threadIdx.x; q < (kA + kB) / 16; q += blockDim.x)
    reinterpret_cast<uint4*>(base)[q] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();   // the zeros, visible to the tensor core
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(bar), 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_f16(0, 128, static_cast<uint32_t>(n_cols));
    const uint64_t da = desc_k_sw128(smem_u32(sA));
    const uint64_t db = desc_k_sw128(smem_u32(sB));
    const long long t0 = clock64();
    for (int q = 0; q < n_mma; ++q) mma_ss(tmem, da, db, idesc, q > 0 ? 1u : 0u);
    mma_commit(smem_u32(bar));
    bool done = false;
    const uint64_t g0 = global_timer_ns();
    while (!done) {
      done = mbar_try_wait(smem_u32(bar), 0);
      if (!done && global_timer_ns() - g0 > 2000000000ull) break;
    }
    const long long t1 = clock64();
    cycles[blockIdx.x] = done ? t1 - t0 : -1;
    if (!done) atomicOr(status, 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tmem, 512);
}

}  // namespace
}  // namespace gs

extern "C" gs_status gs_test_ex2_probe(long long* cycles, float* sink, int blocks, int iters,
                                       gs_stream_t stream) {
  if (!cycles || !sink || blocks < 1 || blocks > 4096 || iters < 1 || iters > (1 << 20))
    return GS_ERR_INVALID_ARG;
  if (cudaFuncSetAttribute(gs::ex2_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gs::kProbeSmem) != cudaSuccess) {
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  gs::ex2_probe_kernel<<<blocks, gs::kEx2Threads, gs::kProbeSmem,
                         reinterpret_cast<cudaStream_t>(stream)>>>(cycles, sink, iters);
  return cudaGetLastError() == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}

extern "C" gs_status gs_test_mma_probe(long long* cycles, int* status, int blocks, int n_mma,
                                       int n_cols, gs_stream_t stream) {
  if (!cycles || !status || blocks < 1 || blocks > 4096 || n_mma < 1 || n_mma > 65536 ||
      (n_cols != 32 && n_cols != 64 && n_cols != 128 && n_cols != 256))
    return GS_ERR_INVALID_ARG;
  if (cudaFuncSetAttribute(gs::mma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gs::kProbeSmem) != cudaSuccess) {
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  gs::mma_probe_kernel<<<blocks, 128, gs::kProbeSmem, reinterpret_cast<cudaStream_t>(stream)>>>(
      cycles, status, n_mma, n_cols);
  return cudaGetLastError() == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}
