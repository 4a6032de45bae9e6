// noalloc.cu -- an allocation-free variant of gauss_sum_fwd.
//
// Some callers cannot allocate device memory for the workspace: a plugin whose
// host application owns the whole device-memory budget, a latency-critical
// loop that must never block in the CUDA allocator, or a process running under
// a hard memory cap where a per-call allocation could fail half-way through a
// job.  For them, gauss_sum_fwd_noalloc runs exactly the kernels of
// gauss_sum_fwd but takes its scratch (packed operands, norms, split partials)
// from a fixed array compiled into this library instead of a caller buffer.
//
// Costs and limits:
//   * the array is part of this file's own module (the library is built
//     without relocatable device code, so each source file is one module):
//     kScratchBytes (32 MiB) of device memory per device context, held until
//     the process exits -- on every context the process creates when modules
//     load eagerly (CUDA_MODULE_LOADING=EAGER), and under lazy loading (the
//     default) only on devices where this entry point has been called;
//   * a call whose scratch need exceeds 32 MiB is rejected with
//     GS_ERR_WORKSPACE (use gauss_sum_fwd with a caller workspace instead);
//   * all calls on a device share the one array, so calls that overlap on the
//     GPU (different streams, or different host threads without ordering) race
//     on it; calls on one stream are ordered and safe;
//   * the array keeps whatever the last call left in it.  Nothing needs to be
//     cleared first: every scratch byte a call reads was written earlier in the
//     same call.
// The first call on each device looks up the device address of the array
// (cudaGetSymbolAddress) with that device current; that first call should come
// before any stream capture.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
gs_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();   // leave no error behind for the next, unrelated call to report
    return GS_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return GS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return GS_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GS_OK;
}

}  // namespace

extern "C" gs_status gauss_sum_fwd_noalloc(const void* x, const void* y, const void* w, float* out,
                                           int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                                           float tau, gs_dtype dt, gs_stream_t stream) {
  // argument errors first, reported exactly as gauss_sum_fwd reports them
  // (that call rejects them before it looks at the workspace or enqueues anything)
  const size_t need = gs_workspace_bytes(GS_OP_SUM, B, M, N, D, C, dt);
  const bool bad_ptr = [&] {
    auto bad = [](const void* p, int64_t n) {
      return n > 0 && (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) != 0);
    };
    return bad(x, B * M * D) || bad(y, B * N * D) || bad(w, B * N * C) || bad(out, B * M * C);
  }();
  if (need == static_cast<size_t>(-1) || !(std::isfinite(tau) && tau > 0.f) || bad_ptr)
    return gauss_sum_fwd(x, y, w, out, B, M, N, D, C, tau, dt, nullptr, 0, stream);
  if (need > kScratchBytes) return GS_ERR_WORKSPACE;
  if (need == 0) return gauss_sum_fwd(x, y, w, out, B, M, N, D, C, tau, dt, nullptr, 0, stream);
  void* scratch = nullptr;
  const gs_status st = scratch_for_current_device(&scratch);
  if (st != GS_OK) return st;
  return gauss_sum_fwd(x, y, w, out, B, M, N, D, C, tau, dt, scratch, kScratchBytes, stream);
}
