// grad.cu -- packing and epilogue kernels of the gradient passes.
//
// Every gradient of the Gauss sum is assembled from forward passes of the fused
// kernels with augmented values ("Kernel matrix reduction", Variants: gradients
// run through the same fused reduction; the kernel tile is recomputed, never
// stored), followed by small per-point epilogues:
//
//   pass over rows x, columns y, values [w, w (y - z), w |y - z|^2]  ->  o_x
//     dL/dx[i,k] = -tau sum_c g_ic ((x_ik - z_k) o_x[i,c] - o_x[i, C + cD + k])
//     dL/dtau    = -1/2 sum_i sum_c g_ic (|x_i - z|^2 o_x[i,c]
//                      - 2 (x_i - z) . o_x[i, C + cD + :] + o_x[i, C(1+D) + c])
//   pass over rows y, columns x, values [g, g (x - z)]              ->  o_y
//     dL/dw[j,c] = o_y[j,c]
//     dL/dy[j,k] = -tau sum_c w_jc ((y_jk - z_k) o_y[j,c] - o_y[j, C + cD + k])
//
// z is the first row point of each batch: the identities hold for any z (the
// kernel only depends on differences), and centring keeps the values, and the
// cancellation between the two terms, at the scale of the point cloud's spread
// rather than of its distance from the origin.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "combine.cuh"
#include "internal.h"
#include "values.cuh"

namespace gs {
namespace {

template <typename T>
__device__ __forceinline__ float tf(T v);
template <>
__device__ __forceinline__ float tf<float>(float v) { return v; }
template <>
__device__ __forceinline__ float tf<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float tf<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148 * 32) b = 148 * 32;
  return static_cast<int>(b);
}

// Value matrix, float32 [B, N, CV] (CUDA-core path) -------------------------------
template <typename TS, typename TP>
__global__ void pack_values_f32_kernel(const TS* __restrict__ src, int64_t src_ld,
                                       const TP* __restrict__ cols, const TP* __restrict__ rows,
                                       float* __restrict__ v, int64_t B, int64_t N, int64_t Mrows,
                                       int D, int C, int mode) {
  const int CV = value_channels(mode, C, D);
  const int64_t total = B * N * CV;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t bj = e / CV;
    const int ch = static_cast<int>(e % CV);
    const int64_t b = bj / N;
    v[e] = value_at(src, cols, rows, b, bj, Mrows, D, C, ch, src_ld);
  }
}

// dL/dx (optional) and the per-row dL/dtau terms (optional) from o_x -------------
template <typename T>
__global__ void grad_x_epilogue_kernel(const T* __restrict__ x, const float* __restrict__ g,
                                       const float* __restrict__ o, float* __restrict__ gx,
                                       float* __restrict__ tau_rows, int64_t B, int64_t M, int D,
                                       int C, int CV, float tau) {
  const int64_t rows = B * M;
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = r / M;
    const T* xi = x + r * D;
    const T* z = x + b * M * D;
    const float* oi = o + r * CV;
    const float* gi = g + r * C;
    float tau_acc = 0.f;
    float xx = 0.f;
    for (int k = 0; k < D; ++k) {
      const float xk = tf(xi[k]) - tf(z[k]);
      xx = fmaf(xk, xk, xx);
      float s = 0.f;
      for (int c = 0; c < C; ++c) s = fmaf(gi[c], fmaf(xk, oi[c], -oi[C + c * D + k]), s);
      if (gx) gx[r * D + k] = -tau * s;
      if (tau_rows) {
        float cross = 0.f;
        for (int c = 0; c < C; ++c) cross = fmaf(gi[c], oi[C + c * D + k], cross);
        tau_acc = fmaf(-2.f * xk, cross, tau_acc);
      }
    }
    if (tau_rows) {
      for (int c = 0; c < C; ++c)
        tau_acc = fmaf(gi[c], fmaf(xx, oi[c], oi[C * (1 + D) + c]), tau_acc);
      tau_rows[r] = -0.5f * tau_acc;
    }
  }
}

// Forward + backward, one value channel (C = 1): the forward sum (unless `out`
// is null) and dL/dx straight from the x pass's split partials part[k][b, i, :] (k < splits,
// `stride` apart), summed in the fixed order of combine.cuh -- the same values
// the combine kernel would have written, so the results equal those of the
// combine followed by grad_x_epilogue_kernel bit for bit:
//     s = sum_k part[k][b,i,:],  out[b,i] = s[0],
//     dL/dx[b,i,k] = -tau g_i ((x_ik - z_k) s[0] - s[1 + k]).
// A block takes `tile_rows` consecutive rows at a time.  Their C V sums in each
// split slice are one contiguous run of floats: the block copies every slice's
// run into shared memory with coalesced loads, eight independent loads in
// flight per thread, then sums each element over the splits there in the fixed
// order (the same split_sum, on shared memory), and computes dL/dx with a warp
// per row.
constexpr int kEpiMaxRows = 32;
constexpr int kEpiThreads = 256;
constexpr int kEpiSmemFloats = 12 * 1024;   // 48 KB: splits + 1 runs of tile_rows * CV floats

template <typename T>
__global__ void __launch_bounds__(kEpiThreads)
    fwd_bwd_epilogue_kernel(const T* __restrict__ x, const float* __restrict__ g,
                            const float* __restrict__ part, int splits, int64_t stride,
                            float* __restrict__ out, float* __restrict__ gx, int64_t B, int64_t M,
                            int D, int CV, float tau, int tile_rows) {
  extern __shared__ float sm[];   // [splits][tile_rows * CV] copies, then [tile_rows * CV] sums
  __shared__ int64_t zoff[kEpiMaxRows];
  // a programmatic dependent of the kernel before it: wait for its results
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x;
  const int64_t rows = B * M;
  for (int64_t r0 = blockIdx.x * static_cast<int64_t>(tile_rows); r0 < rows;
       r0 += static_cast<int64_t>(gridDim.x) * tile_rows) {
    const int nr = static_cast<int>(min(static_cast<int64_t>(tile_rows), rows - r0));
    const int ne = nr * CV;
    const int n = splits * ne;
    const float* base = part + r0 * CV;
    // thread tid copies elements tid, tid + 256, ... of the concatenated runs:
    // (l, e) = split and offset of the next one, src = split l's run
    int l = tid / ne, e = tid - l * ne;
    const float* src = base + l * stride;
    constexpr int kPer = 8;
    for (int i0 = tid; i0 < n; i0 += kPer * kEpiThreads) {
      float v[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        v[u] = (i0 + u * kEpiThreads < n) ? src[e] : 0.f;
        e += kEpiThreads;
        while (e >= ne) {
          e -= ne;
          src += stride;
        }
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int idx = i0 + u * kEpiThreads;
        if (idx < n) sm[idx] = v[u];
      }
    }
    if (tid < nr) zoff[tid] = ((r0 + tid) / M) * M * D;   // the batch's first row point
    __syncthreads();
    float* sums = sm + n;
    for (int e2 = tid; e2 < ne; e2 += kEpiThreads) sums[e2] = split_sum(sm + e2, splits, ne);
    __syncthreads();
    if (out)
      for (int i = tid; i < nr; i += kEpiThreads) out[r0 + i] = sums[i * CV];
    if (gx) {
      // a warp per row, lanes over the dimensions
      const int warp = tid >> 5, lane = tid & 31;
      for (int i = warp; i < nr; i += kEpiThreads / 32) {
        const int64_t r = r0 + i;
        const float gi = g[r], s0 = sums[i * CV];
        const T* xr = x + r * D;
        const T* zr = x + zoff[i];
        float* gr = gx + r * D;
        for (int k = lane; k < D; k += 32) {
          const float xk = tf(xr[k]) - tf(zr[k]);
          const float t = gi * fmaf(xk, s0, -sums[i * CV + 1 + k]);
          gr[k] = -tau * t;
        }
      }
    }
    __syncthreads();
  }
}

// dL/dy (optional) and dL/dw from o_y ---------------------------------------------
template <typename T>
__global__ void grad_y_epilogue_kernel(const T* __restrict__ y, const T* __restrict__ w,
                                       const float* __restrict__ o, float* __restrict__ gy,
                                       float* __restrict__ gw, int64_t B, int64_t N, int D, int C,
                                       int CV, float tau) {
  const int64_t rows = B * N;
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = r / N;
    const T* yj = y + r * D;
    const T* z = y + b * N * D;
    const T* wj = w + r * C;
    const float* oj = o + r * CV;
    if (gw)
      for (int c = 0; c < C; ++c) gw[r * C + c] = oj[c];
    if (gy) {
      for (int k = 0; k < D; ++k) {
        const float yk = tf(yj[k]) - tf(z[k]);
        float s = 0.f;
        for (int c = 0; c < C; ++c) s = fmaf(tf(wj[c]), fmaf(yk, oj[c], -oj[C + c * D + k]), s);
        gy[r * D + k] = -tau * s;
      }
    }
  }
}

// out[r] (+)= factor * sum_{c in [c0, c0 + nc)} g[r, c] * o[r, c - c0]  (o rows nc wide)
__global__ void weighted_rows_kernel(const float* __restrict__ g, const float* __restrict__ o,
                                     float* __restrict__ out, int64_t rows, int C, int c0, int nc,
                                     float factor, int accumulate) {
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int c = 0; c < nc; ++c) s = fmaf(g[r * C + c0 + c], o[r * nc + c], s);
    out[r] = accumulate ? out[r] + factor * s : factor * s;
  }
}

// Fixed-order reduction of the per-row dL/dtau terms: one block, each thread
// sums a strided slice in order, then a fixed tree in shared memory.
__global__ void sum_rows_kernel(const float* __restrict__ v, int64_t n, float* __restrict__ out) {
  __shared__ double part[1024];
  double s = 0.0;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) s += static_cast<double>(v[e]);
  part[threadIdx.x] = s;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = static_cast<float>(part[0]);
}

// Log-sum-exp backward, channel c: o_x row = [A, B_k (D)] with A = sum_j p_ij and
// B = sum_j p_ij (y_j - z), and o_t row = T = sum_j p_ij |x^_i - y^_j|^2 (scaled
// squared distances).  A is 1 up to the rounding of lse, a factor common to
// every p_ij of the row, so dividing by A cancels it:
//   dL/dx_ik   += -tau g_ic ((x_ik - z_k) - B_k / A)
//   dL/dtau(i) += -1/2 g_ic (T / A) / (tau/2 log2 e)
// o rows have ocv channels; with ot == nullptr (ocv = 2 + D) the rows carry a
// third part (values mode 2):
// Q = sum_j p |y_j - z|^2, and sum_j p |x_i - y_j|^2 = Q - 2 (x_i - z).B + |x_i - z|^2 A.
__global__ void lse_x_tau_epilogue_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                          const float* __restrict__ o, const float* __restrict__ ot,
                                          float* __restrict__ gx, float* __restrict__ tau_rows,
                                          int64_t B, int64_t M, int D, int C, int c, float tau,
                                          float inv_cfac, int accumulate, int ocv) {
  const int64_t rows = B * M;
  const int CV = ocv;
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = r / M;
    const float* xi = x + r * D;
    const float* z = x + b * M * D;
    const float* oi = o + r * CV;
    const float gic = g[r * C + c];
    const float inv_a = 1.f / oi[0];
    if (gx) {
      for (int k = 0; k < D; ++k) {
        const float v = -tau * gic * ((xi[k] - z[k]) - oi[1 + k] * inv_a);
        gx[r * D + k] = accumulate ? gx[r * D + k] + v : v;
      }
    }
    if (tau_rows) {
      float dist;   // sum_j p |x_i - y_j|^2
      if (ot) {
        dist = ot[r] * inv_cfac;
      } else {
        float xb = 0.f, xx = 0.f;
        for (int k = 0; k < D; ++k) {
          const float d = xi[k] - z[k];
          xb = fmaf(d, oi[1 + k], xb);
          xx = fmaf(d, d, xx);
        }
        dist = oi[1 + D] - 2.f * xb + xx * oi[0];
      }
      const float v = -0.5f * gic * dist * inv_a;
      tau_rows[r] = accumulate ? tau_rows[r] + v : v;
    }
  }
}

// Log-sum-exp backward, channel c: o_y row = [A', B'_k (D)] with
// A' = sum_i g_ic K_ij e^-lse_ic, B' = sum_i g_ic K_ij e^-lse_ic (x_i - z).
//   dL/dw_jc   = A'
//   dL/dy_jk  += -tau w_jc ((y_jk - z_k) A' - B'_k)
__global__ void lse_grad_y_epilogue_kernel(const float* __restrict__ y, const float* __restrict__ w,
                                           const float* __restrict__ o, float* __restrict__ gy,
                                           float* __restrict__ gw, int64_t B, int64_t N, int D,
                                           int C, int c, float tau, int accumulate) {
  const int64_t rows = B * N;
  const int CV = 1 + D;
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = r / N;
    const float* yj = y + r * D;
    const float* z = y + b * N * D;
    const float* oj = o + r * CV;
    if (gw) gw[r * C + c] = oj[0];
    if (gy) {
      const float wjc = w[r * C + c];
      for (int k = 0; k < D; ++k) {
        const float v = -tau * wjc * fmaf(yj[k] - z[k], oj[0], -oj[1 + k]);
        gy[r * D + k] = accumulate ? gy[r * D + k] + v : v;
      }
    }
  }
}

// Elementwise steps of the diffusion operator (FlashDiffusion XGEMM section).
__global__ void diffusion_elementwise_kernel(int op, const float* __restrict__ a,
                                             const float* __restrict__ b2, float* __restrict__ o1,
                                             float* __restrict__ o2, int64_t n, int C,
                                             float alpha) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    switch (op) {
      case 0:   // o1 = 1
        o1[e] = 1.f;
        break;
      case 1:   // o1 = a^-alpha
        o1[e] = powf(a[e], -alpha);
        break;
      case 2: {   // a = q, b2 = K q^-alpha  ->  o1 = d = q^-alpha b2, o2 = s = q^-alpha d^-1/2
        const float qa = powf(a[e], -alpha);
        const float d = qa * b2[e];
        if (o1) o1[e] = d;
        o2[e] = qa * rsqrtf(d);
        break;
      }
      case 3:   // o1[e] = a[e / C] * b2[e]   (row scale of a [rows, C] block)
        o1[e] = a[e / C] * b2[e];
        break;
      default:
        break;
    }
  }
}

template <typename T>
const T* as(const void* p) {
  return static_cast<const T*>(p);
}

}  // namespace

cudaError_t launch_pack_values_f32(const void* src, int64_t src_ld, const void* cols,
                                   const void* rows, float* v, int64_t B, int64_t N, int64_t Mrows,
                                   int D, int C, int mode, cudaStream_t s) {
  const int64_t n = B * N * value_channels(mode, C, D);
  const int blocks = grid_for(n, 256);
  pack_values_f32_kernel<float, float><<<blocks, 256, 0, s>>>(
      as<float>(src), src_ld, as<float>(cols), as<float>(rows), v, B, N, Mrows, D, C, mode);
  return cudaGetLastError();
}

cudaError_t launch_fwd_bwd_epilogue(const void* x, gs_dtype dt, const float* g, const float* part,
                                    int splits, int64_t stride, float* out, float* grad_x,
                                    int64_t B, int64_t M, int D, int CV, float tau,
                                    cudaStream_t s) {
  // rows a tile: as many as the (splits + 1) runs of CV floats leave room for
  const int64_t fit = kEpiSmemFloats / (static_cast<int64_t>(splits + 1) * CV);
  if (fit < 1) return cudaErrorInvalidValue;   // splits and CV are bounded far below this
  const int tile_rows = static_cast<int>(fit < kEpiMaxRows ? fit : kEpiMaxRows);
  int64_t blocks = (B * M + tile_rows - 1) / tile_rows;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) blocks = 1;
  const unsigned nb = static_cast<unsigned>(blocks);
  const size_t smem = sizeof(float) * static_cast<size_t>(splits + 1) * tile_rows * CV;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nb);
  cfg.blockDim = dim3(kEpiThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (dt) {
    case GS_F32:
      return cudaLaunchKernelEx(&cfg, fwd_bwd_epilogue_kernel<float>, as<float>(x), g, part, splits,
                                stride, out, grad_x, B, M, D, CV, tau, tile_rows);
    case GS_F16:
      return cudaLaunchKernelEx(&cfg, fwd_bwd_epilogue_kernel<__half>, as<__half>(x), g, part,
                                splits, stride, out, grad_x, B, M, D, CV, tau, tile_rows);
    default:
      return cudaLaunchKernelEx(&cfg, fwd_bwd_epilogue_kernel<__nv_bfloat16>, as<__nv_bfloat16>(x),
                                g, part, splits, stride, out, grad_x, B, M, D, CV, tau, tile_rows);
  }
}

cudaError_t launch_grad_x_epilogue(const void* x, gs_dtype dt, const float* g, const float* o,
                                   float* grad_x, float* tau_rows, int64_t B, int64_t M, int D,
                                   int C, int CV, float tau, cudaStream_t s) {
  const int blocks = grid_for(B * M, 256);
  switch (dt) {
    case GS_F32:
      grad_x_epilogue_kernel<float><<<blocks, 256, 0, s>>>(as<float>(x), g, o, grad_x, tau_rows, B,
                                                           M, D, C, CV, tau);
      break;
    case GS_F16:
      grad_x_epilogue_kernel<__half><<<blocks, 256, 0, s>>>(as<__half>(x), g, o, grad_x, tau_rows,
                                                            B, M, D, C, CV, tau);
      break;
    default:
      grad_x_epilogue_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
          as<__nv_bfloat16>(x), g, o, grad_x, tau_rows, B, M, D, C, CV, tau);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_grad_y_epilogue(const void* y, const void* w, gs_dtype dt, const float* o,
                                   float* grad_y, float* grad_w, int64_t B, int64_t N, int D,
                                   int C, int CV, float tau, cudaStream_t s) {
  const int blocks = grid_for(B * N, 256);
  switch (dt) {
    case GS_F32:
      grad_y_epilogue_kernel<float><<<blocks, 256, 0, s>>>(as<float>(y), as<float>(w), o, grad_y,
                                                           grad_w, B, N, D, C, CV, tau);
      break;
    case GS_F16:
      grad_y_epilogue_kernel<__half><<<blocks, 256, 0, s>>>(as<__half>(y), as<__half>(w), o,
                                                            grad_y, grad_w, B, N, D, C, CV, tau);
      break;
    default:
      grad_y_epilogue_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
          as<__nv_bfloat16>(y), as<__nv_bfloat16>(w), o, grad_y, grad_w, B, N, D, C, CV, tau);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_lse_x_tau_epilogue(const float* x, const float* g, const float* o,
                                      const float* ot, float* grad_x, float* tau_rows, int64_t B,
                                      int64_t M, int D, int C, int c, float tau, float inv_cfac,
                                      bool accumulate, cudaStream_t s, int ocv) {
  lse_x_tau_epilogue_kernel<<<grid_for(B * M, 256), 256, 0, s>>>(
      x, g, o, ot, grad_x, tau_rows, B, M, D, C, c, tau, inv_cfac, accumulate ? 1 : 0, ocv);
  return cudaGetLastError();
}

cudaError_t launch_lse_grad_y_epilogue(const float* y, const float* w, const float* o,
                                       float* grad_y, float* grad_w, int64_t B, int64_t N, int D,
                                       int C, int c, float tau, bool accumulate, cudaStream_t s) {
  lse_grad_y_epilogue_kernel<<<grid_for(B * N, 256), 256, 0, s>>>(y, w, o, grad_y, grad_w, B, N, D,
                                                                  C, c, tau, accumulate ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_weighted_rows(const float* g, const float* o, float* tau_rows, int64_t rows,
                                 int C, int c0, int nc, float factor, bool accumulate,
                                 cudaStream_t s) {
  weighted_rows_kernel<<<grid_for(rows, 256), 256, 0, s>>>(g, o, tau_rows, rows, C, c0, nc, factor,
                                                           accumulate ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_diffusion_elementwise(int op, const float* a, const float* b, float* o1,
                                         float* o2, int64_t n, int C, float alpha,
                                         cudaStream_t s) {
  diffusion_elementwise_kernel<<<grid_for(n, 256), 256, 0, s>>>(op, a, b, o1, o2, n, C, alpha);
  return cudaGetLastError();
}

template <typename T>
__global__ void widen_kernel(const T* __restrict__ src, float* __restrict__ dst, int64_t n) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[e] = tf(src[e]);
}

cudaError_t launch_widen_to_f32(const void* src, gs_dtype dt, float* dst, int64_t n,
                                cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int blocks = grid_for(n, 256);
  if (dt == GS_F16)
    widen_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(src), dst, n);
  else if (dt == GS_BF16)
    widen_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), dst, n);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_sum_rows(const float* v, int64_t n, float* out, cudaStream_t s) {
  sum_rows_kernel<<<1, 1024, 0, s>>>(v, n, out);
  return cudaGetLastError();
}

}  // namespace gs
