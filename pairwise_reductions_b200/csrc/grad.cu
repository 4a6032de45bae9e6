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
// One warp per row; lanes over the D dimensions (coalesced reads of x, of each
// split's sums and of the gradient row).
template <typename T>
__global__ void fwd_bwd_epilogue_kernel(const T* __restrict__ x, const float* __restrict__ g,
                                        const float* __restrict__ part, int splits,
                                        int64_t stride, float* __restrict__ out,
                                        float* __restrict__ gx, int64_t B, int64_t M, int D,
                                        int CV, float tau) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = B * M;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    const int64_t b = r / M;
    const float* o = part + r * CV;
    const float s0 = split_sum(o, splits, stride);
    if (lane == 0 && out) out[r] = s0;
    if (!gx) continue;
    const float gi = g[r];
    const T* xi = x + r * D;
    const T* z = x + b * M * D;
    for (int k = lane; k < D; k += 32) {
      const float xk = tf(xi[k]) - tf(z[k]);
      const float t = gi * fmaf(xk, s0, -split_sum(o + 1 + k, splits, stride));
      gx[r * D + k] = -tau * t;
    }
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
  int64_t blocks = (B * M + 7) / 8;   // 8 warps a block, one row each
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) blocks = 1;
  const unsigned nb = static_cast<unsigned>(blocks);
  switch (dt) {
    case GS_F32:
      fwd_bwd_epilogue_kernel<float><<<nb, 256, 0, s>>>(as<float>(x), g, part, splits, stride, out,
                                                        grad_x, B, M, D, CV, tau);
      break;
    case GS_F16:
      fwd_bwd_epilogue_kernel<__half><<<nb, 256, 0, s>>>(as<__half>(x), g, part, splits, stride, out,
                                                         grad_x, B, M, D, CV, tau);
      break;
    default:
      fwd_bwd_epilogue_kernel<__nv_bfloat16><<<nb, 256, 0, s>>>(
          as<__nv_bfloat16>(x), g, part, splits, stride, out, grad_x, B, M, D, CV, tau);
      break;
  }
  return cudaGetLastError();
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
