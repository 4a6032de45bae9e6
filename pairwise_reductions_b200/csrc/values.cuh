// values.cuh -- the value matrices of the forward and gradient passes.
//
// A pass reduces K(row_i, col_j) * v[j, :] over the columns j.  Its values are
// built from a source array src [B, Ncols, C] (the weights, or the upstream
// gradient when the roles of the points are swapped) and the column points:
//   mode 0:  v = src                                               C channels
//   mode 1:  v = [src, src (col - z)]                       C (1 + D) channels
//   mode 2:  v = [src, src (col - z), src |col - z|^2]      C (2 + D) channels
// with z = rows[b, 0, :], the first row point of the batch (see grad.cu).
// Channel C + c D + k holds src[c] (col_k - z_k); channel C (1 + D) + c holds
// src[c] |col - z|^2.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace gs {

__host__ __device__ inline int value_channels(int mode, int C, int D) {
  return mode == 0 ? C : (mode == 1 ? C * (1 + D) : C * (2 + D));
}

__device__ __forceinline__ float vf(float v) { return v; }
__device__ __forceinline__ float vf(__half v) { return __half2float(v); }
__device__ __forceinline__ float vf(__nv_bfloat16 v) { return __bfloat162float(v); }

// Channel ch of the values of column bj = b * Ncols + j; src rows are src_ld apart.
template <typename TS, typename TP>
__device__ __forceinline__ float value_at(const TS* __restrict__ src, const TP* __restrict__ cols,
                                          const TP* __restrict__ rows, int64_t b, int64_t bj,
                                          int64_t Mrows, int D, int C, int ch, int64_t src_ld) {
  if (ch < C) return vf(src[bj * src_ld + ch]);
  const TP* z = rows + b * Mrows * D;
  const TP* col = cols + bj * D;
  if (ch < C * (1 + D)) {
    const int c = (ch - C) / D, k = (ch - C) % D;
    return vf(src[bj * src_ld + c]) * (vf(col[k]) - vf(z[k]));
  }
  const int c = ch - C * (1 + D);
  float q = 0.f;
  for (int k = 0; k < D; ++k) {
    const float d = vf(col[k]) - vf(z[k]);
    q = fmaf(d, d, q);
  }
  return vf(src[bj * src_ld + c]) * q;
}

}  // namespace gs
