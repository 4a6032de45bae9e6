// knn.cu -- the k-nearest reduction (min / argKmin) on the CUDA-core path
// (fp32, 1 <= D <= 128, 1 <= K <= 32).
//
// For each row i: the K smallest squared distances |x_i - y_j|^2 over j,
// ascending, with their indices, equal distances ordered by the lower index
// ("Kernel matrix reduction", Overview: minima and the indices of the K
// smallest entries per row are among the reductions; the .argmin() reduction
// of the LazyTensor API).  The largest Gaussian kernel value of a row is
// exp(-tau/2 * dist[0]).
//
// Every distance is computed as e_k = x_k - y_k, d = e_0 e_0, d = fma(e_k, e_k, d)
// for k = 1 .. D-1, each rounded to nearest in fp32 (two rows per packed
// .f32x2 instruction), so the integer results are decided by exactly the fp32
// values of that formula.  A CTA keeps R rows per thread with a sorted list of
// K (distance, index) in registers and streams the sources through shared
// memory; within one thread the indices arrive in increasing order, so a
// strict "<" against the current K-th distance keeps the lower index on ties.
// Column splits are merged afterwards, ties again by the lower index.
// D > 8: the rows' coordinates no longer fit in registers, so a tile of TJ
// points is staged 8 dimensions at a time and every (row, point) pair keeps
// its partial distance in a register across the chunks -- the same fp32
// operations in the same order (fma(e_k, e_k, d) for ascending k, starting
// from fma(e_0, e_0, +0) = e_0 e_0), so the decisions are unchanged.
#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace gs {
namespace {

constexpr int kThreads = 128;
constexpr int kTileJ = 256;
constexpr int kPer = kTileJ / kThreads;

__host__ __device__ constexpr int knn_rows(int K) { return K <= 8 ? 4 : 2; }

template <int K>
__device__ __forceinline__ void insert(float (&bd)[K], int (&bj)[K], float d, int j) {
  // d < bd[K-1] holds; shift the larger entries up by one and place d
#pragma unroll
  for (int p = K - 1; p >= 0; --p) {
    const bool before = (p > 0) && (d < bd[p > 0 ? p - 1 : 0]);
    const bool here = d < bd[p];
    const float nd = before ? bd[p > 0 ? p - 1 : 0] : (here ? d : bd[p]);
    const int nj = before ? bj[p > 0 ? p - 1 : 0] : (here ? j : bj[p]);
    bd[p] = nd;
    bj[p] = nj;
  }
}

template <int D, int K>
__global__ void __launch_bounds__(kThreads)
    knn_kernel(const float* __restrict__ x, const float* __restrict__ y, float* __restrict__ od,
               int* __restrict__ oi, int64_t M, int64_t N, int64_t cols_per_split,
               int64_t split_stride, int Kout) {
  constexpr int R = knn_rows(K);
  constexpr int RP = R / 2;
  constexpr int PK = ((2 * D + 3) / 4) * 4;   // duplicated negated coordinates per point
  __shared__ __align__(16) float tile[kTileJ * PK];

  const int tid = threadIdx.x;
  const int64_t b = blockIdx.z;
  const int split = blockIdx.y;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (kThreads * R);
  const int64_t jbeg = static_cast<int64_t>(split) * cols_per_split;
  const int64_t jend = min(N, jbeg + cols_per_split);
  const float* __restrict__ yb = y + b * N * D;

  uint64_t xs[RP][D];
#pragma unroll
  for (int q = 0; q < RP; ++q) {
    const int64_t i0 = row0 + tid + (2 * q) * kThreads;
    const int64_t i1 = i0 + kThreads;
#pragma unroll
    for (int k = 0; k < D; ++k)
      xs[q][k] = pk2(i0 < M ? x[(b * M + i0) * D + k] : 0.f, i1 < M ? x[(b * M + i1) * D + k] : 0.f);
  }
  float bd[R][K];
  int bj[R][K];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int p = 0; p < K; ++p) {
      bd[r][p] = INFINITY;
      bj[r][p] = -1;
    }

  for (int64_t j0 = jbeg; j0 < jend; j0 += kTileJ) {
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int64_t j = j0 + tid + q * kThreads;
      float* p = tile + (tid + q * kThreads) * PK;
      // columns past the end sit at +inf distance (never selected)
#pragma unroll
      for (int k = 0; k < D; ++k) {
        const float v = (j < jend) ? -yb[j * D + k] : -INFINITY;
        p[2 * k] = v;
        p[2 * k + 1] = v;
      }
#pragma unroll
      for (int k = 2 * D; k < PK; ++k) p[k] = 0.f;
    }
    __syncthreads();
    const ulonglong2* t2 = reinterpret_cast<const ulonglong2*>(tile);
    const int jlim = static_cast<int>((jend - j0) < kTileJ ? (jend - j0) : kTileJ);
    for (int jj = 0; jj < jlim; ++jj) {
      uint64_t pk[PK / 2];
#pragma unroll
      for (int v = 0; v < PK / 4; ++v) {
        const ulonglong2 u = t2[jj * (PK / 4) + v];
        pk[2 * v] = u.x;
        pk[2 * v + 1] = u.y;
      }
      const int j = static_cast<int>(j0 + jj);
#pragma unroll
      for (int q = 0; q < RP; ++q) {
        uint64_t e = add2(xs[q][0], pk[0]);
        uint64_t d2 = mul2(e, e);
#pragma unroll
        for (int k = 1; k < D; ++k) {
          e = add2(xs[q][k], pk[k]);
          d2 = fma2(e, e, d2);
        }
        float d0, d1;
        upk2(d2, d0, d1);
        if (d0 < bd[2 * q][K - 1]) insert<K>(bd[2 * q], bj[2 * q], d0, j);
        if (d1 < bd[2 * q + 1][K - 1]) insert<K>(bd[2 * q + 1], bj[2 * q + 1], d1, j);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = row0 + tid + r * kThreads;
    if (i >= M) continue;
    const int64_t base = split * split_stride + (b * M + i) * Kout;
#pragma unroll
    for (int p = 0; p < K; ++p) {
      if (p >= Kout) break;
      od[base + p] = bd[r][p];
      oi[base + p] = bj[r][p];
    }
  }
}

constexpr int kDC = 8;   // dimensions per staged chunk (wide kernel)

template <int K, int TJ>
__global__ void __launch_bounds__(kThreads)
    knn_wide_kernel(const float* __restrict__ x, const float* __restrict__ y, float* __restrict__ od,
                    int* __restrict__ oi, int64_t M, int64_t N, int D, int64_t cols_per_split,
                    int64_t split_stride, int Kout) {
  // negated coordinates of TJ points x 8 dimensions, each duplicated for the
  // packed (two-row) arithmetic
  __shared__ __align__(16) float tile[TJ][2 * kDC];
  const int tid = threadIdx.x;
  const int64_t b = blockIdx.z;
  const int split = blockIdx.y;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * (2 * kThreads) + tid;
  const int64_t i1 = i0 + kThreads;
  const int64_t jbeg = static_cast<int64_t>(split) * cols_per_split;
  const int64_t jend = min(N, jbeg + cols_per_split);
  const float* __restrict__ x0 = x + (b * M + i0) * D;
  const float* __restrict__ x1 = x + (b * M + i1) * D;
  const float* __restrict__ yb = y + b * N * D;
  float bd[2][K];
  int bj[2][K];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int p = 0; p < K; ++p) {
      bd[r][p] = INFINITY;
      bj[r][p] = -1;
    }
  for (int64_t j0 = jbeg; j0 < jend; j0 += TJ) {
    uint64_t d[TJ];
#pragma unroll
    for (int jj = 0; jj < TJ; ++jj) d[jj] = 0ull;   // +0: fma(e_0, e_0, +0) = e_0 e_0
    for (int k0 = 0; k0 < D; k0 += kDC) {
      __syncthreads();   // the previous chunk has been read
      for (int idx = tid; idx < TJ * kDC; idx += kThreads) {
        const int jj = idx / kDC, kk = idx % kDC;
        const int64_t j = j0 + jj;
        const int k = k0 + kk;
        const float v = (j < jend && k < D) ? -yb[j * D + k] : 0.f;
        tile[jj][2 * kk] = v;
        tile[jj][2 * kk + 1] = v;
      }
      __syncthreads();
      // dimensions past D are 0 on both sides: fma(0, 0, d) = d exactly
      uint64_t xk[kDC];
#pragma unroll
      for (int kk = 0; kk < kDC; ++kk) {
        const int k = k0 + kk;
        xk[kk] = pk2((i0 < M && k < D) ? x0[k] : 0.f, (i1 < M && k < D) ? x1[k] : 0.f);
      }
      const ulonglong2* t2 = reinterpret_cast<const ulonglong2*>(&tile[0][0]);
#pragma unroll
      for (int jj = 0; jj < TJ; ++jj) {
#pragma unroll
        for (int v = 0; v < kDC / 2; ++v) {
          const ulonglong2 u = t2[jj * (kDC / 2) + v];
          uint64_t e = add2(xk[2 * v], u.x);
          d[jj] = fma2(e, e, d[jj]);
          e = add2(xk[2 * v + 1], u.y);
          d[jj] = fma2(e, e, d[jj]);
        }
      }
    }
#pragma unroll
    for (int jj = 0; jj < TJ; ++jj) {
      const int64_t j = j0 + jj;
      if (j >= jend) break;
      float d0, d1;
      upk2(d[jj], d0, d1);
      if (d0 < bd[0][K - 1]) insert<K>(bd[0], bj[0], d0, static_cast<int>(j));
      if (d1 < bd[1][K - 1]) insert<K>(bd[1], bj[1], d1, static_cast<int>(j));
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int64_t i = r ? i1 : i0;
    if (i >= M) continue;
    const int64_t base = split * split_stride + (b * M + i) * Kout;
#pragma unroll
    for (int p = 0; p < K; ++p) {
      if (p >= Kout) break;
      od[base + p] = bd[r][p];
      oi[base + p] = bj[r][p];
    }
  }
}

// Merge the sorted per-split lists of each row (ties by the lower index) and
// write the final distances and 64-bit indices.
__global__ void knn_merge_kernel(const float* __restrict__ pd, const int* __restrict__ pi,
                                 int splits, int64_t split_stride, int64_t rows, int K,
                                 float* __restrict__ out_d, int64_t* __restrict__ out_i) {
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int head[32];
    for (int s = 0; s < splits; ++s) head[s] = 0;
    for (int p = 0; p < K; ++p) {
      int best = -1;
      float bd = INFINITY;
      int bi = 0x7fffffff;
      for (int s = 0; s < splits; ++s) {
        if (head[s] >= K) continue;
        const int64_t e = s * split_stride + r * K + head[s];
        const float d = pd[e];
        const int j = pi[e];
        if (j < 0) continue;
        if (d < bd || (d == bd && j < bi)) {
          bd = d;
          bi = j;
          best = s;
        }
      }
      if (best >= 0) {
        ++head[best];
        out_d[r * K + p] = bd;
        out_i[r * K + p] = bi;
      } else {
        out_d[r * K + p] = INFINITY;
        out_i[r * K + p] = -1;
      }
    }
  }
}

template <int D, int K>
cudaError_t launch_t(const KnnArgs& a, cudaStream_t s) {
  constexpr int R = knn_rows(K);
  const int64_t tiles = (a.M + kThreads * R - 1) / (kThreads * R);
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(a.splits),
                  static_cast<unsigned>(a.B));
  knn_kernel<D, K><<<grid, kThreads, 0, s>>>(a.x, a.y, a.part_d, a.part_i, a.M, a.N,
                                             a.cols_per_split, a.split_stride, a.K);
  return cudaGetLastError();
}

template <int K>
cudaError_t launch_wide_t(const KnnArgs& a, cudaStream_t s) {
  constexpr int TJ = K >= 16 ? 16 : 32;
  const int64_t tiles = (a.M + 2 * kThreads - 1) / (2 * kThreads);
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(a.splits),
                  static_cast<unsigned>(a.B));
  knn_wide_kernel<K, TJ><<<grid, kThreads, 0, s>>>(a.x, a.y, a.part_d, a.part_i, a.M, a.N, a.D,
                                                   a.cols_per_split, a.split_stride, a.K);
  return cudaGetLastError();
}

cudaError_t launch_wide(const KnnArgs& a, cudaStream_t s) {
  if (a.K <= 1) return launch_wide_t<1>(a, s);
  if (a.K <= 2) return launch_wide_t<2>(a, s);
  if (a.K <= 4) return launch_wide_t<4>(a, s);
  if (a.K <= 8) return launch_wide_t<8>(a, s);
  if (a.K <= 16) return launch_wide_t<16>(a, s);
  return launch_wide_t<32>(a, s);
}

template <int D>
cudaError_t launch_k(const KnnArgs& a, cudaStream_t s) {
  if (a.K <= 1) return launch_t<D, 1>(a, s);
  if (a.K <= 2) return launch_t<D, 2>(a, s);
  if (a.K <= 4) return launch_t<D, 4>(a, s);
  if (a.K <= 8) return launch_t<D, 8>(a, s);
  if (a.K <= 16) return launch_t<D, 16>(a, s);
  return launch_t<D, 32>(a, s);
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148 * 32) b = 148 * 32;
  return static_cast<int>(b);
}

}  // namespace

KnnPlan knn_plan(int64_t B, int64_t M, int64_t N, int64_t D, int K, int sm_count) {
  KnnPlan p{};
  const int R = D > 8 ? 2
                      : knn_rows(K <= 1 ? 1 : (K <= 2 ? 2 : (K <= 4 ? 4 : (K <= 8 ? 8 : (K <= 16 ? 16 : 32)))));
  const int64_t U = B * ((M + kThreads * R - 1) / (kThreads * R));
  int64_t smax = N / 512;
  if (smax > 32) smax = 32;
  if (smax < 1) smax = 1;
  int best = 1;
  double best_cost = 1e300;
  for (int64_t S = 1; S <= smax; ++S) {
    int64_t per_sm = (U * S + sm_count - 1) / sm_count;
    if (per_sm < 8) per_sm = 8;
    const double cost = static_cast<double>(per_sm) * static_cast<double>((N + S - 1) / S + 128);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = static_cast<int>(S);
    }
  }
  p.cols_per_split = (N + best - 1) / best;
  if (p.cols_per_split < 1) p.cols_per_split = 1;
  p.splits = static_cast<int>((N + p.cols_per_split - 1) / p.cols_per_split);
  if (p.splits < 1) p.splits = 1;
  return p;
}

cudaError_t launch_knn(const KnnArgs& a, cudaStream_t s) {
  cudaError_t e;
  switch (a.D) {
    case 1: e = launch_k<1>(a, s); break;
    case 2: e = launch_k<2>(a, s); break;
    case 3: e = launch_k<3>(a, s); break;
    case 4: e = launch_k<4>(a, s); break;
    case 5: e = launch_k<5>(a, s); break;
    case 6: e = launch_k<6>(a, s); break;
    case 7: e = launch_k<7>(a, s); break;
    case 8: e = launch_k<8>(a, s); break;
    default:
      if (a.D > 128) return cudaErrorInvalidValue;
      e = launch_wide(a, s);
      break;
  }
  if (e != cudaSuccess) return e;
  const int64_t rows = a.B * a.M;
  knn_merge_kernel<<<grid_for(rows, 128), 128, 0, s>>>(a.part_d, a.part_i, a.splits,
                                                       a.split_stride, rows, a.K, a.out_d, a.out_i);
  return cudaGetLastError();
}

}  // namespace gs
