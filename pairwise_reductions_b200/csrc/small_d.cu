// small_d.cu -- CUDA-core kernels for the Gaussian kernel sum and its
// log-sum-exp at small feature width (fp32, 1 <= D <= 8).
//
// Computes ("Kernel matrix reduction", Implementation sketch, eq. 1)
//     a[b,i,c] = sum_j exp(-tau/2 |x_i - y_j|^2) w[b,j,c]
// and the weighted log-sum-exp of the same page's Overview, without forming
// the kernel matrix.  Design:
//   * coordinates are pre-multiplied by s = sqrt(tau/2 * log2 e), so each
//     kernel value is a single MUFU ex2 of -|x^ - y^|^2 (direct difference
//     form: 3 FADD + 1 FMUL + 2 FFMA per pair at D = 3, one FFMA to
//     accumulate);
//   * a CTA keeps R rows per thread (x^ and accumulators in registers) and
//     streams y/w through shared memory in tiles of 256 points, packed
//     per point as {y^_0 .. y^_{D-1}, v_0 .. v_{CP-1}} so one broadcast
//     LDS.128 feeds R * CP kernel evaluations;
//   * each tile is summed into a tile accumulator before it joins the running
//     total (two-level summation keeps fp32 rounding well below 1e-5 relative
//     at 10^6 terms with signed weights);
//   * the column range is split over CTAs when there are too few row tiles
//     to fill 148 SMs; partials are combined in a fixed order afterwards.
// Log-sum-exp: the weights enter as log2 w; every tile shifts them by the
// running maximum of log2 w over the tiles seen so far (a uniform upper bound
// of every exponent, since the kernel is at most 1), rescaling the
// accumulator when the maximum grows -- the online normaliser of Milakov and
// Gimelshein that the FlashDiffusion page cites, with the bound taken from
// the weights.  Rows whose scaled sum comes out tiny are recomputed exactly
// (per-row maximum) by the finalisation kernel.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "../../include/gauss_testing.h"
#include "combine.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace gs {
namespace {

constexpr int kTileJ = 256;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, int CP, int SHIFT = 0>
struct PackShape {
  // floats per staged point: D duplicated negated coordinates, CP duplicated
  // values (and, for a per-column exponent shift, the duplicated shift), so
  // every operand of the packed (two-row) arithmetic is one 64-bit load
  static constexpr int NPAIR = D + CP + (SHIFT == 2 ? 1 : 0);
  static constexpr int PK = ((2 * NPAIR + 3) / 4) * 4;
};

// Row pairs per thread that take the FMA-pipe exp2 instead of MUFU ex2.  None:
// measured on B200, the packed distance arithmetic already keeps the FMA pipe
// about as busy as the exponentials keep MUFU, and the polynomial (about five
// FMA-pipe instructions per value) costs more than the MUFU slot it frees.
template <int D, int CP, int R>
__host__ __device__ constexpr int poly_pairs() {
  return 0;
}

// 2^e for an integer e (0 below 2^-126), built from its exponent bits: exact.
__device__ __forceinline__ float pow2i(float e) {
  if (!(e >= -126.f)) return 0.f;
  return __int_as_float((static_cast<int>(e) + 127) << 23);
}

// SHIFT: 0 none; 1 per-row and 2 per-column exponent shift (SdArgs), so that
// each kernel value is K_ij * 2^shift -- used by the log-sum-exp backward to
// sum the normalised weights w K e^-lse directly; 3 multiplies each kernel
// value by the scaled squared distance |x^ - y^|^2 = (tau/2 log2 e) |x - y|^2,
// which gives the bandwidth gradient sum_j K w |x - y|^2 without cancellation;
// 4 does both the per-row shift and the squared-distance factor.
// Resident CTAs per SM asked of the register allocator.  Eight (at most 64
// registers a thread) is worth 1-4 % on the single-channel D <= 3 kernels and
// costs them no spill; the other instantiations keep the default, where the
// same bound would spill.
__host__ __device__ constexpr int sd_min_blocks(int D, int CP, int SHIFT) {
  return (CP == 1 && D <= 3 && SHIFT != 1 && SHIFT != 4) ? 8 : 1;
}

// NT threads per CTA, the same kSdThreads * sd_rows_per_thread rows per CTA:
// NT = 256 halves the rows of each thread and doubles the warps.  A grid of
// one partial wave (too few CTAs to fill every SM with 128-thread CTAs) has
// few warps per SM to hide the latency of the pair loop; measured at
// M = N = 10^4 (730 CTAs of 128 threads): 16 warps per SM, MUFU busy 73% of
// the active cycles.  (Register bound as for NT = 128: 64 a thread.)
template <int D, int CP, bool LSE, int SHIFT, int NT>
__global__ void __launch_bounds__(NT, sd_min_blocks(D, CP, SHIFT) * kSdThreads / NT)
    sd_kernel(const SdArgs a) {
  constexpr int R = sd_rows_per_thread(D, CP) * kSdThreads / NT;
  constexpr int kPer = kTileJ / NT;   // points each thread stages per tile
  // a programmatic dependent (the split combine) may be scheduled as soon as
  // every block of this grid has started; it waits for this grid to complete
  asm volatile("griddepcontrol.launch_dependents;");
  constexpr int RP = R / 2;                     // row pairs per thread
  constexpr int NPOLY = poly_pairs<D, CP, R>();
  constexpr int PK = PackShape<D, CP, SHIFT>::PK;
  static_assert(!(LSE && SHIFT), "shifts apply to the sum kernel");
  constexpr int NW = NT / 32;
  static_assert(R % 2 == 0, "rows are processed in pairs");
  __shared__ __align__(16) float tile[kTileJ * PK];
  __shared__ float red[NW][CP];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t b = blockIdx.z;
  const int split = blockIdx.y;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (NT * R);
  const int64_t jbeg = static_cast<int64_t>(split) * a.plan.cols_per_split;
  const int64_t jend = min(a.N, jbeg + a.plan.cols_per_split);
  const float* __restrict__ yb = a.y + b * a.N * D;
  const float* __restrict__ wb = a.w + b * a.N * a.ldw + a.c0;

  // scaled coordinates of my rows, two rows per 64-bit pair
  uint64_t xs[RP][D];
#pragma unroll
  for (int q = 0; q < RP; ++q) {
    const int64_t i0 = row0 + tid + (2 * q) * NT;
    const int64_t i1 = i0 + NT;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      const float v0 = (i0 < a.M) ? a.x[(b * a.M + i0) * D + k] * a.scale : 0.f;
      const float v1 = (i1 < a.M) ? a.x[(b * a.M + i1) * D + k] * a.scale : 0.f;
      xs[q][k] = pk2(v0, v1);
    }
  }
  uint64_t rho[RP];   // SHIFT == 1: per-row exponent shift of my row pairs
#pragma unroll
  for (int q = 0; q < RP; ++q) {
    if constexpr (SHIFT == 1 || SHIFT == 4) {
      const int64_t i0 = row0 + tid + (2 * q) * NT;
      const int64_t i1 = i0 + NT;
      const float s0 = (i0 < a.M) ? a.shift_scale * a.shift_src[(b * a.M + i0) * a.shift_ld + a.shift_c] : 0.f;
      const float s1 = (i1 < a.M) ? a.shift_scale * a.shift_src[(b * a.M + i1) * a.shift_ld + a.shift_c] : 0.f;
      rho[q] = pk2(s0, s1);
    } else {
      rho[q] = 0ull;
    }
  }
  uint64_t acc[RP][CP];
  float mrun[CP];   // LSE: integer log2 shift of the weights (-inf before any positive weight)
#pragma unroll
  for (int c = 0; c < CP; ++c) {
    mrun[c] = -INFINITY;
#pragma unroll
    for (int q = 0; q < RP; ++q) acc[q][c] = 0ull;
  }

  for (int64_t j0 = jbeg; j0 < jend; j0 += kTileJ) {
    // ---- stage one tile: negated scaled y and the (shifted) weights
    float sy[kPer][D], sv[kPer][CP], sk[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int64_t j = j0 + tid + q * NT;
      const bool ok = j < jend;
      if constexpr (SHIFT == 2)
        sk[q] = ok ? a.shift_scale * a.shift_src[(b * a.N + j) * a.shift_ld + a.shift_c] : 0.f;
      else
        sk[q] = 0.f;
#pragma unroll
      for (int k = 0; k < D; ++k) sy[q][k] = ok ? -(yb[j * D + k] * a.scale) : 0.f;
#pragma unroll
      for (int c = 0; c < CP; ++c) sv[q][c] = (ok && c < a.cw) ? wb[j * a.ldw + c] : 0.f;
    }
    if constexpr (LSE) {
      // running power-of-two bound of the weights: w * 2^-m stays <= 1, so every
      // term w K 2^-m <= 1 (K <= 1); accumulators follow the bound exactly
#pragma unroll
      for (int c = 0; c < CP; ++c) {
        float m = sv[0][c];
#pragma unroll
        for (int q = 1; q < kPer; ++q) m = fmaxf(m, sv[q][c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[warp][c] = m;
      }
      __syncthreads();
#pragma unroll
      for (int c = 0; c < CP; ++c) {
        float mt = red[0][c];
#pragma unroll
        for (int v = 1; v < NW; ++v) mt = fmaxf(mt, red[v][c]);
        // smallest integer e with max w < 2^e (from the exponent bits)
        const float et = (mt > 0.f) ? static_cast<float>(((__float_as_int(mt) >> 23) & 0xff) - 126)
                                    : -INFINITY;
        const float mnew = fmaxf(mrun[c], et);
        if (mnew > mrun[c]) {
          const float fac = pow2i(mrun[c] - mnew);
#pragma unroll
          for (int q = 0; q < RP; ++q) {
            acc[q][c] = mul2(acc[q][c], pk2(fac, fac));
          }
          mrun[c] = mnew;
        }
        const float sc = (mnew == -INFINITY) ? 1.f : pow2i(-mnew);
#pragma unroll
        for (int q = 0; q < kPer; ++q) sv[q][c] *= sc;
      }
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      float* p = tile + (tid + q * NT) * PK;
#pragma unroll
      for (int k = 0; k < D; ++k) {
        p[2 * k] = sy[q][k];
        p[2 * k + 1] = sy[q][k];
      }
#pragma unroll
      for (int c = 0; c < CP; ++c) {
        p[2 * (D + c)] = sv[q][c];
        p[2 * (D + c) + 1] = sv[q][c];
      }
      if constexpr (SHIFT == 2) {
        p[2 * (D + CP)] = sk[q];
        p[2 * (D + CP) + 1] = sk[q];
      }
#pragma unroll
      for (int k = 2 * PackShape<D, CP, SHIFT>::NPAIR; k < PK; ++k) p[k] = 0.f;
    }
    __syncthreads();

    // ---- all pairs (my R rows) x (256 staged points)
    uint64_t tacc[RP][CP];
#pragma unroll
    for (int q = 0; q < RP; ++q)
#pragma unroll
      for (int c = 0; c < CP; ++c) tacc[q][c] = 0ull;

    const ulonglong2* t2 = reinterpret_cast<const ulonglong2*>(tile);
    // staged points past jend carry zero weight: a short last tile stops at
    // its own width (rounded up to the unroll pair) instead of the full tile
    const int nj = static_cast<int>(min(static_cast<int64_t>(kTileJ), jend - j0) + 1) & ~1;
#pragma unroll 2
    for (int jj = 0; jj < nj; ++jj) {
      uint64_t pk[PK / 2];
#pragma unroll
      for (int v = 0; v < PK / 4; ++v) {
        const ulonglong2 u = t2[jj * (PK / 4) + v];
        pk[2 * v] = u.x;
        pk[2 * v + 1] = u.y;
      }
#pragma unroll
      for (int q = 0; q < RP; ++q) {
        // d = |x^ - y^|^2 for two rows at once
        uint64_t e = add2(xs[q][0], pk[0]);
        uint64_t d = mul2(e, e);
#pragma unroll
        for (int k = 1; k < D; ++k) {
          e = add2(xs[q][k], pk[k]);
          d = fma2(e, e, d);
        }
        uint64_t kv;
        if constexpr (SHIFT == 3) {
          float d0, d1;
          upk2(d, d0, d1);
          kv = mul2(pk2(ex2(-d0), ex2(-d1)), d);
        } else if constexpr (SHIFT == 4) {
          float t0, t1;
          upk2(sub2(rho[q], d), t0, t1);
          kv = mul2(pk2(ex2(t0), ex2(t1)), d);
        } else if constexpr (SHIFT != 0) {
          // exponent = shift - d (per row, or per column from the staged pair)
          float t0, t1;
          upk2(sub2(SHIFT == 1 ? rho[q] : pk[D + CP], d), t0, t1);
          kv = pk2(ex2(t0), ex2(t1));
        } else {
          float d0, d1;
          upk2(d, d0, d1);
          if (q >= RP - NPOLY) {
            kv = exp2_poly2<5, true>(pk2(fminf(d0, 125.f), fminf(d1, 125.f)));
          } else {
            kv = pk2(ex2(-d0), ex2(-d1));
          }
        }
#pragma unroll
        for (int c = 0; c < CP; ++c) tacc[q][c] = fma2(kv, pk[D + c], tacc[q][c]);
      }
    }
#pragma unroll
    for (int q = 0; q < RP; ++q)
#pragma unroll
      for (int c = 0; c < CP; ++c) acc[q][c] = add2(acc[q][c], tacc[q][c]);
    __syncthreads();
  }

  // ---- write this split's result (final sum, or shift + scaled sum)
#pragma unroll
  for (int q = 0; q < RP; ++q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t i = row0 + tid + (2 * q + h) * NT;
      if (i >= a.M) continue;
      const int64_t base = split * a.split_stride + (b * a.M + i) * a.ldo + a.c0;
#pragma unroll
      for (int c = 0; c < CP; ++c) {
        if (c >= a.cw) break;
        float lo, hi;
        upk2(acc[q][c], lo, hi);
        const float v = h ? hi : lo;
        if constexpr (LSE) {
          a.out[base + c] = mrun[c];
          a.out_l[base + c] = v;
        } else {
          a.out[base + c] = v;
        }
      }
    }
  }
}

template <int D, int CP, bool LSE>
cudaError_t launch_t(const SdArgs& a, cudaStream_t s) {
  constexpr int R = sd_rows_per_thread(D, CP);
  const int64_t tiles = (a.M + kSdThreads * R - 1) / (kSdThreads * R);
  dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(a.plan.splits),
            static_cast<unsigned>(a.B));
  constexpr bool kWide = !LSE && sd_min_blocks(D, CP, 0) == 8;   // NT = 256 instantiated
  if constexpr (LSE) {
    sd_kernel<D, CP, true, 0, kSdThreads><<<grid, kSdThreads, 0, s>>>(a);
  } else {
    if constexpr (kWide) {
      if (a.plan.threads == 2 * kSdThreads && (a.shift_mode == 0 || a.shift_mode == 2 ||
                                               a.shift_mode == 3)) {
        switch (a.shift_mode) {
          case 2: sd_kernel<D, CP, false, 2, 2 * kSdThreads><<<grid, 2 * kSdThreads, 0, s>>>(a); break;
          case 3: sd_kernel<D, CP, false, 3, 2 * kSdThreads><<<grid, 2 * kSdThreads, 0, s>>>(a); break;
          default: sd_kernel<D, CP, false, 0, 2 * kSdThreads><<<grid, 2 * kSdThreads, 0, s>>>(a); break;
        }
        return cudaGetLastError();
      }
    }
    switch (a.shift_mode) {
      case 1: sd_kernel<D, CP, false, 1, kSdThreads><<<grid, kSdThreads, 0, s>>>(a); break;
      case 2: sd_kernel<D, CP, false, 2, kSdThreads><<<grid, kSdThreads, 0, s>>>(a); break;
      case 3: sd_kernel<D, CP, false, 3, kSdThreads><<<grid, kSdThreads, 0, s>>>(a); break;
      case 4: sd_kernel<D, CP, false, 4, kSdThreads><<<grid, kSdThreads, 0, s>>>(a); break;
      default: sd_kernel<D, CP, false, 0, kSdThreads><<<grid, kSdThreads, 0, s>>>(a); break;
    }
  }
  return cudaGetLastError();
}

template <int D, bool LSE>
cudaError_t launch_cp(const SdArgs& a, cudaStream_t s) {
  switch (sd_chunk_pad(a.cw)) {
    case 1: return launch_t<D, 1, LSE>(a, s);
    case 2: return launch_t<D, 2, LSE>(a, s);
    case 4: return launch_t<D, 4, LSE>(a, s);
    default: return launch_t<D, 8, LSE>(a, s);
  }
}

template <bool LSE>
cudaError_t launch_d(const SdArgs& a, cudaStream_t s) {
  switch (a.D) {
    case 1: return launch_cp<1, LSE>(a, s);
    case 2: return launch_cp<2, LSE>(a, s);
    case 3: return launch_cp<3, LSE>(a, s);
    case 4: return launch_cp<4, LSE>(a, s);
    case 5: return launch_cp<5, LSE>(a, s);
    case 6: return launch_cp<6, LSE>(a, s);
    case 7: return launch_cp<7, LSE>(a, s);
    case 8: return launch_cp<8, LSE>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

// ------------------------------------------------------------------ combine
// out[e] = sum_k part[k * total + e] in the fixed order of combine.cuh.  A block
// takes 32 consecutive elements with one warp per lane of that order: warp l
// sums splits l, l + kCombineLanes, ... in turn (reading 128 contiguous bytes
// of a split at a time), then the lane sums are added in lane order.
// Launched as a programmatic dependent of the pass that wrote the partials:
// its blocks may start while that kernel drains, and griddepcontrol.wait holds
// them until it has completed and its stores are visible.
__global__ void __launch_bounds__(32 * kCombineLanes)
    combine_sum_kernel(const float* __restrict__ part, int splits, int64_t total,
                       float* __restrict__ out) {
  __shared__ float red[kCombineLanes][33];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int64_t e0 = blockIdx.x * 32ll; e0 < total; e0 += gridDim.x * 32ll) {
    const int64_t e = e0 + tx;
    const float s = (e < total) ? split_lane_sum(part + e, ty, splits, total) : 0.f;
    red[ty][tx] = s;
    __syncthreads();
    if (ty == 0 && e < total) {
      float t = red[0][tx];
#pragma unroll
      for (int v = 1; v < kCombineLanes; ++v) t += red[v][tx];
      out[e] = t;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ LSE finalisation
// One warp per (batch, row).  Lane k holds split k's (shift, scaled sum); the
// merge m = max m_k, l = sum_k l_k 2^(m_k - m) runs as a fixed xor-tree.
// Rows whose merged l is below 2^-64 (terms may have been flushed to zero)
// are recomputed from scratch with their own exact maximum.
__device__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void lse_finalize_kernel(const LseFinalizeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t rows = a.B * a.M;
  const float kTiny = 5.421010862427522e-20f;   // 2^-64
  for (int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       row < rows; row += warps_total) {
    const int64_t b = row / a.M;
    const int64_t i = row % a.M;
    for (int c = 0; c < a.C; ++c) {
      const int64_t e = row * a.C + c;
      float mk = -INFINITY, lk = 0.f;
      if (lane < a.splits) {
        mk = a.part_m[lane * a.split_stride + e];
        lk = a.part_l[lane * a.split_stride + e];
      }
      const float m = warp_max(mk);
      const float contrib = (mk == -INFINITY) ? 0.f : lk * ex2(mk - m);
      const float l = warp_sum(contrib);
      float res;
      if (!(l < kTiny) || a.D > kSdMaxD || a.no_fallback) {
        // (the tensor-core path for D > 8 shifts by the running maximum, so
        // its l is at least 1 whenever any term is nonzero)
        res = (m + log2f(l)) * kLn2;
      } else {
        // exact per-row recompute: pass 1 maximum, pass 2 shifted sum
        const float* xi = a.x + (b * a.M + i) * a.D;
        float xs[kSdMaxD];
        for (int k = 0; k < a.D; ++k) xs[k] = xi[k] * a.scale;
        float mx = -INFINITY;
        for (int64_t j = lane; j < a.N; j += 32) {
          const float* yj = a.y + (b * a.N + j) * a.D;
          float t = lg2(a.w[(b * a.N + j) * a.C + c]);
          for (int k = 0; k < a.D; ++k) {
            const float d = xs[k] - yj[k] * a.scale;
            t = fmaf(-d, d, t);
          }
          mx = fmaxf(mx, t);
        }
        mx = warp_max(mx);
        float outer = 0.f;
        if (mx != -INFINITY) {
          float inner = 0.f;
          int n_in = 0;
          for (int64_t j = lane; j < a.N; j += 32) {
            const float* yj = a.y + (b * a.N + j) * a.D;
            float t = lg2(a.w[(b * a.N + j) * a.C + c]);
            for (int k = 0; k < a.D; ++k) {
              const float d = xs[k] - yj[k] * a.scale;
              t = fmaf(-d, d, t);
            }
            inner += ex2(t - mx);
            if (++n_in == 64) {
              outer += inner;
              inner = 0.f;
              n_in = 0;
            }
          }
          outer += inner;
        }
        const float ls = warp_sum(outer);
        res = (mx == -INFINITY) ? -INFINITY : (mx + log2f(ls)) * kLn2;
      }
      if (lane == 0) a.out[e] = res;
    }
  }
}

__global__ void fill_kernel(float* __restrict__ out, int64_t n, float value) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[e] = value;
}

template <int DEG>
__global__ void exp2_poly_eval_kernel(const float* __restrict__ x, float* __restrict__ out,
                                      int64_t n) {
  const int64_t pairs = (n + 1) / 2;
  for (int64_t p = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; p < pairs;
       p += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = 2 * p;
    const float a = fmaxf(x[i], -125.f);
    const float b = (i + 1 < n) ? fmaxf(x[i + 1], -125.f) : 0.f;
    float ra, rb;
    upk2(exp2_poly2<DEG, false>(pk2(a, b)), ra, rb);
    out[i] = ra;
    if (i + 1 < n) out[i + 1] = rb;
  }
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148 * 32) b = 148 * 32;
  return static_cast<int>(b);
}

}  // namespace

SdPlan sd_plan(int64_t B, int64_t M, int64_t N, int D, int64_t C, int sm_count, int max_splits,
               bool wide_ok) {
  SdPlan p{};
  p.threads = kSdThreads;
  const int cw = static_cast<int>(C < kSdMaxChunk ? C : kSdMaxChunk);
  const int R = sd_rows_per_thread(D, sd_chunk_pad(cw));
  p.rows_per_cta = kSdThreads * R;
  const int64_t U = B * ((M + p.rows_per_cta - 1) / p.rows_per_cta);
  // candidates: at least 128 columns a split, at most max_splits, and split
  // partials of at most 2^25 floats
  int64_t smax = N / 128;
  if (smax > max_splits) smax = max_splits;
  const int64_t part_cap = (int64_t(1) << 25) / (B * M * C > 0 ? B * M * C : 1);
  if (smax > part_cap) smax = part_cap;
  if (smax < 1) smax = 1;
  // Cost of S splits, fit to B200 timings of the D = 3 kernel from 10^4 to
  // 10^6 points: the U x S CTAs run in W = U S / (SMs x 8 resident) waves; a
  // partial last wave costs at least half a wave (with fewer than about four
  // CTAs on an SM its MUFU pipe idles); every CTA pays about 16 columns of
  // fixed work; a tenth of one CTA's columns goes to the ragged end.
  int best = 1;
  double best_cost = 1e300;
  const double wave = static_cast<double>(sm_count) * 8.0;
  for (int64_t S = 1; S <= smax; ++S) {
    const double W = static_cast<double>(U * S) / wave;
    const double full = std::floor(W), frac = W - full;
    const double phases = (full == 0.0) ? std::fmax(W, 0.5)
                                        : full + (frac > 1e-9 ? std::fmax(frac, 0.5) : 0.0);
    const double cols = static_cast<double>((N + S - 1) / S);
    const double cost = phases * (cols + 16.0) + 0.1 * cols;
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = static_cast<int>(S);
    }
  }
  // One partial wave of 128-thread CTAs leaves too few warps per SM to keep
  // MUFU busy: 256-thread CTAs (4 resident per SM at 64 registers), and the
  // split count that fills one wave of them.
  if (wide_ok && static_cast<double>(U * best) < wave) {
    int64_t s2 = static_cast<int64_t>(sm_count) * 4 / U;
    if (s2 > smax) s2 = smax;
    if (s2 >= 1) {
      best = static_cast<int>(s2);
      p.threads = 2 * kSdThreads;
    }
  }
  p.cols_per_split = (N + best - 1) / best;
  // keep every split non-empty
  if (p.cols_per_split < 1) p.cols_per_split = 1;
  p.splits = static_cast<int>((N + p.cols_per_split - 1) / p.cols_per_split);
  if (p.splits < 1) p.splits = 1;
  return p;
}

cudaError_t launch_small_d_sum(const SdArgs& a, cudaStream_t s) { return launch_d<false>(a, s); }
cudaError_t launch_small_d_lse(const SdArgs& a, cudaStream_t s) { return launch_d<true>(a, s); }

cudaError_t launch_combine_sum(const float* part, int splits, int64_t total, float* out,
                               cudaStream_t s) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid_for(total, 32)));
  cfg.blockDim = dim3(32 * kCombineLanes);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_sum_kernel, part, splits, total, out);
}

cudaError_t launch_lse_finalize(const LseFinalizeArgs& a, cudaStream_t s) {
  const int64_t rows = a.B * a.M;
  int64_t blocks = (rows + 7) / 8;   // 8 warps per block
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) blocks = 1;
  lse_finalize_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fill(float* out, int64_t n, float value, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  fill_kernel<<<grid_for(n, 256), 256, 0, s>>>(out, n, value);
  return cudaGetLastError();
}

}  // namespace gs

extern "C" gs_status gs_test_exp2_poly(const float* x, float* out, int64_t n, int degree,
                                       gs_stream_t stream) {
  if (n < 0 || (degree != 3 && degree != 5)) return GS_ERR_INVALID_ARG;
  if (n == 0) return GS_OK;
  if (!x || !out) return GS_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int blocks = gs::grid_for((n + 1) / 2, 256);
  if (degree == 3)
    gs::exp2_poly_eval_kernel<3><<<blocks, 256, 0, s>>>(x, out, n);
  else
    gs::exp2_poly_eval_kernel<5><<<blocks, 256, 0, s>>>(x, out, n);
  return cudaGetLastError() == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}
