// internal.h -- host-side interface between the C ABI front end (api.cpp)
// and the kernel translation units.  Not part of the public ABI.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/gauss.h"

namespace gs {

constexpr int kSmCountDefault = 148;   // B200

// ------------------------------------------------------------- small-D path
// Rows per CTA of the CUDA-core kernel and its widest channel chunk.
constexpr int kSdThreads = 128;
constexpr int kSdMaxChunk = 8;
constexpr int kSdMaxD = 8;

// Rows each thread of the small-D kernel keeps in registers, by feature
// width D and padded channel chunk CP (register budget ~ R * (D + 2 CP)).
__host__ __device__ constexpr int sd_rows_per_thread(int D, int CP) {
  return (D + 2 * CP <= 8) ? 8 : ((D + 2 * CP <= 20) ? 4 : 2);
}
// Channel chunk width the kernel is instantiated for (1, 2, 4 or 8).
__host__ __device__ constexpr int sd_chunk_pad(int c) {
  return c <= 1 ? 1 : (c <= 2 ? 2 : (c <= 4 ? 4 : 8));
}

struct SdPlan {
  int rows_per_cta;    // kSdThreads * rows per thread
  int splits;          // j-splits (partials combined afterwards when > 1)
  int64_t cols_per_split;
  int threads;         // threads per CTA: kSdThreads, or twice that (same rows per CTA)
};

// Choose rows per CTA and the j-split for the small-D kernel.
// max_splits: 32 for the log-sum-exp (its finalize merges the splits in one warp).
// wide_ok: the 256-thread sum kernel may run this pass (one channel, D <= 3,
// exponent modes 0, 2 and 3).
SdPlan sd_plan(int64_t B, int64_t M, int64_t N, int D, int64_t C, int sm_count, int max_splits,
               bool wide_ok = false);

struct SdArgs {
  const float* x;
  const float* y;
  const float* w;      // [B, N, ldw]
  int ldw;             // channels in w rows
  int c0;              // first channel of this chunk
  int cw;              // channels in this chunk (<= kSdMaxChunk)
  float* out;          // sum: [S?][B][M][ldo]; lse: shift part
  float* out_l;        // lse only: scaled sums, same layout as out
  int ldo;
  int64_t split_stride;  // elements between split slices (0 if one split)
  int64_t B, M, N;
  int D;
  float scale;         // sqrt(tau / 2 * log2 e)
  SdPlan plan;
  // optional exponent shift (log2 units), sum kernel only: every kernel value
  // becomes K_ij * 2^shift with shift = shift_scale * shift_src[(b * n + p) * shift_ld + shift_c],
  // p the row i (shift_mode 1, n = M) or the column j (shift_mode 2, n = N)
  int shift_mode;      // 0 none, 1 per row, 2 per column, 3 kernel x scaled |x - y|^2, 4 = 1 and 3
  const float* shift_src;
  int64_t shift_ld;
  int shift_c;
  float shift_scale;
};

cudaError_t launch_small_d_sum(const SdArgs& a, cudaStream_t s);
cudaError_t launch_small_d_lse(const SdArgs& a, cudaStream_t s);

// Combine `splits` partial sums [S][total] into out[total] in fixed order.
cudaError_t launch_combine_sum(const float* part, int splits, int64_t total, float* out,
                               cudaStream_t s);

// Combine (shift, scaled sum) partials into the log-sum-exp and recompute
// exactly any row whose scaled sum came out too small to trust.
struct LseFinalizeArgs {
  const float* part_m;
  const float* part_l;
  int splits;
  int64_t split_stride;
  float* out;          // [B, M, C]
  const float* x;
  const float* y;
  const float* w;
  int64_t B, M, N;
  int D, C;
  float scale;
  // the tensor-core path shifts by the running maximum (l >= 1): no recompute,
  // and x, y, w may not be fp32
  int no_fallback;
};
cudaError_t launch_lse_finalize(const LseFinalizeArgs& a, cudaStream_t s);

// Value matrix of a pass on the CUDA-core path, float32 [B, N, CV] (values.cuh);
// src rows are src_ld floats apart (src_ld >= C; a channel slice of a wider array).
cudaError_t launch_pack_values_f32(const void* src, int64_t src_ld, const void* cols,
                                   const void* rows, float* v, int64_t B, int64_t N, int64_t Mrows,
                                   int D, int C, int mode, cudaStream_t s);

// Log-sum-exp backward epilogues for channel c of C (grad.cu): o_x [B, M, 1 + D]
// holds [sum_j p, sum_j p (y - z)] and o_y [B, N, 1 + D] holds
// [sum_i g p / w, sum_i g p (x - z) / w]; with `accumulate` the results add to
// the outputs of the previous channels.
// ot [B, M] holds sum_j p |x^ - y^|^2; when it is NULL (and tau_rows is not),
// o has 2 + D channels per row, the last sum_j p |y - z|^2 (values mode 2)
cudaError_t launch_lse_x_tau_epilogue(const float* x, const float* g, const float* o,
                                      const float* ot, float* grad_x, float* tau_rows, int64_t B,
                                      int64_t M, int D, int C, int c, float tau, float inv_cfac,
                                      bool accumulate, cudaStream_t s, int ocv);
cudaError_t launch_lse_grad_y_epilogue(const float* y, const float* w, const float* o,
                                       float* grad_y, float* grad_w, int64_t B, int64_t N, int D,
                                       int C, int c, float tau, bool accumulate, cudaStream_t s);

// Gradient epilogues (grad.cu).  grad_x and tau_rows may each be NULL; so may
// grad_y and grad_w.
cudaError_t launch_grad_x_epilogue(const void* x, gs_dtype dt, const float* g, const float* o,
                                   float* grad_x, float* tau_rows, int64_t B, int64_t M, int D,
                                   int C, int CV, float tau, cudaStream_t s);
// Forward + backward (C = 1): out and grad_x from the x pass's `splits` partials.
cudaError_t launch_fwd_bwd_epilogue(const void* x, gs_dtype dt, const float* g, const float* part,
                                    int splits, int64_t stride, float* out, float* grad_x,
                                    int64_t B, int64_t M, int D, int CV, float tau,
                                    cudaStream_t s);
cudaError_t launch_grad_y_epilogue(const void* y, const void* w, gs_dtype dt, const float* o,
                                   float* grad_y, float* grad_w, int64_t B, int64_t N, int D,
                                   int C, int CV, float tau, cudaStream_t s);
// tau_rows[r] (+)= factor * sum_{c in [c0, c0 + nc)} g[r, c] * o[r, c - c0]
cudaError_t launch_weighted_rows(const float* g, const float* o, float* tau_rows, int64_t rows,
                                 int C, int c0, int nc, float factor, bool accumulate,
                                 cudaStream_t s);
// Diffusion operator elementwise steps (grad.cu): op 0 o1 = 1; op 1 o1 = a^-alpha;
// op 2 (a = q, b = K q^-alpha) o1 = d = q^-alpha b, o2 = s = q^-alpha d^-1/2;
// op 3 o1[e] = a[e / C] * b[e].
cudaError_t launch_diffusion_elementwise(int op, const float* a, const float* b, float* o1,
                                         float* o2, int64_t n, int C, float alpha, cudaStream_t s);
// dst[0 .. n) = the fp16 / bf16 values of src as float32 (exact).
cudaError_t launch_widen_to_f32(const void* src, gs_dtype dt, float* dst, int64_t n,
                                cudaStream_t s);
// out[0] = sum of v[0 .. n) in a fixed order (double accumulation).
cudaError_t launch_sum_rows(const float* v, int64_t n, float* out, cudaStream_t s);

// ------------------------------------------------------------- tensor-core path
constexpr int kTcMaxD = 128;
constexpr int kTcMaxChunk = 128;   // channels per tensor-core pass

struct TcPlan {
  int KP;              // padded feature width of the packed operands (64, 128 or 192)
  int splits;
  int64_t cols_per_split;   // multiple of 128
};
TcPlan tc_plan(int64_t B, int64_t M, int64_t N, int64_t D, int sm_count);
// Channels per tensor-core pass for a packed width KP, and the padded value
// chunk (16, 32, 48, 64, 96 or 128) a pass of cw channels is compiled for.
int tc_max_chunk(int KP);
int tc_chunk_pad(int cw);

// Which values the tensor-core pass multiplies by the kernel (values.cuh modes).
enum TcValues { kValuesW = 0, kValuesBwd = 1, kValuesBwdTau = 2 };

struct TcArgs {
  const void* x;       // rows side [B, M, D]
  const void* y;       // column side [B, N, D]
  const void* w;       // values source [B, N, C] (dtype dt, or float32 if w_is_f32)
  bool w_is_f32;
  TcValues values;     // value mode (values.cuh), columns centred at x[b, 0]
  int C;               // channels of w
  int CV;              // channels of the value matrix
  float* out;          // [S?][B][M][CV]
  int64_t split_stride;
  int64_t B, M, N;
  int D;
  gs_dtype dt;
  float tau;
  TcPlan plan;
  // workspace pieces
  void* xpack;         // [B, M, KP]
  float* rnorm;        // [B, M]
  void* ypack;         // [B, N, KP]
  void* vt;            // [B, CP, Nst] f16
  // forward + backward sweep (gw_part != nullptr): dL/dw column sums as well
  const float* g;      // [B, M, g_ld] upstream gradient, channel 0
  int64_t g_ld;
  uint32_t* gpack;     // [B, M] packed parts of g
  float* gscale;       // [B] their scales
  float* gtmax;        // [B, ceil(M / 128)] largest |g| of each 128-row tile
  float* gw_part;      // [ceil(M / 128), B, N]
};
cudaError_t launch_tc_sum(const TcArgs& a, cudaStream_t s);

// 3-D tiled TMA descriptor: dims {d0, d1, d2} (d0 innermost, in elements),
// strides of dims 1 and 2 in bytes, box {box0, box1, 1}, 128-byte swizzle or none.
bool make_tmap_3d(CUtensorMap* m, CUtensorMapDataType dt, void* base, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0,
                  uint32_t box1, bool swizzle128 = true);

// ------------------------------------------------------------- fp32 tensor-core path
// fp32 inputs with kSdMaxD < D <= kTcMaxD: MMAs on split fp16 parts (tc_f32_sm100.cu).
struct F32Plan {
  bool split;          // fp32 inputs: fp16 rows [hi | lo]; fp16 / bf16: the input values, unsplit
  int Kp;              // 16-bit elements per half of a packed row: D rounded up to 16
  int atoms;           // 128-byte atoms per packed row (2 Kp or Kp 16-bit values)
  int max_chunk;       // channels per pass (64)
  int splits;
  int64_t cols_per_split;   // multiple of 128
};
F32Plan f32_plan(int64_t B, int64_t M, int64_t N, int64_t D, int sm_count, bool split = true);
int f32_chunk_pad(int cw);            // 16, 32 or 64
int f32_tile_cols(int KA, int mode);  // columns per tile of an instantiation

struct F32Args {
  const void* x;       // rows side [B, M, D], dtype dt
  const void* y;       // column side [B, N, D], dtype dt
  const void* w;       // values source [B, N, C], dtype dt
  gs_dtype dt;         // fp32 (split operands); fp16 / bf16 (log-sum-exp only)
  TcValues values;     // value mode (values.cuh; its own centre x[b, 0])
  int C, CV;
  int64_t src_ld;      // row stride of the value source (C when it is a whole array)
  // optional exponent shift (log2 units) added to the row norms (shift_mode 1)
  // or to the column norms (2): shift_scale * shift_src[(b * n + p) * shift_ld + shift_c]
  int shift_mode;
  const float* shift_src;
  int64_t shift_ld;
  int shift_c;
  float shift_scale;
  float* out;          // [S?][B][M][CV]; log-sum-exp: the shifts m (log2 units)
  float* out_l;        // log-sum-exp only: the scaled sums l, same layout
  bool lse;            // log-sum-exp of w K per channel (w > 0) instead of the sum
  int64_t split_stride;
  int64_t B, M, N;
  int D;
  float tau;
  F32Plan plan;
  // workspace pieces
  float* zc;           // [B, D] centre of each batch (the mean of its column points)
  float* xpack;        // [B, M, 2 Kp] (or [B, M, Kp] unsplit)
  float* rnorm;        // [B, M]
  float* ypack;        // [B, N, 2 Kp]
  float* qw;           // [B, 4, Nq] lane by lane, Nq = N rounded up to 128: lane 0 -c |y'|^2 (-inf past N)
                       // and up to 3 value channels
  float* vt;           // [2 B, CP, Nst] (hi, lo), Nst = N rounded up to 4
};
cudaError_t launch_tc_f32_sum(const F32Args& a, cudaStream_t s);
cudaError_t read_and_clear_device_error_f32(int* value);
cudaError_t set_test_waits_f32(uint64_t limit_ns, int stall);

// out[0 .. n) = value
cudaError_t launch_fill(float* out, int64_t n, float value, cudaStream_t s);

// ------------------------------------------------------------- k-nearest reduction
constexpr int kKnnMaxK = 32;
struct KnnPlan {
  int splits;
  int64_t cols_per_split;
};
KnnPlan knn_plan(int64_t B, int64_t M, int64_t N, int64_t D, int K, int sm_count);
struct KnnArgs {
  const float* x;
  const float* y;
  float* part_d;       // [splits][B][M][K] per-split sorted lists
  int* part_i;
  float* out_d;        // [B, M, K]
  int64_t* out_i;
  int64_t B, M, N;
  int D, K;
  int splits;
  int64_t cols_per_split;
  int64_t split_stride;   // B * M * K
};
cudaError_t launch_knn(const KnnArgs& a, cudaStream_t s);

// Device error word (set by kernels whose waits time out).
cudaError_t read_and_clear_device_error(int* value);
// Test hook: the wait limit and stall mode of the tensor-core kernels.
cudaError_t set_test_waits(uint64_t limit_ns, int stall);

}  // namespace gs
