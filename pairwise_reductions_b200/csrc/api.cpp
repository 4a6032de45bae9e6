// api.cpp -- the C ABI front end: argument validation, workspace sizing and
// dispatch to the CUDA-core (fp32, small D) or tensor-core (fp16/bf16) path.
// Nothing here synchronises or allocates; all work goes onto the caller's
// stream.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "gauss_testing.h"
#include "internal.h"
#include "values.cuh"

using namespace gs;

namespace {

constexpr size_t kAlign = 1024;
constexpr size_t kBad = static_cast<size_t>(-1);

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return kSmCountDefault;
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return kSmCountDefault;
  }
  return n;
}

size_t elem_size(gs_dtype dt) { return dt == GS_F32 ? 4 : 2; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape and type checks shared by every entry point (no pointers).
gs_status check_dims(gs_op op, int64_t B, int64_t M, int64_t N, int64_t D, int64_t C, gs_dtype dt) {
  if (B < 0 || M < 0 || N < 0 || D < 1 || C < 1) return GS_ERR_INVALID_ARG;
  if (dt != GS_F32 && dt != GS_F16 && dt != GS_BF16) return GS_ERR_INVALID_ARG;
  // index arithmetic stays in int64, grid.z holds B, TMA coordinates are int32
  const int64_t lim = int64_t(1) << 31;
  if (B >= 65536 || M >= lim || N >= lim || C >= lim || D >= lim) return GS_ERR_UNSUPPORTED;
  const double big = 9.0e18;
  if (double(B) * double(M > N ? M : N) * double((D > C ? D : C) + 1) * double(D + 2) > big)
    return GS_ERR_UNSUPPORTED;
  // every dtype: the CUDA-core path up to D = 8 (fp32), the tensor-core paths up to 128
  if (D > kTcMaxD) return GS_ERR_UNSUPPORTED;
  return GS_OK;
}

gs_status check_tau(float tau) {
  return (std::isfinite(tau) && tau > 0.f) ? GS_OK : GS_ERR_INVALID_ARG;
}

gs_status check_ptr(const void* p, int64_t n_elems) {
  if (n_elems == 0) return GS_OK;
  if (p == nullptr) return GS_ERR_INVALID_ARG;
  if (!aligned16(p)) return GS_ERR_ALIGNMENT;
  return GS_OK;
}

#define GS_TRY(expr)                    \
  do {                                  \
    gs_status _st = (expr);             \
    if (_st != GS_OK) return _st;       \
  } while (0)

#define GS_CUDA(expr)                   \
  do {                                  \
    cudaError_t _e = (expr);            \
    if (_e != cudaSuccess) return GS_ERR_CUDA; \
  } while (0)

float coord_scale(float tau) {
  return static_cast<float>(std::sqrt(0.5 * static_cast<double>(tau) * 1.4426950408889634074));
}

// ------------------------------------------------------------------ one Gauss-sum pass
// out[B, rows, CV] = sum over cols of K(rows, cols) * values, where values are
// w (CV = C) or the gradient values [w, w (x) col points] (CV = C (1 + D)).
struct Pass {
  const void* rows_pts;
  const void* cols_pts;
  const void* w;       // value source [B, N, C] (values.cuh)
  bool w_is_f32;
  int vmode;           // values.cuh mode: 0 = w, 1 = [w, w (col - z)], 2 = + w |col - z|^2
  int64_t B, R, N;     // rows, columns
  int D, C, CV;
  gs_dtype dt;
  float tau;
  int64_t src_ld;      // row stride of the value source (0 = C)
  // exponent shift (CUDA-core path only, see SdArgs)
  int shift_mode;
  const float* shift_src;
  int64_t shift_ld;
  int shift_c;
  float shift_scale;
};

// Which kernel family runs a pass: the CUDA-core small-D kernel (fp32, D <= 8),
// the fp16/bf16 tensor-core kernel, or the split-tf32 tensor-core kernel
// (fp32, D > 8).
enum PassPath { kPathSmallD = 0, kPathTcHalf = 1, kPathTcF32 = 2 };

PassPath pass_path(gs_dtype dt, int D) {
  if (dt != GS_F32) return kPathTcHalf;
  return D <= kSdMaxD ? kPathSmallD : kPathTcF32;
}

struct PassLayout {
  bool tc;
  PassPath path;
  SdPlan sd;
  TcPlan tcp;
  F32Plan f32;
  size_t off_part, off_vals, off_xpack, off_rnorm, off_ypack, off_vt, off_qw, off_zc;
  size_t total;
};

PassLayout pass_layout(const Pass& p, int sm) {
  PassLayout L{};
  size_t off = 0;
  L.path = pass_path(p.dt, p.D);
  L.tc = L.path != kPathSmallD;
  if (L.path == kPathTcF32) {
    L.f32 = f32_plan(p.B, p.R, p.N, p.D, sm);
    const size_t rowb = size_t(2) * L.f32.Kp * 4;
    const size_t CPmax = static_cast<size_t>(
        f32_chunk_pad(p.CV < L.f32.max_chunk ? p.CV : L.f32.max_chunk));
    const size_t Nst = (p.N + 3) / 4 * 4;
    const size_t Nq = (p.N + 127) / 128 * 128;
    L.off_zc = off;   // column centres [B, D], one max word per batch, 64 per value chunk
    off = align_up(off + size_t(p.B) * (p.D + 1 + 64) * 4);
    L.off_xpack = off;
    off = align_up(off + size_t(p.B) * p.R * rowb);
    L.off_rnorm = off;
    off = align_up(off + size_t(p.B) * p.R * 4);
    L.off_ypack = off;
    off = align_up(off + size_t(p.B) * p.N * rowb);
    L.off_qw = off;
    off = align_up(off + size_t(p.B) * Nq * 16);
    L.off_vt = off;
    off = align_up(off + size_t(2) * p.B * CPmax * Nst * 4);
    if (L.f32.splits > 1) {
      L.off_part = off;
      off = align_up(off + size_t(L.f32.splits) * p.B * p.R * p.CV * 4);
    }
  } else if (!L.tc) {
    L.sd = sd_plan(p.B, p.R, p.N, p.D, p.CV, sm, 256,
                   p.CV == 1 && p.D <= 3 &&
                       (p.shift_mode == 0 || p.shift_mode == 2 || p.shift_mode == 3));
    if (p.vmode != 0) {
      L.off_vals = off;
      off = align_up(off + size_t(p.B) * p.N * p.CV * 4);
    }
    if (L.sd.splits > 1) {
      L.off_part = off;
      off = align_up(off + size_t(L.sd.splits) * p.B * p.R * p.CV * 4);
    }
  } else {
    L.tcp = tc_plan(p.B, p.R, p.N, p.D, sm);
    const size_t KP = static_cast<size_t>(L.tcp.KP);
    const int maxc = tc_max_chunk(L.tcp.KP);
    const size_t CPmax = static_cast<size_t>(tc_chunk_pad(p.CV < maxc ? p.CV : maxc));
    const size_t Nst = (p.N + 7) / 8 * 8;
    L.off_xpack = off;
    off = align_up(off + size_t(p.B) * p.R * KP * 2);
    L.off_rnorm = off;
    off = align_up(off + size_t(p.B) * p.R * 4);
    L.off_ypack = off;
    off = align_up(off + size_t(p.B) * p.N * KP * 2);
    L.off_vt = off;
    off = align_up(off + size_t(p.B) * CPmax * Nst * 2);
    if (L.tcp.splits > 1) {
      L.off_part = off;
      off = align_up(off + size_t(L.tcp.splits) * p.B * p.R * p.CV * 4);
    }
  }
  L.total = off;
  return L;
}

// The forward + backward sweep's extra outputs (tensor-core fp16/bf16 path).
struct GwArgs {
  const float* g;      // [B, R, g_ld], channel 0
  int64_t g_ld;
  uint32_t* gpack;     // [B, R]
  float* gscale;       // [B]
  float* gtmax;        // [B, ceil(R / 128)]
  float* gw_part;      // [ceil(R / 128), B, N]
  bool keep_splits;    // leave the pass's split partials uncombined (the caller reads them)
};

// Run one pass into `out` ([B, R, CV] float32) using workspace `ws`; with
// `gw`, the same sweep also writes the column sums sum_i K_ij g_i of every
// 128-row tile (tensor-core fp16/bf16 path only).
gs_status run_pass(const Pass& p, const PassLayout& L, float* out, uint8_t* ws, cudaStream_t s,
                   const GwArgs* gw = nullptr) {
  if (gw && L.path != kPathTcHalf) return GS_ERR_UNSUPPORTED;
  const int64_t total = p.B * p.R * p.CV;
  if (total == 0) return GS_OK;
  if (p.N == 0) {
    GS_CUDA(cudaMemsetAsync(out, 0, size_t(total) * 4, s));
    return GS_OK;
  }
  if (!L.tc) {
    const float* values = static_cast<const float*>(p.w);
    if (p.vmode != 0) {
      float* v = reinterpret_cast<float*>(ws + L.off_vals);
      GS_CUDA(launch_pack_values_f32(p.w, p.src_ld > 0 ? p.src_ld : p.C, p.cols_pts, p.rows_pts,
                                     v, p.B, p.N, p.R, p.D, p.C, p.vmode, s));
      values = v;
    }
    const int S = L.sd.splits;
    float* dst = S > 1 ? reinterpret_cast<float*>(ws + L.off_part) : out;
    for (int c0 = 0; c0 < p.CV; c0 += kSdMaxChunk) {
      SdArgs a{};
      a.x = static_cast<const float*>(p.rows_pts);
      a.y = static_cast<const float*>(p.cols_pts);
      a.w = values;
      a.ldw = (p.vmode == 0 && p.src_ld > 0) ? static_cast<int>(p.src_ld) : p.CV;
      a.c0 = c0;
      a.cw = (p.CV - c0) < kSdMaxChunk ? (p.CV - c0) : kSdMaxChunk;
      a.out = dst;
      a.out_l = nullptr;
      a.ldo = p.CV;
      a.split_stride = S > 1 ? total : 0;
      a.B = p.B;
      a.M = p.R;
      a.N = p.N;
      a.D = p.D;
      a.scale = coord_scale(p.tau);
      a.plan = L.sd;
      a.shift_mode = p.shift_mode;
      a.shift_src = p.shift_src;
      a.shift_ld = p.shift_ld;
      a.shift_c = p.shift_c;
      a.shift_scale = p.shift_scale;
      GS_CUDA(launch_small_d_sum(a, s));
    }
    if (S > 1) GS_CUDA(launch_combine_sum(dst, S, total, out, s));
    return GS_OK;
  }
  if (L.path == kPathTcF32) {
    const int S = L.f32.splits;
    float* dst = S > 1 ? reinterpret_cast<float*>(ws + L.off_part) : out;
    F32Args a{};
    a.x = p.rows_pts;
    a.y = p.cols_pts;
    a.w = p.w;
    a.dt = GS_F32;
    a.values = static_cast<TcValues>(p.vmode);
    a.src_ld = p.src_ld;
    if (p.shift_mode == 1 || p.shift_mode == 2) {
      a.shift_mode = p.shift_mode;
      a.shift_src = p.shift_src;
      a.shift_ld = p.shift_ld;
      a.shift_c = p.shift_c;
      a.shift_scale = p.shift_scale;
    } else if (p.shift_mode != 0) {
      return GS_ERR_UNSUPPORTED;   // squared-distance modes: CUDA-core path only
    }
    a.C = p.C;
    a.CV = p.CV;
    a.out = dst;
    a.split_stride = S > 1 ? total : 0;
    a.B = p.B;
    a.M = p.R;
    a.N = p.N;
    a.D = p.D;
    a.tau = p.tau;
    a.plan = L.f32;
    a.zc = reinterpret_cast<float*>(ws + L.off_zc);
    a.xpack = reinterpret_cast<float*>(ws + L.off_xpack);
    a.rnorm = reinterpret_cast<float*>(ws + L.off_rnorm);
    a.ypack = reinterpret_cast<float*>(ws + L.off_ypack);
    a.qw = reinterpret_cast<float*>(ws + L.off_qw);
    a.vt = reinterpret_cast<float*>(ws + L.off_vt);
    GS_CUDA(launch_tc_f32_sum(a, s));
    if (S > 1) GS_CUDA(launch_combine_sum(dst, S, total, out, s));
    return GS_OK;
  }
  const int S = L.tcp.splits;
  float* dst = S > 1 ? reinterpret_cast<float*>(ws + L.off_part) : out;
  TcArgs a{};
  a.x = p.rows_pts;
  a.y = p.cols_pts;
  a.w = p.w;
  a.w_is_f32 = p.w_is_f32;
  a.values = static_cast<TcValues>(p.vmode);
  a.C = p.C;
  a.CV = p.CV;
  a.out = dst;
  a.split_stride = S > 1 ? total : 0;
  a.B = p.B;
  a.M = p.R;
  a.N = p.N;
  a.D = p.D;
  a.dt = p.dt;
  a.tau = p.tau;
  a.plan = L.tcp;
  a.xpack = ws + L.off_xpack;
  a.rnorm = reinterpret_cast<float*>(ws + L.off_rnorm);
  a.ypack = ws + L.off_ypack;
  a.vt = ws + L.off_vt;
  if (gw) {
    a.g = gw->g;
    a.g_ld = gw->g_ld;
    a.gpack = gw->gpack;
    a.gscale = gw->gscale;
    a.gtmax = gw->gtmax;
    a.gw_part = gw->gw_part;
  }
  GS_CUDA(launch_tc_sum(a, s));
  if (S > 1 && !(gw && gw->keep_splits)) GS_CUDA(launch_combine_sum(dst, S, total, out, s));
  return GS_OK;
}

Pass fwd_pass(const void* x, const void* y, const void* w, int64_t B, int64_t M, int64_t N,
              int64_t D, int64_t C, float tau, gs_dtype dt) {
  Pass p{};
  p.rows_pts = x;
  p.cols_pts = y;
  p.w = w;
  p.w_is_f32 = dt == GS_F32;
  p.vmode = 0;
  p.B = B;
  p.R = M;
  p.N = N;
  p.D = static_cast<int>(D);
  p.C = static_cast<int>(C);
  p.CV = static_cast<int>(C);
  p.dt = dt;
  p.tau = tau;
  return p;
}

// Forward + backward in one call: the x-gradient pass (values [w, w (y - z)],
// whose first C channels are the forward sum) into `saved`, and dL/dw either
// from the same sweep (fp16 / bf16, C = 1, 1 + D <= 48: each kernel value
// computed once) or from the separate pass rows y / columns x / values g.
constexpr int kFusedMaxD = 47;

struct FwdBwdLayout {
  Pass px, py;
  PassLayout lx, ly;
  bool fused;
  int CV;
  int64_t RT;          // 128-row tiles of the fused sweep's dL/dw partials
  size_t off_saved, off_gpack, off_gscale, off_gtmax, off_gwpart, off_pass;
  size_t total;
};

FwdBwdLayout fwd_bwd_layout(const void* x, const void* y, const void* w, const float* g, int64_t B,
                            int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                            int sm, bool want_w) {
  FwdBwdLayout L{};
  L.CV = value_channels(1, static_cast<int>(C), static_cast<int>(D));
  L.px = fwd_pass(x, y, w, B, M, N, D, C, tau, dt);
  L.px.vmode = 1;
  L.px.CV = L.CV;
  L.lx = pass_layout(L.px, sm);
  L.fused = want_w && dt != GS_F32 && C == 1 && D <= kFusedMaxD;
  L.RT = (M + 127) / 128;
  size_t off = 0;
  L.off_saved = off;
  off = align_up(off + size_t(B) * M * L.CV * 4);
  size_t pass = L.lx.total;
  if (L.fused) {
    L.off_gpack = off;
    off = align_up(off + size_t(B) * M * 4);
    L.off_gscale = off;
    off = align_up(off + size_t(B) * 4);
    L.off_gtmax = off;
    off = align_up(off + size_t(B) * L.RT * 4);
    L.off_gwpart = off;
    off = align_up(off + size_t(L.RT) * B * N * 4);
  } else if (want_w) {
    L.py = fwd_pass(y, x, g, B, N, M, D, C, tau, dt);
    L.py.w_is_f32 = true;
    L.ly = pass_layout(L.py, sm);
    if (L.ly.total > pass) pass = L.ly.total;
  }
  L.off_pass = off;
  L.total = align_up(off + pass);
  return L;
}

// Gradients = up to two passes (grad.cu): rows y / columns x with values
// [g, g (x - z)] for dL/dw and dL/dy, and rows x / columns y with values
// [w, w (y - z) (, w |y - z|^2)] for dL/dx (and dL/dtau), each followed by an
// epilogue.  They run one after the other and share the pass scratch; the
// pass outputs o_y, o_x and the per-row dL/dtau terms sit after it.
struct VjpLayout {
  Pass py, px, pt;
  PassLayout ly, lx, lt;
  bool do_y, do_x, do_t, y_direct;   // y_direct: the y pass writes grad_w itself
  size_t off_oy, off_ox, off_ot, off_tau;
  size_t total;
};

VjpLayout vjp_layout(const void* x, const void* y, const void* w, const float* g, int64_t B,
                     int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt, int sm,
                     bool want_x, bool want_y, bool want_w, bool want_tau) {
  VjpLayout L{};
  L.do_y = want_w || want_y;
  L.py = fwd_pass(y, x, g, B, N, M, D, C, tau, dt);
  L.py.w_is_f32 = true;
  L.py.vmode = want_y ? 1 : 0;
  L.py.CV = value_channels(L.py.vmode, static_cast<int>(C), static_cast<int>(D));
  L.y_direct = !want_y;
  // dL/dtau: on the CUDA-core path a pass whose kernel values carry the scaled
  // squared distance (no cancellation); on the tensor-core path the extra
  // value channel w |y - z|^2 of the grad_x pass
  L.do_t = want_tau && pass_path(dt, static_cast<int>(D)) == kPathSmallD;
  L.do_x = want_x || (want_tau && !L.do_t);
  L.px = fwd_pass(x, y, w, B, M, N, D, C, tau, dt);
  L.px.vmode = (want_tau && !L.do_t) ? 2 : 1;
  L.px.CV = value_channels(L.px.vmode, static_cast<int>(C), static_cast<int>(D));
  L.pt = fwd_pass(x, y, w, B, M, N, D, C, tau, dt);
  L.pt.shift_mode = 3;
  size_t scratch = 0;
  if (L.do_y) {
    L.ly = pass_layout(L.py, sm);
    scratch = L.ly.total;
  }
  if (L.do_x) {
    L.lx = pass_layout(L.px, sm);
    if (L.lx.total > scratch) scratch = L.lx.total;
  }
  if (L.do_t) {
    L.lt = pass_layout(L.pt, sm);
    if (L.lt.total > scratch) scratch = L.lt.total;
  }
  size_t off = align_up(scratch);
  if (L.do_y && !L.y_direct) {
    L.off_oy = off;
    off = align_up(off + size_t(B) * N * L.py.CV * 4);
  }
  if (L.do_x) {
    L.off_ox = off;
    off = align_up(off + size_t(B) * M * L.px.CV * 4);
  }
  if (L.do_t) {
    L.off_ot = off;
    off = align_up(off + size_t(B) * M * C * 4);
  }
  if (want_tau) {
    L.off_tau = off;
    off = align_up(off + size_t(B) * M * 4);
  }
  L.total = off;
  return L;
}

// fp16 / bf16 inputs of the k-nearest reduction and of the log-sum-exp
// backward are widened (exactly) to fp32 copies at the front of the workspace;
// the fp32 implementation then runs on them.
size_t widened_bytes(gs_dtype dt, int64_t B, int64_t M, int64_t N, int64_t D, int64_t Cw) {
  if (dt == GS_F32) return 0;
  return align_up(size_t(B) * M * D * 4) + align_up(size_t(B) * N * D * 4) +
         align_up(size_t(B) * N * Cw * 4);
}

// Log-sum-exp forward on the fp32 tensor-core path (D > 8): packed operands,
// the column norms / log-weights, and the per-split (m, l) partials.
struct LseF32Layout {
  F32Plan plan;
  size_t off_zc, off_xpack, off_rnorm, off_ypack, off_qw, off_m, off_l, total;
};

LseF32Layout lse_f32_layout(int64_t B, int64_t M, int64_t N, int64_t D, int64_t C, gs_dtype dt,
                            int sm) {
  LseF32Layout L{};
  // fp16 / bf16 values are exact in tf32: unsplit rows, one MMA per K step
  L.plan = f32_plan(B, M, N, D, sm, dt == GS_F32);
  const size_t rowb = size_t(L.plan.split ? 2 : 1) * L.plan.Kp * 4;
  const size_t Nq = (N + 127) / 128 * 128;
  size_t off = 0;
  L.off_zc = off;   // column centres [B, D], then one max word per batch
  off = align_up(off + size_t(B) * (D + 1) * 4);
  L.off_xpack = off;
  off = align_up(off + size_t(B) * M * rowb);
  L.off_rnorm = off;
  off = align_up(off + size_t(B) * M * 4);
  L.off_ypack = off;
  off = align_up(off + size_t(B) * N * rowb);
  L.off_qw = off;
  off = align_up(off + size_t(B) * Nq * 16);
  L.off_m = off;
  off = align_up(off + size_t(L.plan.splits) * B * M * C * 4);
  L.off_l = off;
  off = align_up(off + size_t(L.plan.splits) * B * M * C * 4);
  L.total = off;
  return L;
}

// Log-sum-exp backward (CUDA-core path), per channel c with the shift
// -lse_c log2 e folded into the exponent: rows x / columns y with values
// [w_c, w_c (y - z)] and a per-row shift (dL/dx), the same rows with values w_c,
// the per-row shift and the squared-distance factor (dL/dtau), and rows y /
// columns x with values [g_c, g_c (x - z)] and a per-column shift (dL/dw, dL/dy).
struct LseBwdLayout {
  bool tau_in_x;
  Pass px, pt, py;
  PassLayout lx, lt, ly;
  size_t off_ox, off_ot, off_oy, off_tau, total;
};

LseBwdLayout lse_bwd_layout(const void* x, const void* y, const void* w, const float* lse,
                            const float* g, int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                            float tau, int sm) {
  LseBwdLayout L{};
  const float kNegLog2e = -1.4426950408889634f;
  // D > 8 (tf32 tensor-core passes): the dL/dtau sums ride as a third value
  // part of the x pass instead of a squared-distance pass
  L.tau_in_x = pass_path(GS_F32, static_cast<int>(D)) != kPathSmallD;
  L.px = fwd_pass(x, y, w, B, M, N, D, 1, tau, GS_F32);
  L.px.vmode = L.tau_in_x ? 2 : 1;
  L.px.CV = value_channels(L.px.vmode, 1, static_cast<int>(D));
  L.px.src_ld = C;
  L.px.shift_mode = 1;
  L.px.shift_src = lse;
  L.px.shift_ld = C;
  L.px.shift_scale = kNegLog2e;
  L.pt = fwd_pass(x, y, w, B, M, N, D, 1, tau, GS_F32);
  L.pt.src_ld = C;
  L.pt.shift_mode = 4;
  L.pt.shift_src = lse;
  L.pt.shift_ld = C;
  L.pt.shift_scale = kNegLog2e;
  L.py = fwd_pass(y, x, g, B, N, M, D, 1, tau, GS_F32);
  L.py.vmode = 1;
  L.py.CV = value_channels(1, 1, static_cast<int>(D));
  L.py.src_ld = C;
  L.py.shift_mode = 2;
  L.py.shift_src = lse;
  L.py.shift_ld = C;
  L.py.shift_scale = kNegLog2e;
  L.lx = pass_layout(L.px, sm);
  if (!L.tau_in_x) L.lt = pass_layout(L.pt, sm);
  L.ly = pass_layout(L.py, sm);
  size_t scratch = L.lx.total;
  if (L.lt.total > scratch) scratch = L.lt.total;
  if (L.ly.total > scratch) scratch = L.ly.total;
  size_t off = align_up(scratch);
  L.off_ox = off;
  off = align_up(off + size_t(B) * M * L.px.CV * 4);
  L.off_ot = off;
  off = align_up(off + size_t(B) * M * 4);
  L.off_oy = off;
  off = align_up(off + size_t(B) * N * L.py.CV * 4);
  L.off_tau = off;
  off = align_up(off + size_t(B) * M * 4);
  L.total = off;
  return L;
}

// Diffusion operator: q = K 1 and u = K q^-alpha (scales), and K (s V) (apply),
// each one forward pass over a single point set, with f32 value blocks.
struct DiffusionLayout {
  PassLayout lp;
  size_t off_vals, off_a, off_b, total;
};

DiffusionLayout diffusion_layout(int64_t B, int64_t N, int64_t D, int64_t C, gs_dtype dt, int sm) {
  DiffusionLayout L{};
  Pass p = fwd_pass(nullptr, nullptr, nullptr, B, N, N, D, C, 1.f, dt);
  p.w_is_f32 = true;
  L.lp = pass_layout(p, sm);
  size_t off = align_up(L.lp.total);
  L.off_vals = off;
  off = align_up(off + size_t(B) * N * C * 4);
  L.off_a = off;
  off = align_up(off + size_t(B) * N * 4);
  L.off_b = off;
  off = align_up(off + size_t(B) * N * 4);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

int gs_version(void) { return 100; }

const char* gs_status_string(gs_status st) {
  switch (st) {
    case GS_OK: return "ok";
    case GS_ERR_INVALID_ARG: return "invalid argument";
    case GS_ERR_UNSUPPORTED: return "unsupported dtype/shape combination";
    case GS_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case GS_ERR_WORKSPACE: return "workspace too small";
    case GS_ERR_TIMEOUT: return "device-side wait timed out";
    case GS_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

size_t gs_workspace_bytes(gs_op op, int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                          gs_dtype dt) {
  if (op != GS_OP_SUM && op != GS_OP_LSE && op != GS_OP_SUM_BWD && op != GS_OP_LSE_BWD &&
      op != GS_OP_KNN && op != GS_OP_DIFFUSION && op != GS_OP_SUM_FWD_BWD &&
      op != GS_OP_DIFFUSION_BLOCK)
    return kBad;
  if (op == GS_OP_DIFFUSION) {
    // one point set: M = N; C = columns of the block V (1 for the scales)
    if (check_dims(GS_OP_SUM, B, N, N, D, C, dt) != GS_OK || M != N) return kBad;
    if (B == 0 || N == 0) return 0;
    return diffusion_layout(B, N, D, C, dt, sm_count()).total;
  }
  if (op == GS_OP_KNN) {
    // C carries K for this op
    if (C < 1 || C > kKnnMaxK || check_dims(GS_OP_KNN, B, M, N, D, 1, dt) != GS_OK)
      return kBad;
    if (B == 0 || M == 0 || N == 0) return 0;
    const KnnPlan kp = knn_plan(B, M, N, D, static_cast<int>(C), sm_count());
    return widened_bytes(dt, B, M, N, D, 0) + align_up(size_t(kp.splits) * B * M * C * 8);
  }
  if (check_dims(op, B, M, N, D, C, dt) != GS_OK) return kBad;
  if (B == 0) return 0;
  const int sm = sm_count();
  if (op == GS_OP_SUM) {
    if (M == 0 || N == 0) return 0;
    return pass_layout(fwd_pass(nullptr, nullptr, nullptr, B, M, N, D, C, 1.f, dt), sm).total;
  }
  if (op == GS_OP_LSE) {
    if (M == 0 || N == 0) return 0;
    if (dt != GS_F32 || D > kSdMaxD) return lse_f32_layout(B, M, N, D, C, dt, sm).total;
    const SdPlan sp = sd_plan(B, M, N, static_cast<int>(D), C, sm, 32);
    return align_up(size_t(2) * sp.splits * B * M * C * 4);
  }
  if (op == GS_OP_DIFFUSION_BLOCK) {
    if (M == 0 || N == 0) return 0;
    Pass p = fwd_pass(nullptr, nullptr, nullptr, B, M, N, D, C, 1.f, dt);
    p.w_is_f32 = true;
    return pass_layout(p, sm).total;
  }
  if (op == GS_OP_SUM_FWD_BWD) {
    if (M == 0 || N == 0) return 0;
    return fwd_bwd_layout(nullptr, nullptr, nullptr, nullptr, B, M, N, D, C, 1.f, dt, sm, true)
        .total;
  }
  if (op == GS_OP_LSE_BWD) {
    if (M == 0 || N == 0) return 0;
    return widened_bytes(dt, B, M, N, D, C) +
           lse_bwd_layout(nullptr, nullptr, nullptr, nullptr, nullptr, B, M, N, D, C, 1.f, sm).total;
  }
  if (M == 0 || N == 0) return 0;
  return vjp_layout(nullptr, nullptr, nullptr, nullptr, B, M, N, D, C, 1.f, dt, sm, true, true, true,
                    true)
      .total;
}

gs_status gauss_sum_fwd(const void* x, const void* y, const void* w, float* out, int64_t B,
                        int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                        void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(w, B * N * C));
  GS_TRY(check_ptr(out, B * M * C));
  if (B == 0 || M == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Pass p = fwd_pass(x, y, w, B, M, N, D, C, tau, dt);
  const PassLayout L = pass_layout(p, sm_count());
  if (N > 0 && L.total > 0) {
    if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
    GS_TRY(check_ptr(ws, 1));
  }
  return run_pass(p, L, out, static_cast<uint8_t*>(ws), s);
}

gs_status gauss_lse_fwd(const void* x, const void* y, const void* w, float* out, int64_t B,
                        int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                        void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_LSE, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(w, B * N * C));
  GS_TRY(check_ptr(out, B * M * C));
  if (B == 0 || M == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N == 0) {
    GS_CUDA(launch_fill(out, B * M * C, -INFINITY, s));
    return GS_OK;
  }
  const int sm = sm_count();
  if (dt != GS_F32 || D > kSdMaxD) {
    // tensor-core (tf32) path: running-maximum (m, l) per split, then the finalize
    const LseF32Layout L = lse_f32_layout(B, M, N, D, C, dt, sm);
    if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
    GS_TRY(check_ptr(ws, 1));
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    const int64_t tot = B * M * C;
    F32Args a{};
    a.x = x;
    a.y = y;
    a.w = w;
    a.dt = dt;
    a.values = kValuesW;
    a.C = static_cast<int>(C);
    a.CV = static_cast<int>(C);
    a.out = reinterpret_cast<float*>(w8 + L.off_m);
    a.out_l = reinterpret_cast<float*>(w8 + L.off_l);
    a.lse = true;
    a.split_stride = tot;
    a.B = B;
    a.M = M;
    a.N = N;
    a.D = static_cast<int>(D);
    a.tau = tau;
    a.plan = L.plan;
    a.zc = reinterpret_cast<float*>(w8 + L.off_zc);
    a.xpack = reinterpret_cast<float*>(w8 + L.off_xpack);
    a.rnorm = reinterpret_cast<float*>(w8 + L.off_rnorm);
    a.ypack = reinterpret_cast<float*>(w8 + L.off_ypack);
    a.qw = reinterpret_cast<float*>(w8 + L.off_qw);
    a.vt = nullptr;
    GS_CUDA(launch_tc_f32_sum(a, s));
    LseFinalizeArgs f{};
    f.part_m = a.out;
    f.part_l = a.out_l;
    f.splits = L.plan.splits;
    f.split_stride = tot;
    f.out = out;
    f.x = static_cast<const float*>(x);
    f.y = static_cast<const float*>(y);
    f.w = static_cast<const float*>(w);
    f.B = B;
    f.M = M;
    f.N = N;
    f.D = static_cast<int>(D);
    f.C = static_cast<int>(C);
    f.scale = coord_scale(tau);
    f.no_fallback = 1;
    GS_CUDA(launch_lse_finalize(f, s));
    return GS_OK;
  }
  const SdPlan sp = sd_plan(B, M, N, static_cast<int>(D), C, sm, 32);
  const size_t need = align_up(size_t(2) * sp.splits * B * M * C * 4);
  if (ws_bytes < need) return GS_ERR_WORKSPACE;
  GS_TRY(check_ptr(ws, 1));
  const int64_t total = B * M * C;
  float* part_m = static_cast<float*>(ws);
  float* part_l = part_m + size_t(sp.splits) * total;
  const float scale = coord_scale(tau);
  for (int c0 = 0; c0 < C; c0 += kSdMaxChunk) {
    SdArgs a{};
    a.x = static_cast<const float*>(x);
    a.y = static_cast<const float*>(y);
    a.w = static_cast<const float*>(w);
    a.ldw = static_cast<int>(C);
    a.c0 = c0;
    a.cw = static_cast<int>((C - c0) < kSdMaxChunk ? (C - c0) : kSdMaxChunk);
    a.out = part_m;
    a.out_l = part_l;
    a.ldo = static_cast<int>(C);
    a.split_stride = total;
    a.B = B;
    a.M = M;
    a.N = N;
    a.D = static_cast<int>(D);
    a.scale = scale;
    a.plan = sp;
    GS_CUDA(launch_small_d_lse(a, s));
  }
  LseFinalizeArgs f{};
  f.part_m = part_m;
  f.part_l = part_l;
  f.splits = sp.splits;
  f.split_stride = total;
  f.out = out;
  f.x = static_cast<const float*>(x);
  f.y = static_cast<const float*>(y);
  f.w = static_cast<const float*>(w);
  f.B = B;
  f.M = M;
  f.N = N;
  f.D = static_cast<int>(D);
  f.C = static_cast<int>(C);
  f.scale = scale;
  GS_CUDA(launch_lse_finalize(f, s));
  return GS_OK;
}

gs_status gauss_sum_vjp(const void* x, const void* y, const void* w, const float* g,
                        float* grad_x, float* grad_y, float* grad_w, float* grad_tau, int64_t B,
                        int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                        void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM_BWD, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(w, B * N * C));
  GS_TRY(check_ptr(g, B * M * C));
  if (grad_x) GS_TRY(check_ptr(grad_x, B * M * D));
  if (grad_y) GS_TRY(check_ptr(grad_y, B * N * D));
  if (grad_w) GS_TRY(check_ptr(grad_w, B * N * C));
  if (!grad_x && !grad_y && !grad_w && !grad_tau) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (grad_tau) GS_CUDA(cudaMemsetAsync(grad_tau, 0, sizeof(float), s));
  if (B == 0) return GS_OK;
  if (M == 0 || N == 0) {   // every kernel sum is empty: all gradients vanish
    if (grad_x && M > 0) GS_CUDA(cudaMemsetAsync(grad_x, 0, size_t(B) * M * D * 4, s));
    if (grad_y && N > 0) GS_CUDA(cudaMemsetAsync(grad_y, 0, size_t(B) * N * D * 4, s));
    if (grad_w && N > 0) GS_CUDA(cudaMemsetAsync(grad_w, 0, size_t(B) * N * C * 4, s));
    return GS_OK;
  }
  const VjpLayout L = vjp_layout(x, y, w, g, B, M, N, D, C, tau, dt, sm_count(), grad_x != nullptr,
                                 grad_y != nullptr, grad_w != nullptr, grad_tau != nullptr);
  if (L.total > 0) {
    if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
    GS_TRY(check_ptr(ws, 1));
  }
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  if (L.do_y) {
    if (L.y_direct) {
      GS_TRY(run_pass(L.py, L.ly, grad_w, wsb, s));
    } else {
      float* oy = reinterpret_cast<float*>(wsb + L.off_oy);
      GS_TRY(run_pass(L.py, L.ly, oy, wsb, s));
      GS_CUDA(launch_grad_y_epilogue(y, w, dt, oy, grad_y, grad_w, B, N, static_cast<int>(D),
                                     static_cast<int>(C), L.py.CV, tau, s));
    }
  }
  float* tau_rows = grad_tau ? reinterpret_cast<float*>(wsb + L.off_tau) : nullptr;
  if (L.do_x) {
    float* ox = reinterpret_cast<float*>(wsb + L.off_ox);
    GS_TRY(run_pass(L.px, L.lx, ox, wsb, s));
    GS_CUDA(launch_grad_x_epilogue(x, dt, g, ox, grad_x, L.do_t ? nullptr : tau_rows, B, M,
                                   static_cast<int>(D), static_cast<int>(C), L.px.CV, tau, s));
  }
  if (L.do_t) {
    // o[i,c] = sum_j K_ij w_jc (tau/2 log2 e) |x_i - y_j|^2, so
    // dL/dtau(i) = -1/2 sum_c g_ic o[i,c] / (tau/2 log2 e)
    float* ot = reinterpret_cast<float*>(wsb + L.off_ot);
    GS_TRY(run_pass(L.pt, L.lt, ot, wsb, s));
    const double cfac = 0.5 * static_cast<double>(tau) * 1.4426950408889634074;
    GS_CUDA(launch_weighted_rows(g, ot, tau_rows, B * M, static_cast<int>(C), 0,
                                 static_cast<int>(C), static_cast<float>(-0.5 / cfac), false, s));
  }
  if (grad_tau) GS_CUDA(launch_sum_rows(tau_rows, B * M, grad_tau, s));
  return GS_OK;
}

gs_status gauss_sum_bwd(const void* x, const void* y, const void* w, const float* g,
                        float* grad_x, float* grad_w, int64_t B, int64_t M, int64_t N, int64_t D,
                        int64_t C, float tau, gs_dtype dt, void* ws, size_t ws_bytes,
                        gs_stream_t stream) {
  return gauss_sum_vjp(x, y, w, g, grad_x, nullptr, grad_w, nullptr, B, M, N, D, C, tau, dt, ws,
                       ws_bytes, stream);
}

gs_status gauss_sum_fwd_saved(const void* x, const void* y, const void* w, float* out,
                              float* saved, int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                              float tau, gs_dtype dt, void* ws, size_t ws_bytes,
                              gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM_BWD, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(w, B * N * C));
  GS_TRY(check_ptr(out, B * M * C));
  const int CV = value_channels(1, static_cast<int>(C), static_cast<int>(D));
  GS_TRY(check_ptr(saved, B * M * CV));
  if (B == 0 || M == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N == 0) {
    GS_CUDA(cudaMemsetAsync(out, 0, size_t(B) * M * C * 4, s));
    GS_CUDA(cudaMemsetAsync(saved, 0, size_t(B) * M * CV * 4, s));
    return GS_OK;
  }
  // the x-gradient pass: values [w, w (y - z)]; its first C channels are the sum
  Pass px = fwd_pass(x, y, w, B, M, N, D, C, tau, dt);
  px.vmode = 1;
  px.CV = CV;
  const PassLayout lx = pass_layout(px, sm_count());
  if (lx.total > 0) {
    if (ws_bytes < lx.total) return GS_ERR_WORKSPACE;
    GS_TRY(check_ptr(ws, 1));
  }
  GS_TRY(run_pass(px, lx, saved, static_cast<uint8_t*>(ws), s));
  GS_CUDA(cudaMemcpy2DAsync(out, size_t(C) * 4, saved, size_t(CV) * 4, size_t(C) * 4,
                            size_t(B) * M, cudaMemcpyDeviceToDevice, s));
  return GS_OK;
}

gs_status gauss_sum_bwd_saved(const void* x, const void* y, const void* w, const float* g,
                              const float* saved, float* grad_x, float* grad_w, int64_t B,
                              int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                              void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM_BWD, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(w, B * N * C));
  GS_TRY(check_ptr(g, B * M * C));
  const int CV = value_channels(1, static_cast<int>(C), static_cast<int>(D));
  GS_TRY(check_ptr(saved, B * M * CV));
  if (grad_x) GS_TRY(check_ptr(grad_x, B * M * D));
  if (grad_w) GS_TRY(check_ptr(grad_w, B * N * C));
  if (!grad_x && !grad_w) return GS_OK;
  if (B == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M == 0 || N == 0) {   // every kernel sum is empty: all gradients vanish
    if (grad_x && M > 0) GS_CUDA(cudaMemsetAsync(grad_x, 0, size_t(B) * M * D * 4, s));
    if (grad_w && N > 0) GS_CUDA(cudaMemsetAsync(grad_w, 0, size_t(B) * N * C * 4, s));
    return GS_OK;
  }
  if (grad_w) {   // rows y, columns x, values g: dL/dw directly
    Pass py = fwd_pass(y, x, g, B, N, M, D, C, tau, dt);
    py.w_is_f32 = true;
    const PassLayout ly = pass_layout(py, sm_count());
    if (ly.total > 0) {
      if (ws_bytes < ly.total) return GS_ERR_WORKSPACE;
      GS_TRY(check_ptr(ws, 1));
    }
    GS_TRY(run_pass(py, ly, grad_w, static_cast<uint8_t*>(ws), s));
  }
  if (grad_x && C == 1)   // one row per warp; the same arithmetic as the general epilogue
    GS_CUDA(launch_fwd_bwd_epilogue(x, dt, g, saved, 1, 0, nullptr, grad_x, B, M,
                                    static_cast<int>(D), CV, tau, s));
  else if (grad_x)
    GS_CUDA(launch_grad_x_epilogue(x, dt, g, saved, grad_x, nullptr, B, M, static_cast<int>(D),
                                   static_cast<int>(C), CV, tau, s));
  return GS_OK;
}

gs_status gauss_sum_fwd_bwd(const void* x, const void* y, const void* w, const float* g, float* out,
                            float* grad_x, float* grad_w, int64_t B, int64_t M, int64_t N,
                            int64_t D, int64_t C, float tau, gs_dtype dt, void* ws, size_t ws_bytes,
                            gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM_FWD_BWD, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(w, B * N * C));
  GS_TRY(check_ptr(g, B * M * C));
  GS_TRY(check_ptr(out, B * M * C));
  if (grad_x) GS_TRY(check_ptr(grad_x, B * M * D));
  if (grad_w) GS_TRY(check_ptr(grad_w, B * N * C));
  if (B == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M == 0 || N == 0) {   // empty sums: out = 0 and every gradient vanishes
    if (M > 0) GS_CUDA(cudaMemsetAsync(out, 0, size_t(B) * M * C * 4, s));
    if (grad_x && M > 0) GS_CUDA(cudaMemsetAsync(grad_x, 0, size_t(B) * M * D * 4, s));
    if (grad_w && N > 0) GS_CUDA(cudaMemsetAsync(grad_w, 0, size_t(B) * N * C * 4, s));
    return GS_OK;
  }
  const FwdBwdLayout L =
      fwd_bwd_layout(x, y, w, g, B, M, N, D, C, tau, dt, sm_count(), grad_w != nullptr);
  if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
  GS_TRY(check_ptr(ws, 1));
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* saved = reinterpret_cast<float*>(wsb + L.off_saved);
  if (L.fused) {
    // one sweep; the x-side sums stay as the sweep's split partials, which the
    // epilogue adds in the combine's fixed order while it forms out and grad_x
    GwArgs ga{};
    ga.g = g;
    ga.g_ld = C;
    ga.gpack = reinterpret_cast<uint32_t*>(wsb + L.off_gpack);
    ga.gscale = reinterpret_cast<float*>(wsb + L.off_gscale);
    ga.gtmax = reinterpret_cast<float*>(wsb + L.off_gtmax);
    ga.gw_part = reinterpret_cast<float*>(wsb + L.off_gwpart);
    ga.keep_splits = true;
    GS_TRY(run_pass(L.px, L.lx, saved, wsb + L.off_pass, s, &ga));
    const int S = L.lx.tcp.splits;
    const float* part = S > 1 ? reinterpret_cast<const float*>(wsb + L.off_pass + L.lx.off_part)
                              : saved;
    GS_CUDA(launch_combine_sum(ga.gw_part, static_cast<int>(L.RT), B * N, grad_w, s));
    GS_CUDA(launch_fwd_bwd_epilogue(x, dt, g, part, S, B * M * L.CV, out, grad_x, B, M,
                                    static_cast<int>(D), L.CV, tau, s));
    return GS_OK;
  }
  GS_TRY(run_pass(L.px, L.lx, saved, wsb + L.off_pass, s));
  if (grad_w) GS_TRY(run_pass(L.py, L.ly, grad_w, wsb + L.off_pass, s));
  if (C == 1) {
    GS_CUDA(launch_fwd_bwd_epilogue(x, dt, g, saved, 1, 0, out, grad_x, B, M, static_cast<int>(D),
                                    L.CV, tau, s));
    return GS_OK;
  }
  GS_CUDA(cudaMemcpy2DAsync(out, size_t(C) * 4, saved, size_t(L.CV) * 4, size_t(C) * 4,
                            size_t(B) * M, cudaMemcpyDeviceToDevice, s));
  if (grad_x)
    GS_CUDA(launch_grad_x_epilogue(x, dt, g, saved, grad_x, nullptr, B, M, static_cast<int>(D),
                                   static_cast<int>(C), L.CV, tau, s));
  return GS_OK;
}

gs_status gauss_lse_bwd(const void* x, const void* y, const void* w, const float* lse,
                        const float* g, float* grad_x, float* grad_y, float* grad_w,
                        float* grad_tau, int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                        float tau, gs_dtype dt, void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_LSE_BWD, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(w, B * N * C));
  GS_TRY(check_ptr(lse, B * M * C));
  GS_TRY(check_ptr(g, B * M * C));
  if (grad_x) GS_TRY(check_ptr(grad_x, B * M * D));
  if (grad_y) GS_TRY(check_ptr(grad_y, B * N * D));
  if (grad_w) GS_TRY(check_ptr(grad_w, B * N * C));
  if (!grad_x && !grad_y && !grad_w && !grad_tau) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dt != GS_F32 && B > 0 && M > 0 && N > 0) {
    // exact fp32 copies of x, y, w, then the fp32 backward on them
    const size_t pre = widened_bytes(dt, B, M, N, D, C);
    if (ws_bytes < pre) return GS_ERR_WORKSPACE;
    GS_TRY(check_ptr(ws, 1));
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    float* wx = reinterpret_cast<float*>(w8);
    float* wy = reinterpret_cast<float*>(w8 + align_up(size_t(B) * M * D * 4));
    float* ww = reinterpret_cast<float*>(w8 + align_up(size_t(B) * M * D * 4) +
                                         align_up(size_t(B) * N * D * 4));
    GS_CUDA(launch_widen_to_f32(x, dt, wx, B * M * D, s));
    GS_CUDA(launch_widen_to_f32(y, dt, wy, B * N * D, s));
    GS_CUDA(launch_widen_to_f32(w, dt, ww, B * N * C, s));
    return gauss_lse_bwd(wx, wy, ww, lse, g, grad_x, grad_y, grad_w, grad_tau, B, M, N, D, C, tau,
                         GS_F32, w8 + pre, ws_bytes - pre, stream);
  }
  if (grad_tau) GS_CUDA(cudaMemsetAsync(grad_tau, 0, sizeof(float), s));
  if (B == 0) return GS_OK;
  if (M == 0 || N == 0) {   // no terms: every gradient vanishes
    if (grad_x && M > 0) GS_CUDA(cudaMemsetAsync(grad_x, 0, size_t(B) * M * D * 4, s));
    if (grad_y && N > 0) GS_CUDA(cudaMemsetAsync(grad_y, 0, size_t(B) * N * D * 4, s));
    if (grad_w && N > 0) GS_CUDA(cudaMemsetAsync(grad_w, 0, size_t(B) * N * C * 4, s));
    return GS_OK;
  }
  LseBwdLayout L = lse_bwd_layout(x, y, w, lse, g, B, M, N, D, C, tau, sm_count());
  if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
  GS_TRY(check_ptr(ws, 1));
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* ox = reinterpret_cast<float*>(wsb + L.off_ox);
  float* ot = reinterpret_cast<float*>(wsb + L.off_ot);
  float* oy = reinterpret_cast<float*>(wsb + L.off_oy);
  float* tau_rows = reinterpret_cast<float*>(wsb + L.off_tau);
  const float* wf = static_cast<const float*>(w);
  const double cfac = 0.5 * static_cast<double>(tau) * 1.4426950408889634074;
  for (int c = 0; c < static_cast<int>(C); ++c) {
    const bool acc = c > 0;
    if (grad_x || grad_tau) {
      L.px.w = wf + c;
      L.px.shift_c = c;
      GS_TRY(run_pass(L.px, L.lx, ox, wsb, s));
      if (grad_tau && !L.tau_in_x) {
        L.pt.w = wf + c;
        L.pt.shift_c = c;
        GS_TRY(run_pass(L.pt, L.lt, ot, wsb, s));
      }
      GS_CUDA(launch_lse_x_tau_epilogue(static_cast<const float*>(x), g, ox,
                                        (grad_tau && !L.tau_in_x) ? ot : nullptr,
                                        grad_x, grad_tau ? tau_rows : nullptr, B, M,
                                        static_cast<int>(D), static_cast<int>(C), c, tau,
                                        static_cast<float>(1.0 / cfac), acc, s, L.px.CV));
    }
    if (grad_y || grad_w) {
      L.py.w = g + c;
      L.py.shift_c = c;
      GS_TRY(run_pass(L.py, L.ly, oy, wsb, s));
      GS_CUDA(launch_lse_grad_y_epilogue(static_cast<const float*>(y), wf, oy, grad_y, grad_w, B,
                                         N, static_cast<int>(D), static_cast<int>(C), c, tau, acc,
                                         s));
    }
  }
  if (grad_tau) GS_CUDA(launch_sum_rows(tau_rows, B * M, grad_tau, s));
  return GS_OK;
}

gs_status gauss_knn(const void* x, const void* y, float* out_sqdist, int64_t* out_index, int64_t B,
                    int64_t M, int64_t N, int64_t D, int64_t K, gs_dtype dt, void* ws,
                    size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_KNN, B, M, N, D, 1, dt));
  if (K < 1) return GS_ERR_INVALID_ARG;
  if (K > kKnnMaxK) return GS_ERR_UNSUPPORTED;
  GS_TRY(check_ptr(x, B * M * D));
  GS_TRY(check_ptr(y, B * N * D));
  GS_TRY(check_ptr(out_sqdist, B * M * K));
  GS_TRY(check_ptr(out_index, B * M * K));
  if (B == 0 || M == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N == 0) {   // no source: +inf distances, index -1 (all bytes 0xff)
    GS_CUDA(launch_fill(out_sqdist, B * M * K, INFINITY, s));
    GS_CUDA(cudaMemsetAsync(out_index, 0xff, size_t(B) * M * K * sizeof(int64_t), s));
    return GS_OK;
  }
  const KnnPlan kp = knn_plan(B, M, N, D, static_cast<int>(K), sm_count());
  const size_t pre = widened_bytes(dt, B, M, N, D, 0);
  const size_t need = pre + align_up(size_t(kp.splits) * B * M * K * 8);
  if (ws_bytes < need) return GS_ERR_WORKSPACE;
  GS_TRY(check_ptr(ws, 1));
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const float* xf = static_cast<const float*>(x);
  const float* yf = static_cast<const float*>(y);
  if (dt != GS_F32) {   // exact fp32 copies: the decisions are those of fp32 on the same values
    float* wx = reinterpret_cast<float*>(w8);
    float* wy = reinterpret_cast<float*>(w8 + align_up(size_t(B) * M * D * 4));
    GS_CUDA(launch_widen_to_f32(x, dt, wx, B * M * D, s));
    GS_CUDA(launch_widen_to_f32(y, dt, wy, B * N * D, s));
    xf = wx;
    yf = wy;
  }
  KnnArgs a{};
  a.x = xf;
  a.y = yf;
  a.part_d = reinterpret_cast<float*>(w8 + pre);
  a.part_i = reinterpret_cast<int*>(w8 + pre + size_t(kp.splits) * B * M * K * 4);
  a.out_d = out_sqdist;
  a.out_i = out_index;
  a.B = B;
  a.M = M;
  a.N = N;
  a.D = static_cast<int>(D);
  a.K = static_cast<int>(K);
  a.splits = kp.splits;
  a.cols_per_split = kp.cols_per_split;
  a.split_stride = B * M * K;
  GS_CUDA(launch_knn(a, s));
  return GS_OK;
}

gs_status gauss_diffusion_block(const void* x_rows, const void* x_cols, const float* v, float* out,
                                int64_t B, int64_t M, int64_t N, int64_t D, int64_t C, float tau,
                                gs_dtype dt, void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM, B, M, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x_rows, B * M * D));
  GS_TRY(check_ptr(x_cols, B * N * D));
  GS_TRY(check_ptr(v, B * N * C));
  GS_TRY(check_ptr(out, B * M * C));
  if (B == 0 || M == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N == 0) {
    GS_CUDA(cudaMemsetAsync(out, 0, size_t(B) * M * C * 4, s));
    return GS_OK;
  }
  Pass p = fwd_pass(x_rows, x_cols, v, B, M, N, D, C, tau, dt);
  p.w_is_f32 = true;
  const PassLayout L = pass_layout(p, sm_count());
  if (L.total > 0) {
    if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
    GS_TRY(check_ptr(ws, 1));
  }
  return run_pass(p, L, out, static_cast<uint8_t*>(ws), s);
}

gs_status gauss_diffusion_scales(const void* x, float* q_out, float* d_out, float* s_out,
                                 int64_t B, int64_t N, int64_t D, float tau, float alpha,
                                 gs_dtype dt, void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM, B, N, N, D, 1, dt));
  GS_TRY(check_tau(tau));
  if (!std::isfinite(alpha)) return GS_ERR_INVALID_ARG;
  GS_TRY(check_ptr(x, B * N * D));
  GS_TRY(check_ptr(s_out, B * N));
  if (q_out) GS_TRY(check_ptr(q_out, B * N));
  if (d_out) GS_TRY(check_ptr(d_out, B * N));
  if (B == 0 || N == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const DiffusionLayout L = diffusion_layout(B, N, D, 1, dt, sm_count());
  if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
  GS_TRY(check_ptr(ws, 1));
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* vals = reinterpret_cast<float*>(wsb + L.off_vals);
  float* q = q_out ? q_out : reinterpret_cast<float*>(wsb + L.off_a);
  float* u = reinterpret_cast<float*>(wsb + L.off_b);
  Pass p = fwd_pass(x, x, vals, B, N, N, D, 1, tau, dt);
  p.w_is_f32 = true;
  GS_CUDA(launch_diffusion_elementwise(0, nullptr, nullptr, vals, nullptr, B * N, 1, alpha, s));
  GS_TRY(run_pass(p, L.lp, q, wsb, s));                       // q = K 1
  GS_CUDA(launch_diffusion_elementwise(1, q, nullptr, vals, nullptr, B * N, 1, alpha, s));
  GS_TRY(run_pass(p, L.lp, u, wsb, s));                       // u = K q^-alpha
  GS_CUDA(launch_diffusion_elementwise(2, q, u, d_out, s_out, B * N, 1, alpha, s));
  return GS_OK;
}

gs_status gauss_diffusion_apply(const void* x, const float* s_scale, const float* v, float* out,
                                int64_t B, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                                void* ws, size_t ws_bytes, gs_stream_t stream) {
  GS_TRY(check_dims(GS_OP_SUM, B, N, N, D, C, dt));
  GS_TRY(check_tau(tau));
  GS_TRY(check_ptr(x, B * N * D));
  GS_TRY(check_ptr(s_scale, B * N));
  GS_TRY(check_ptr(v, B * N * C));
  GS_TRY(check_ptr(out, B * N * C));
  if (B == 0 || N == 0) return GS_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const DiffusionLayout L = diffusion_layout(B, N, D, C, dt, sm_count());
  if (ws_bytes < L.total) return GS_ERR_WORKSPACE;
  GS_TRY(check_ptr(ws, 1));
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* sv = reinterpret_cast<float*>(wsb + L.off_vals);
  const int64_t n = B * N * C;
  GS_CUDA(launch_diffusion_elementwise(3, s_scale, v, sv, nullptr, n, static_cast<int>(C), 0.f, s));
  Pass p = fwd_pass(x, x, sv, B, N, N, D, C, tau, dt);
  p.w_is_f32 = true;
  GS_TRY(run_pass(p, L.lp, out, wsb, s));                     // K (s V)
  GS_CUDA(launch_diffusion_elementwise(3, s_scale, out, out, nullptr, n, static_cast<int>(C), 0.f,
                                       s));                    // left scaling
  return GS_OK;
}

gs_status gs_test_set_waits(uint64_t limit_ns, int stall) {
  if (limit_ns < 1000 || limit_ns > 10000000000ull || stall < 0 || stall > 2)
    return GS_ERR_INVALID_ARG;
  if (set_test_waits(limit_ns, stall) != cudaSuccess) return GS_ERR_CUDA;
  if (set_test_waits_f32(limit_ns, stall) != cudaSuccess) return GS_ERR_CUDA;
  return GS_OK;
}

gs_status gs_test_read_error_word(int* word, gs_stream_t stream) {
  if (!word) return GS_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GS_ERR_CUDA;
  int v = 0, v32 = 0;
  if (read_and_clear_device_error(&v) != cudaSuccess) return GS_ERR_CUDA;
  if (read_and_clear_device_error_f32(&v32) != cudaSuccess) return GS_ERR_CUDA;
  *word = v | v32;
  return GS_OK;
}

gs_status gs_last_device_error(gs_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GS_ERR_CUDA;
  int v = 0, v32 = 0;
  if (read_and_clear_device_error(&v) != cudaSuccess) return GS_ERR_CUDA;
  if (read_and_clear_device_error_f32(&v32) != cudaSuccess) return GS_ERR_CUDA;
  return (v || v32) ? GS_ERR_TIMEOUT : GS_OK;
}

}  // extern "C"
