// tc_sm100.cu -- tensor-core Gaussian kernel sum for fp16 / bf16 inputs
// (1 <= D <= 128) on sm_100a: tcgen05 MMAs with TMEM accumulators, operands
// staged by TMA, nothing of size M x N ever leaves the SM.
//
// The fold.  With c = tau/2 * log2 e,
//     exp(-tau/2 |x_i - y_j|^2) = 2^(2c (x_i.y_j - |y_j|^2/2) - c |x_i|^2)
// ("Fast Gauss Sums via Flash Attention", Algorithm 1: the two norm factors
// exp(-tau/2 |q|^2) and exp(-tau/2 |k|^2) around a dot-product exponent).
// The column norm is folded into the first MMA by augmenting the operands
// (as Algorithm 2 of the same page augments q and k): x~ = [x, 1, 1, 0..],
// y~ = [y, h, l, 0..] with h + l = -|y|^2/2 split over two fp16 (or bf16)
// values so the augmented product keeps ~22 bits.  Then per pair
//     P_ij = ex2(fma(S~_ij, 2c, r_i)),  S~ = x~ . y~,  r_i = -c |x_i|^2 + 14
// is one FFMA and one MUFU ex2; the +14 (undone on output) keeps P in the
// normal fp16 range down to kernel values of 2^-28.
//
// CTA = 256 rows (two 128-row MMA tiles) x one column split, 10 warps (one
// register-summed channel: 384 rows, three row tiles, 14 warps):
//   warp 0      TMA producer: x~ tiles once, then a ring of (y~, v^T) stages
//   warp 1      TMEM owner + single-thread MMA issuer
//   warps 2-5   exp warpgroup of row tile 0 (TMEM lane quarters 2,3,0,1)
//   warps 6-9   exp warpgroup of row tile 1 (warps 10-13: row tile 2)
// Per 128-column tile t and row tile h:
//   S_h = x~_h . y~(t)^T        (tcgen05.mma, smem x smem -> TMEM fp32)
//   P_h = ex2(fma(S_h, 2c, r))  (tcgen05.ld -> MUFU -> fp16 -> tcgen05.st)
//   O_h += P_h . v(t)           (tcgen05.mma, A = P from TMEM, B = v^T smem)
// The issue order S0(t+1) before O1(t) lets both exp warpgroups run at once.
// One value channel (CP = 1): no P.v MMAs; the exp warps sum P w in registers
// against an fp32 record per column that rides with the stage.
// Forward + backward in one sweep (GW): the exp warps also write P_h to shared
// memory, and the issuer adds Gw_h = P_h^T . g_h (P_h read MN-major, i.e.
// transposed, g_h the rows' upstream gradient as fp16 hi + lo parts), the
// tile's column sums sum_i K_ij g_i, into TMEM; warpgroup h moves Gw_h to a
// per-row-tile partial in global memory at its next tile.  Each kernel value
// is then computed once for the forward sum, the x-gradient sums and dL/dw.
// Every mbarrier wait is bounded (2 s); on expiry the kernel raises the device
// error word and the other warps leave their loops; before TMEM is freed and
// the CTA exits, the producer waits for the loads it issued and the issuer for
// the MMAs it issued (bounded, deaf to the abort), so nothing is in flight.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "values.cuh"

namespace gs {

__device__ int g_device_error;
// The bounded waits' limit, and a stall mode that makes them run out on
// purpose (0: off; 1: the MMA issuer issues nothing; 2: the exp warps do
// nothing): test hooks, set by gs_test_set_waits.
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;
__device__ int g_test_stall;

namespace {

constexpr int kBM = 128;   // rows per MMA tile
constexpr int kBN = 128;   // columns per tile
constexpr int kNT = 2;     // row tiles per CTA (three for one register-summed channel: TcCfg::NT)
constexpr float kPShift = 14.f;
constexpr float kLog2e = 1.4426950408889634f;

struct TcKParams {
  const float* rnorm;   // [B, M]
  float* out;
  int64_t split_stride;
  int64_t M, N;
  int64_t ldo;          // row stride of out (floats)
  int c0, cw;           // first output channel, channels written
  int64_t cols_per_split;
  float two_c;
  float out_scale;
  int s_ksteps;         // K steps of 16 holding the D + 2 nonzero packed columns
  // forward + backward sweep only
  const uint32_t* gpack;   // [B, M] the rows' upstream gradient: fp16 hi | lo << 16, scaled 2^e_b
  const float* gscale;     // [B] 2^-e_b
  float* gw_part;          // [RT, B, N] column sums of each 128-row tile
  int64_t rt_count;        // RT = ceil(M / 128)
};

template <int KP, int CP, bool GW = false>
struct TcCfg {
  static constexpr int KC = KP / 64;            // 128-byte swizzle atoms along K
  static constexpr int ATOM = kBM * 128;        // one 128-row x 64-col block: 16 KB
  // Row tiles per CTA, one exp warpgroup each.  One register-summed value
  // channel with rows of at most two atoms: three (S of three tiles fits TMEM,
  // each y tile serves 384 rows, and a third warp per sub-partition hides more
  // of the exponent chain's latency); else two.
  static constexpr int NT = (CP == 1 && KC <= 2) ? 3 : kNT;
  static constexpr int THREADS = 64 + 128 * NT;
  static constexpr int X_BYTES = NT * KC * ATOM;
  static constexpr int Y_BYTES = KC * ATOM;
  // One value channel (CP == 1) is summed in registers from an fp32 record per
  // column (512 bytes a tile, padded to keep the stages 1024-byte aligned);
  // wider chunks go through the tensor cores from v^T, two 64-column atoms of
  // CP rows.
  static constexpr bool REG = CP == 1;
  static constexpr int V_BYTES = REG ? 1024 : 2 * CP * 128;
  static constexpr int STAGE = Y_BYTES + V_BYTES;
  static constexpr int TX = Y_BYTES + (REG ? kBN * 4 : V_BYTES);   // bytes a stage's TMA loads
  // Forward + backward sweep: P of both row tiles in shared memory as the
  // MN-major operand of P^T . g (per tile: two 64-column atoms of 128 rows x
  // 128 B, 32 KB), and g of both row tiles as its K-major B operand (16 rows
  // x 128 K in two 64-element atoms, 4 KB).
  static constexpr int P_TILE = kBM * kBN * 2;
  static constexpr int G_TILE = 2 * 16 * 128;
  static constexpr int PG_BYTES = GW ? NT * (P_TILE + G_TILE) : 0;
  // 200 KB of operand stages; the three-atom rows (D > 126) may take 220 KB
  static constexpr int BUDGET = (KC > 2 || GW ? 220 : 200) * 1024 - PG_BYTES;
  static constexpr int NST_FIT = (BUDGET - X_BYTES) / STAGE;
  static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
  static constexpr int NBARS = 2 * NST + 2 + 4 * NT;
  static constexpr int SMEM_RAW = 1024 + X_BYTES + NST * STAGE + PG_BYTES + 8 * NBARS + 16;
  // at least ~120 KB so that a second CTA never lands on the SM and blocks on
  // the 512-column TMEM allocation
  static constexpr int SMEM = SMEM_RAW < 122880 ? 122880 : SMEM_RAW;
  // TMEM columns (512 allocated): S0 | S1 | O0 | O1 | P0 | P1.  When the value
  // chunk is wider than 64 the fp16 P tiles overwrite the S tile they came
  // from (the next S MMA is issued after the P MMA that reads it).
  static constexpr bool P_SEPARATE = CP <= 64;
  __host__ __device__ static constexpr uint32_t col_s(int h) { return 128u * h; }
  __host__ __device__ static constexpr uint32_t col_o(int h) {
    return 256u + (P_SEPARATE ? 64u : 128u) * h;
  }
  __host__ __device__ static constexpr uint32_t col_p(int h) {
    return P_SEPARATE ? 384u + 64u * h : 128u * h;
  }
  // Gw_h: 16 columns after O_h's CP (the sweep needs CP <= 48)
  __host__ __device__ static constexpr uint32_t col_g(int h) { return col_o(h) + 48u; }
  static_assert(!GW || (P_SEPARATE && CP >= 16 && CP <= 48 && KC == 1), "forward + backward sweep");
  static_assert(SMEM_RAW <= 227 * 1024, "shared memory per CTA");
  static_assert(NST >= 2, "shared memory budget");
  static_assert(NT == kNT || (CP == 1 && !GW), "three row tiles: register values only (TMEM holds S only)");
  static_assert(CP == 1 || (CP % 16 == 0 && CP >= 16 && CP <= 128), "value chunk");
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++n & 63u) == 0u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(&g_device_error, 1);
        return false;
      }
    }
  }
}

// After an abort: wait for asynchronous work this CTA already started (a TMA
// load's bytes, an MMA commit), bounded but not cut short by the abort flag.
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  uint32_t n = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++n & 63u) == 0u && global_timer_ns() - t0 > limit_ns) {
      atomicOr(&g_device_error, 4);
      return;
    }
  }
}

// Pairs of P columns (out of 16 per 32-column chunk) that take the FMA-pipe
// exp2; the rest use MUFU ex2.  Measured on B200 (d32_c32, d32_c1): once the
// next S tile overlaps the exponentials, 0 beats 2, 3, 4 and 5 -- the exp warps
// are partly latency-bound and the polynomial's longer dependency chain costs
// more than the MUFU slots it frees.  Kept as a tuning knob.
constexpr int kPolyPairs = 0;

// 32 S values of one row -> 16 packed fp16 pairs of P = 2^(2c S + r).
__device__ __forceinline__ void exp_chunk(const uint32_t (&v)[32], uint64_t two_c2, uint64_t r2,
                                          uint32_t (&pk)[16]) {
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const uint64_t s2 = pk2(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1]));
    const uint64_t t2 = fma2(s2, two_c2, r2);
    float t0, t1;
    upk2(t2, t0, t1);
    float e0, e1;
    if (((q * kPolyPairs) & 15) < kPolyPairs) {   // kPolyPairs of the 16 pairs, evenly spread
      // FMA pipe; exponents below -125 would leave the normal range (P is 0 in fp16 there)
      const uint64_t e2 = exp2_poly2<3, false>(pk2(fmaxf(t0, -125.f), fmaxf(t1, -125.f)));
      upk2(e2, e0, e1);
    } else {
      e0 = ex2(t0);
      e1 = ex2(t1);
    }
    pk[q] = pack_f16x2(e0, e1);
  }
}

template <int KP, int CP, int DTFMT, bool GW>
__global__ void __launch_bounds__(TcCfg<KP, CP, GW>::THREADS, 1)
    tc_gauss_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                    const __grid_constant__ CUtensorMap tmV, const TcKParams p) {
  using Cfg = TcCfg<KP, CP, GW>;
  constexpr int NST = Cfg::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sX = smem;
  uint8_t* sStage = smem + Cfg::X_BYTES;
  uint8_t* sP = sStage + NST * Cfg::STAGE;               // GW: P_0 | P_1 (1024-aligned)
  constexpr int NT = Cfg::NT;
  uint8_t* sG = sP + NT * Cfg::P_TILE;                    // GW: g_0 | g_1
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStage + NST * Cfg::STAGE + Cfg::PG_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t bar0 = smem_u32(bars);
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (NST + s); };
  const uint32_t bar_x = bar0 + 8u * (2 * NST);
  auto bar_s = [&](int h) { return bar0 + 8u * (2 * NST + 1 + h); };            // S tile h ready
  auto bar_p = [&](int h) { return bar0 + 8u * (2 * NST + 1 + NT + h); };       // P tile h written
  auto bar_f = [&](int h) { return bar0 + 8u * (2 * NST + 1 + 2 * NT + h); };   // S tile h read out
  auto bar_q = [&](int h) { return bar0 + 8u * (2 * NST + 1 + 3 * NT + h); };   // P tile h consumed
  const uint32_t bar_o = bar0 + 8u * (2 * NST + 1 + 4 * NT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = blockIdx.z;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (NT * kBM);
  const int64_t jbeg = static_cast<int64_t>(blockIdx.y) * p.cols_per_split;
  const int64_t jend = min(p.N, jbeg + p.cols_per_split);
  const int T = (jend > jbeg) ? static_cast<int>((jend - jbeg + kBN - 1) / kBN) : 0;
  const uint64_t wlim = g_wait_limit_ns;
  const int stall = g_test_stall;
  int issued = 0;   // producer lane: column tiles whose loads were issued

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), Cfg::REG ? 4 * NT : 1);   // register values: the exp warps release it
    }
    mbar_init(bar_x, 1);
    for (int h = 0; h < NT; ++h) {
      mbar_init(bar_s(h), 1);
      mbar_init(bar_p(h), 4 * 32);
      mbar_init(bar_f(h), 4 * 32);
      mbar_init(bar_q(h), 1);
    }
    mbar_init(bar_o, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Launched as a programmatic dependent of the packing kernel: the set-up
  // above overlaps its tail; the packed operands are read only after it has
  // completed.  The next kernel (the split combine) may be scheduled now.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmY);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar_x, Cfg::X_BYTES);
      for (int h = 0; h < NT; ++h)
        for (int kc = 0; kc < Cfg::KC; ++kc)
          tma_load_3d(smem_u32(sX + (h * Cfg::KC + kc) * Cfg::ATOM), &tmX, bar_x, kc * 64,
                      static_cast<int>(row0 + h * kBM), static_cast<int>(b));
      for (int t = 0; t < T; ++t) {
        const int st = t % NST;
        if (t >= NST && !wait_bar(bar_empty(st), ((t / NST) - 1) & 1, abort_flag, wlim)) break;
        uint8_t* sy = sStage + st * Cfg::STAGE;
        uint8_t* sv = sy + Cfg::Y_BYTES;
        const int j0 = static_cast<int>(jbeg + static_cast<int64_t>(t) * kBN);
        mbar_arrive_expect_tx(bar_full(st), Cfg::TX);
        for (int kc = 0; kc < Cfg::KC; ++kc)
          tma_load_3d(smem_u32(sy + kc * Cfg::ATOM), &tmY, bar_full(st), kc * 64, j0,
                      static_cast<int>(b));
        if constexpr (Cfg::REG) {
          tma_load_3d(smem_u32(sv), &tmV, bar_full(st), j0, 0, static_cast<int>(b));
        } else {
          for (int hh = 0; hh < 2; ++hh)
            tma_load_3d(smem_u32(sv + hh * CP * 128), &tmV, bar_full(st), j0 + hh * 64, 0,
                        static_cast<int>(b));
        }
        issued = t + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_f16(DTFMT, kBM, kBN);
      const uint32_t idO = idesc_f16(0, kBM, CP);
      const int s_ksteps = p.s_ksteps;
      auto issue_S = [&](int h, int st) {
        const uint8_t* sy = sStage + st * Cfg::STAGE;
#pragma unroll
        for (int ks = 0; ks < KP / 16; ++ks) {
          if (ks >= s_ksteps) break;   // the packed columns past D + 2 are zero
          const int kc = ks >> 2, kw = ks & 3;
          const uint64_t ad = desc_k_sw128(smem_u32(sX + (h * Cfg::KC + kc) * Cfg::ATOM) + kw * 32);
          const uint64_t bd = desc_k_sw128(smem_u32(sy + kc * Cfg::ATOM) + kw * 32);
          mma_ss(tmem + Cfg::col_s(h), ad, bd, idS, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_O = [&](int h, int st, bool acc_prev) {
        const uint8_t* sv = sStage + st * Cfg::STAGE + Cfg::Y_BYTES;
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks) {
          const int kc = ks >> 2, kw = ks & 3;
          const uint64_t bd = desc_k_sw128(smem_u32(sv + kc * CP * 128) + kw * 32);
          mma_ts(tmem + Cfg::col_o(h), tmem + Cfg::col_p(h) + ks * 8, bd, idO,
                 (acc_prev || ks > 0) ? 1u : 0u);
        }
        if constexpr (GW) {
          // Gw_h = P_h^T . g_h: M = the tile's 128 columns, N = 16 (g hi, lo,
          // zeros), K = the 128 rows, 16 per MMA (two 8-row groups of P_h)
          const uint32_t idG = idesc_f16(0, kBM, 16) | kIdescAMajorMN;
          const uint32_t pa = smem_u32(sP + h * Cfg::P_TILE);
          const uint32_t ga = smem_u32(sG + h * Cfg::G_TILE);
#pragma unroll
          for (int ks = 0; ks < kBM / 16; ++ks) {
            const uint64_t ad = desc_mn_sw128(pa + ks * 2048, 64 * 2 * kBM, 1024);
            const uint64_t bd = desc_k_sw128(ga + (ks >> 2) * 2048 + (ks & 3) * 32);
            mma_ss(tmem + Cfg::col_g(h), ad, bd, idG, ks > 0 ? 1u : 0u);
          }
        }
      };
      bool ok = wait_bar(bar_x, 0, abort_flag, wlim) && stall != 1;
      if (ok && T > 0) {
        ok = wait_bar(bar_full(0), 0, abort_flag, wlim);
        if (ok) {
          tc_fence_after();
          for (int h = 0; h < NT; ++h) {
            issue_S(h, 0);
            mma_commit(bar_s(h));
          }
        }
      }
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % NST;
        const int st1 = (t + 1) % NST;
        if constexpr (Cfg::REG) {
          // register values: only the similarity MMAs; S_h(t+1) once warpgroup h
          // has read S_h(t) (the exp warps release the stages themselves)
          if (t + 1 < T) {
            if (!(ok = wait_bar(bar_full(st1), ((t + 1) / NST) & 1, abort_flag, wlim))) break;
            for (int h = 0; ok && h < NT; ++h) {
              if (!(ok = wait_bar(bar_f(h), t & 1, abort_flag, wlim))) break;
              tc_fence_after();
              issue_S(h, st1);
              mma_commit(bar_s(h));
            }
            if (!ok) break;
          }
        } else if constexpr (Cfg::P_SEPARATE) {
          // S_h(t+1) may overwrite S_h as soon as warpgroup h has read S_h(t)
          // into registers: it then runs while the exponentials of tile t are
          // still being computed.
          if (t + 1 < T) {
            if (!(ok = wait_bar(bar_f(0), t & 1, abort_flag, wlim))) break;
            if (!(ok = wait_bar(bar_full(st1), ((t + 1) / NST) & 1, abort_flag, wlim))) break;
            tc_fence_after();
            issue_S(0, st1);
            mma_commit(bar_s(0));
          }
          if (!(ok = wait_bar(bar_p(0), t & 1, abort_flag, wlim))) break;
          tc_fence_after();
          issue_O(0, st, t > 0);
          mma_commit(bar_q(0));
          if (t + 1 < T) {
            if (!(ok = wait_bar(bar_f(1), t & 1, abort_flag, wlim))) break;
            tc_fence_after();
            issue_S(1, st1);
            mma_commit(bar_s(1));
          }
          if (!(ok = wait_bar(bar_p(1), t & 1, abort_flag, wlim))) break;
          tc_fence_after();
          issue_O(1, st, t > 0);
          mma_commit(bar_q(1));
          mma_commit(bar_empty(st));
        } else {
          // P lives in the S columns: the next S MMA must follow the P MMA
          if (!(ok = wait_bar(bar_p(0), t & 1, abort_flag, wlim))) break;
          tc_fence_after();
          issue_O(0, st, t > 0);
          if (t + 1 < T) {
            if (!(ok = wait_bar(bar_full(st1), ((t + 1) / NST) & 1, abort_flag, wlim))) break;
            tc_fence_after();
            issue_S(0, st1);
            mma_commit(bar_s(0));
          }
          if (!(ok = wait_bar(bar_p(1), t & 1, abort_flag, wlim))) break;
          tc_fence_after();
          issue_O(1, st, t > 0);
          mma_commit(bar_empty(st));
          if (t + 1 < T) {
            issue_S(1, st1);
            mma_commit(bar_s(1));
          }
        }
      }
      // the drain point for whatever was issued (register values: the exp
      // warps wait for every S MMA themselves; only an abort waits on it)
      mma_commit(bar_o);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ exp warpgroups
    const int h = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int64_t i = row0 + h * kBM + row;
    const bool valid = i < p.M;
    const float r = valid ? p.rnorm[b * p.M + i] : 0.f;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + Cfg::col_s(h);
    const uint32_t tP = tmem + lane_base + Cfg::col_p(h);
    const uint32_t tO = tmem + lane_base + Cfg::col_o(h);
    const float two_c = p.two_c;
    bool ok = true;
    const uint64_t two_c2 = pk2(two_c, two_c);
    const uint64_t r2 = pk2(r, r);
    float row_sum = 0.f;   // register values: the row's sum over the tiles
    // Forward + backward sweep.  TMEM lane `row` of Gw_h is column j0 + row of
    // the tile; row tile rt of the matrix.
    const int64_t rt = static_cast<int64_t>(blockIdx.x) * NT + h;
    uint8_t* const sPh = sP + h * Cfg::P_TILE;
    if constexpr (GW) {
      // this row's (g hi, g lo) as column `row` of g_h: rows 0 and 1 of the
      // 16-row K-major operand, rows 2..15 zero
      const uint32_t gv = valid ? p.gpack[b * p.M + i] : 0u;
      uint8_t* gh = sG + h * Cfg::G_TILE + (row >> 6) * 2048;
      const int kin = row & 63;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const uint16_t v = n == 0 ? static_cast<uint16_t>(gv & 0xffffu)
                                  : (n == 1 ? static_cast<uint16_t>(gv >> 16) : uint16_t(0));
        *reinterpret_cast<uint16_t*>(gh + n * 128 + ((((kin >> 3) ^ (n & 7)) << 4) | ((kin & 7) << 1))) = v;
      }
      fence_proxy_async_smem();
    }
    // P columns [32 c, 32 c + 32) of this row into P_h: row `row` of 8-row
    // group row / 8, 64-column atom c / 2, 16-byte pieces swizzled by row % 8
    auto store_p = [&](int c, const uint32_t(&pk)[16]) {
      uint8_t* base = sPh + (c >> 1) * (64 * 2 * kBM) + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int piece = (((c & 1) << 2) + q) ^ (row & 7);
        *reinterpret_cast<uint4*>(base + piece * 16) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
    };
    // Gw_h of column tile tt (complete: its MMAs were waited for) to the
    // row tile's partial; also completes any TMEM load still in flight
    const float gsc = GW ? p.gscale[b] * p.out_scale : 0.f;
    auto drain_gw = [&](int tt) {
      uint32_t gq[2];
      tmem_ld2(tmem + lane_base + Cfg::col_g(h), gq);
      tmem_wait_ld();
      asm volatile("" : "+r"(gq[0]), "+r"(gq[1]));
      const int64_t j = jbeg + static_cast<int64_t>(tt) * kBN + row;
      if (rt < p.rt_count && j < jend)
        p.gw_part[(rt * gridDim.z + b) * p.N + j] =
            (__uint_as_float(gq[0]) + __uint_as_float(gq[1])) * gsc;
    };
    if (stall == 2) {   // test hook: wait on a barrier nobody arrives on, until the limit
      wait_bar(bar_p(h), 0, abort_flag, wlim);
      ok = false;
    }
    for (int t = 0; ok && t < T; ++t) {
      ok = wait_bar(bar_s(h), t & 1, abort_flag, wlim);
      // register values read the stage's records themselves: its loads landed
      if (Cfg::REG && ok) ok = wait_bar(bar_full(t % NST), (t / NST) & 1, abort_flag, wlim);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // TMEM loads run up to three chunks of 32 columns deep: chunks 0 and 1
      // first, chunk 2 while chunk 0 is exponentiated, chunk 3 while chunk 1
      // is.  After chunk 1 the whole S tile is in registers and its columns
      // are released, so the next S MMA has the second half of this tile's
      // exponentials to complete in.
      static_assert(kBN == 128, "four 32-column chunks per tile");
      uint32_t va[32], vb[32], vc[32];
      uint32_t pk[16];
      tmem_ld32(tS, va);
      tmem_ld32(tS + 32, vb);
      tmem_wait_ld();
      reg_fence32(va);
      reg_fence32(vb);
      tmem_ld32(tS + 64, vc);
      if constexpr (Cfg::REG) {
        // one value channel: P w summed in registers (fp32 P, exact products),
        // two columns per packed operation, a partial per tile
        const float* wr =
            reinterpret_cast<const float*>(sStage + (t % NST) * Cfg::STAGE + Cfg::Y_BYTES);
        uint64_t acc2 = 0ull;
        auto reg_chunk = [&](const uint32_t(&v)[32], const float* w) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 w4 = *reinterpret_cast<const float4*>(w + 4 * e4);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              float t0, t1;
              upk2(fma2(pk2(__uint_as_float(v[4 * e4 + 2 * hh]),
                            __uint_as_float(v[4 * e4 + 2 * hh + 1])),
                        two_c2, r2),
                   t0, t1);
              acc2 = fma2(pk2(ex2(t0), ex2(t1)), hh ? pk2(w4.z, w4.w) : pk2(w4.x, w4.y), acc2);
            }
          }
        };
        reg_chunk(va, wr);
        tmem_ld32(tS + 96, va);
        reg_chunk(vb, wr + 32);
        tmem_wait_ld();
        reg_fence32(vc);
        reg_fence32(va);
        tc_fence_before();
        mbar_arrive(bar_f(h));
        reg_chunk(vc, wr + 64);
        reg_chunk(va, wr + 96);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(t % NST));   // this warp is done with the records
        float lo, hi;
        upk2(acc2, lo, hi);
        row_sum += lo + hi;
      } else {
        exp_chunk(va, two_c2, r2, pk);
        if (Cfg::P_SEPARATE && t > 0) {
          // a warp that runs ahead must not overwrite its rows of P(t-1) before
          // the P MMA of tile t-1 has read them (waited for as late as possible)
          ok = __all_sync(0xffffffffu, wait_bar(bar_q(h), (t - 1) & 1, abort_flag, wlim));
          if (!ok) {
            tmem_wait_ld();   // chunk 2's load may still be in flight
            break;
          }
          tc_fence_after();
          if constexpr (GW) drain_gw(t - 1);
        }
        tmem_st16(tP, pk);
        if constexpr (GW) store_p(0, pk);
        tmem_ld32(tS + 96, va);
        exp_chunk(vb, two_c2, r2, pk);
        tmem_st16(tP + 16, pk);
        if constexpr (GW) store_p(1, pk);
        tmem_wait_ld();
        reg_fence32(vc);
        reg_fence32(va);
        tc_fence_before();
        mbar_arrive(bar_f(h));
        exp_chunk(vc, two_c2, r2, pk);
        tmem_st16(tP + 32, pk);
        if constexpr (GW) store_p(2, pk);
        exp_chunk(va, two_c2, r2, pk);
        tmem_st16(tP + 48, pk);
        if constexpr (GW) store_p(3, pk);
        tmem_wait_st();
        if constexpr (GW) fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_p(h));
      }
    }
    if constexpr (Cfg::REG) {
      ok = __all_sync(0xffffffffu, ok);
      if (ok && valid && !*abort_flag) {
        float* orow = p.out + static_cast<int64_t>(blockIdx.y) * p.split_stride +
                      (b * p.M + i) * p.ldo + p.c0;
        orow[0] = (T > 0) ? row_sum * p.out_scale : 0.f;
      }
    } else {
      if (ok) ok = wait_bar(bar_o, 0, abort_flag, wlim);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if constexpr (GW) {
        if (ok && T > 0) drain_gw(T - 1);
      }
      if (ok) {
        float* orow = p.out + static_cast<int64_t>(blockIdx.y) * p.split_stride +
                      (b * p.M + i) * p.ldo + p.c0;
#pragma unroll
        for (int ch = 0; ch < CP / 16; ++ch) {
          uint32_t v[16];
          tmem_ld16(tO + ch * 16, v);
          tmem_wait_ld();
          reg_fence16(v);
          if (valid) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int c = ch * 16 + q;
              if (c < p.cw) orow[c] = (T > 0) ? __uint_as_float(v[q]) * p.out_scale : 0.f;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // Every warp has left its loop.  The loads and MMAs already issued must land
  // before the shared memory and TMEM they write are given up: after an abort
  // some were never waited for (in a normal run these waits return at once).
  if (warp == 0 && lane == 0) {
    for (int t = issued > NST ? issued - NST : 0; t < issued; ++t)
      drain_bar(bar_full(t % NST), (t / NST) & 1, wlim);
    drain_bar(bar_x, 0, wlim);
  }
  if (warp == 1 && lane == 0) drain_bar(bar_o, 0, wlim);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ packing prologue
template <typename T>
__device__ __forceinline__ float tof(T v);
template <>
__device__ __forceinline__ float tof<float>(float v) { return v; }
template <>
__device__ __forceinline__ float tof<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float tof<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T fromf(float v);
template <>
__device__ __forceinline__ __half fromf<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 fromf<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ uint16_t bits16(__half v) { return __half_as_ushort(v); }
__device__ __forceinline__ uint16_t bits16(__nv_bfloat16 v) { return __bfloat16_as_ushort(v); }

// Packed operand rows.  Row side (is_x): [x, 1, 1, 0 ...] and
// rnorm = -c |x|^2 + shift.  Column side: [y, h, l, 0 ...] with h + l = -|y|^2/2.
// Both sides in one launch: blocks below `blocks_x` pack the rows, the rest the
// columns.  A group of 8 consecutive threads builds one row, KP/8 elements
// each, written as 8-element (16-byte) pieces: thread `part` owns pieces part,
// part + 8, ...
template <typename T, int KP>
__global__ void pack_rows_kernel(const T* __restrict__ src_x, T* __restrict__ dst_x,
                                 float* __restrict__ rnorm, int64_t rows_x,
                                 const T* __restrict__ src_y, T* __restrict__ dst_y,
                                 int64_t rows_y, int64_t blocks_x, int D, float c, float shift) {
  constexpr int G = 8;          // threads per row
  constexpr int NPC = KP / 64;  // pieces per thread (1, 2 or 3)
  const bool is_x = blockIdx.x < blocks_x;
  const T* __restrict__ src = is_x ? src_x : src_y;
  T* __restrict__ dst = is_x ? dst_x : dst_y;
  const int64_t rows = is_x ? rows_x : rows_y;
  const int64_t blk = is_x ? static_cast<int64_t>(blockIdx.x) : blockIdx.x - blocks_x;
  const int64_t gt = blk * blockDim.x + threadIdx.x;
  const int64_t row = gt / G;
  const int part = static_cast<int>(gt % G);
  const bool live = row < rows;
  float vals[NPC][8];
  float sq = 0.f;
#pragma unroll
  for (int pc = 0; pc < NPC; ++pc)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = (part + pc * G) * 8 + e;
      float v = 0.f;
      if (live && k < D) v = tof(src[row * D + k]);
      vals[pc][e] = v;
      sq = fmaf(v, v, sq);
    }
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o, G);
  if (!live) return;
  float aug0, aug1;
  if (is_x) {
    aug0 = 1.f;
    aug1 = 1.f;
  } else {
    const float hn = -0.5f * sq;
    aug0 = tof(fromf<T>(hn));
    aug1 = hn - aug0;
  }
#pragma unroll
  for (int pc = 0; pc < NPC; ++pc) {
    uint32_t packed[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float v0 = vals[pc][e], v1 = vals[pc][e + 1];
      const int k = (part + pc * G) * 8 + e;
      if (k == D) v0 = aug0;
      if (k == D + 1) v0 = aug1;
      if (k + 1 == D) v1 = aug0;
      if (k + 1 == D + 1) v1 = aug1;
      packed[e / 2] = static_cast<uint32_t>(bits16(fromf<T>(v0))) |
                      (static_cast<uint32_t>(bits16(fromf<T>(v1))) << 16);
    }
    *reinterpret_cast<uint4*>(dst + row * KP + (part + pc * G) * 8) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
  if (is_x && part == 0) rnorm[row] = fmaf(-c, sq, shift);
}

// Transposed fp16 value matrix v^T [B, CP, Nst] for channels [c0, c0 + CP) of
// the pass's value matrix (values.cuh; columns = the y side of this pass,
// centre = its first row point).  Channels past CV are written as zeros.
// One thread per column (b, j) and group of kPackGroup channels (blockIdx.y):
// consecutive threads take consecutive j, so each channel's store is
// coalesced, and a thread reads its column's point and weights once for the
// channels of its group.
constexpr int kPackGroup = 16;

template <typename TW, typename TY>
__global__ void pack_values_kernel(const TW* __restrict__ w, const TY* __restrict__ y,
                                   const TY* __restrict__ rows, __half* __restrict__ vt, int64_t B,
                                   int64_t N, int64_t Nst, int64_t Mrows, int C, int D, int CV,
                                   int c0, int CP) {
  asm volatile("griddepcontrol.launch_dependents;");   // the sweep may set up meanwhile
  const int64_t total = B * N;
  const int g0 = blockIdx.y * kPackGroup;
  const int g1 = min(CP, g0 + kPackGroup);
  for (int64_t bj = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; bj < total;
       bj += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = bj / N, j = bj - b * N;
    __half* dst = vt + b * CP * Nst + j;
    for (int cc = g0; cc < g1; ++cc) {
      const int ch = c0 + cc;
      const float v = (ch < CV) ? value_at(w, y, rows, b, bj, Mrows, D, C, ch, C) : 0.f;
      dst[cc * Nst] = __float2half_rn(v);
    }
  }
}

// One value channel (CV == 1): its fp32 values rec [B, Nw] (zeros past N), the
// per-column records the register-value kernel sums against.
template <typename TW, typename TY>
__global__ void pack_records_kernel(const TW* __restrict__ w, const TY* __restrict__ y,
                                    const TY* __restrict__ rows, float* __restrict__ rec, int64_t B,
                                    int64_t N, int64_t Nw, int64_t Mrows, int C, int D) {
  asm volatile("griddepcontrol.launch_dependents;");   // the sweep may set up meanwhile
  const int64_t total = B * Nw;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / Nw, j = e % Nw;
    rec[e] = (j < N) ? value_at(w, y, rows, b, b * N + j, Mrows, D, C, 0, C) : 0.f;
  }
}

// The rows' upstream gradient g[b, :, 0] for the forward + backward sweep, as
// fp16 hi + lo parts of g 2^e_b (~22 significant bits together), e_b per batch
// putting the batch's largest |g 2^e_b| in [2^13, 2^14): hi = fp16(g 2^e),
// lo = fp16(g 2^e - hi), gpack = hi | lo << 16, gscale[b] = 2^-e_b.  Two
// launches over (128-row tile, batch) blocks: the tiles' largest |g|, then
// each block reduces its batch's tile maxima and packs its tile.
__global__ void __launch_bounds__(128) g_tile_max_kernel(const float* __restrict__ g, int64_t ldg,
                                                         float* __restrict__ tmax, int64_t M,
                                                         int64_t RT) {
  __shared__ float red[4];
  const int64_t rt = blockIdx.x, b = blockIdx.y;
  const int64_t i = rt * 128 + threadIdx.x;
  float mx = i < M ? fabsf(g[(b * M + i) * ldg]) : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) tmax[b * RT + rt] = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

__global__ void __launch_bounds__(128) pack_g_kernel(const float* __restrict__ g, int64_t ldg,
                                                     const float* __restrict__ tmax,
                                                     uint32_t* __restrict__ gpack,
                                                     float* __restrict__ gscale, int64_t M,
                                                     int64_t RT) {
  __shared__ float red[4];
  const int64_t rt = blockIdx.x, b = blockIdx.y;
  float mx = 0.f;
  for (int64_t t = threadIdx.x; t < RT; t += 128) mx = fmaxf(mx, tmax[b * RT + t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  int e = 0;   // from the exponent bits; within [-126, 126]
  if (mx > 0.f) e = 13 - (((__float_as_int(mx) >> 23) & 0xff) - 127);
  e = e > 126 ? 126 : (e < -126 ? -126 : e);
  const int64_t i = rt * 128 + threadIdx.x;
  if (i < M) {
    const float v = g[(b * M + i) * ldg] * __int_as_float((e + 127) << 23);
    const __half hi = __float2half_rn(v);
    const __half lo = __float2half_rn(v - __half2float(hi));
    gpack[b * M + i] = static_cast<uint32_t>(__half_as_ushort(hi)) |
                       (static_cast<uint32_t>(__half_as_ushort(lo)) << 16);
  }
  if (rt == 0 && threadIdx.x == 0) gscale[b] = __int_as_float((127 - e) << 23);
}

// ------------------------------------------------------------------ host side
int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148 * 32) b = 148 * 32;
  return static_cast<int>(b);
}

template <typename T>
cudaError_t pack_operands(const TcArgs& a, cudaStream_t s) {
  const float c = 0.5f * a.tau * kLog2e;
  const int KP = a.plan.KP;
  const int64_t rows_x = a.B * a.M, rows_y = a.B * a.N;
  const int64_t blocks_x = (rows_x * 8 + 255) / 256, blocks_y = (rows_y * 8 + 255) / 256;
  if (blocks_x + blocks_y > 0x7fffffff) return cudaErrorInvalidValue;
  const unsigned blocks = static_cast<unsigned>(blocks_x + blocks_y);
  const T* xs = static_cast<const T*>(a.x);
  const T* ys = static_cast<const T*>(a.y);
  T* xd = static_cast<T*>(a.xpack);
  T* yd = static_cast<T*>(a.ypack);
  if (KP == 64)
    pack_rows_kernel<T, 64><<<blocks, 256, 0, s>>>(xs, xd, a.rnorm, rows_x, ys, yd, rows_y, blocks_x,
                                                   a.D, c, kPShift);
  else if (KP == 128)
    pack_rows_kernel<T, 128><<<blocks, 256, 0, s>>>(xs, xd, a.rnorm, rows_x, ys, yd, rows_y, blocks_x,
                                                    a.D, c, kPShift);
  else
    pack_rows_kernel<T, 192><<<blocks, 256, 0, s>>>(xs, xd, a.rnorm, rows_x, ys, yd, rows_y, blocks_x,
                                                    a.D, c, kPShift);
  return cudaGetLastError();
}

template <typename T>
cudaError_t pack_records(const TcArgs& a, int64_t Nw, cudaStream_t s) {
  const int blocks = grid_for(a.B * Nw, 256);
  const T* y = static_cast<const T*>(a.y);
  const T* rows = static_cast<const T*>(a.x);
  float* rec = static_cast<float*>(a.vt);
  if (a.w_is_f32)
    pack_records_kernel<float, T><<<blocks, 256, 0, s>>>(static_cast<const float*>(a.w), y, rows, rec,
                                                         a.B, a.N, Nw, a.M, a.C, a.D);
  else
    pack_records_kernel<T, T><<<blocks, 256, 0, s>>>(static_cast<const T*>(a.w), y, rows, rec, a.B,
                                                     a.N, Nw, a.M, a.C, a.D);
  return cudaGetLastError();
}

template <typename T>
cudaError_t pack_values(const TcArgs& a, int c0, int CP, int64_t Nst, cudaStream_t s) {
  const dim3 blocks(grid_for(a.B * a.N, 128), (CP + kPackGroup - 1) / kPackGroup);
  const T* y = static_cast<const T*>(a.y);
  const T* rows = static_cast<const T*>(a.x);
  if (a.w_is_f32)
    pack_values_kernel<float, T><<<blocks, 128, 0, s>>>(static_cast<const float*>(a.w), y, rows,
                                                        static_cast<__half*>(a.vt), a.B, a.N, Nst,
                                                        a.M, a.C, a.D, a.CV, c0, CP);
  else
    pack_values_kernel<T, T><<<blocks, 128, 0, s>>>(static_cast<const T*>(a.w), y, rows,
                                                    static_cast<__half*>(a.vt), a.B, a.N, Nst, a.M,
                                                    a.C, a.D, a.CV, c0, CP);
  return cudaGetLastError();
}

template <int KP, int CP, int DTFMT, bool GW = false>
cudaError_t launch_kernel(const CUtensorMap& tx, const CUtensorMap& ty, const CUtensorMap& tv,
                          const TcKParams& kp, dim3 grid, cudaStream_t s) {
  using Cfg = TcCfg<KP, CP, GW>;
  auto fn = tc_gauss_kernel<KP, CP, DTFMT, GW>;
  static bool attr_done = false;   // idempotent; a benign race at worst repeats the call
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg{};
  // row blocks of Cfg::NT row tiles
  cfg.gridDim = dim3(static_cast<unsigned>((kp.M + Cfg::NT * kBM - 1) / (Cfg::NT * kBM)), grid.y, grid.z);
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, tx, ty, tv, kp);
}

// The forward + backward sweep: 64-wide packed rows, one chunk of 16, 32 or 48
// value channels.
template <int DTFMT>
cudaError_t launch_gw(int CP, const CUtensorMap& tx, const CUtensorMap& ty, const CUtensorMap& tv,
                      const TcKParams& kp, dim3 grid, cudaStream_t s) {
  switch (CP) {
    case 16: return launch_kernel<64, 16, DTFMT, true>(tx, ty, tv, kp, grid, s);
    case 32: return launch_kernel<64, 32, DTFMT, true>(tx, ty, tv, kp, grid, s);
    case 48: return launch_kernel<64, 48, DTFMT, true>(tx, ty, tv, kp, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int KP, int DTFMT>
cudaError_t launch_cp(int CP, const CUtensorMap& tx, const CUtensorMap& ty, const CUtensorMap& tv,
                      const TcKParams& kp, dim3 grid, cudaStream_t s) {
  if constexpr (KP > 128) {
    // three-atom rows: value chunks of at most 48 channels fit two stages
    switch (CP) {
      case 1: return launch_kernel<KP, 1, DTFMT>(tx, ty, tv, kp, grid, s);
      case 16: return launch_kernel<KP, 16, DTFMT>(tx, ty, tv, kp, grid, s);
      case 32: return launch_kernel<KP, 32, DTFMT>(tx, ty, tv, kp, grid, s);
      default: return launch_kernel<KP, 48, DTFMT>(tx, ty, tv, kp, grid, s);
    }
  } else {
    switch (CP) {
      case 1: return launch_kernel<KP, 1, DTFMT>(tx, ty, tv, kp, grid, s);
      case 16: return launch_kernel<KP, 16, DTFMT>(tx, ty, tv, kp, grid, s);
      case 32: return launch_kernel<KP, 32, DTFMT>(tx, ty, tv, kp, grid, s);
      case 48: return launch_kernel<KP, 48, DTFMT>(tx, ty, tv, kp, grid, s);
      case 64: return launch_kernel<KP, 64, DTFMT>(tx, ty, tv, kp, grid, s);
      case 96: return launch_kernel<KP, 96, DTFMT>(tx, ty, tv, kp, grid, s);
      default: return launch_kernel<KP, 128, DTFMT>(tx, ty, tv, kp, grid, s);
    }
  }
}

}  // namespace

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  });
  return fn;
}

bool make_tmap_3d(CUtensorMap* m, CUtensorMapDataType dt, void* base, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0,
                  uint32_t box1, bool swizzle128) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int tc_max_chunk(int KP) { return KP > 128 ? 48 : kTcMaxChunk; }

int tc_chunk_pad(int cw) {
  const int c16 = (cw + 15) / 16 * 16;
  if (c16 <= 64) return c16 == 0 ? 16 : c16;
  return c16 <= 96 ? 96 : 128;
}

TcPlan tc_plan(int64_t B, int64_t M, int64_t N, int64_t D, int sm_count) {
  TcPlan p{};
  p.KP = (D + 2 <= 64) ? 64 : ((D + 2 <= 128) ? 128 : 192);
  const int64_t U = B * ((M + kNT * kBM - 1) / (kNT * kBM));
  const int64_t ntj = (N + kBN - 1) / kBN;
  int64_t smax = ntj / 4;
  if (smax > 32) smax = 32;
  if (smax < 1) smax = 1;
  int best = 1;
  double best_cost = 1e300;
  for (int64_t S = 1; S <= smax; ++S) {
    const int64_t waves = (U * S + sm_count - 1) / sm_count;
    const double cost = static_cast<double>(waves) * static_cast<double>((ntj + S - 1) / S + 3);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = static_cast<int>(S);
    }
  }
  const int64_t tiles_per_split = (ntj + best - 1) / best;
  p.cols_per_split = (tiles_per_split < 1 ? 1 : tiles_per_split) * kBN;
  p.splits = static_cast<int>((N + p.cols_per_split - 1) / p.cols_per_split);
  if (p.splits < 1) p.splits = 1;
  return p;
}

cudaError_t launch_tc_sum(const TcArgs& a, cudaStream_t s) {
  if (a.B == 0 || a.M == 0) return cudaSuccess;
  const bool bf = a.dt == GS_BF16;
  cudaError_t e = bf ? pack_operands<__nv_bfloat16>(a, s) : pack_operands<__half>(a, s);
  if (e != cudaSuccess) return e;
  const int KP = a.plan.KP;
  const CUtensorMapDataType tdt = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tx, ty;
  if (!make_tmap_3d(&tx, tdt, a.xpack, KP, a.M, a.B, KP * 2ull, a.M * KP * 2ull, 64, kBM) ||
      !make_tmap_3d(&ty, tdt, a.ypack, KP, a.N, a.B, KP * 2ull, a.N * KP * 2ull, 64, kBN))
    return cudaErrorInvalidValue;
  const int64_t Nst = (a.N + 7) / 8 * 8;
  // (launch_kernel sets the row-block count from the instantiation's row tiles per CTA)
  const dim3 grid(static_cast<unsigned>((a.M + kNT * kBM - 1) / (kNT * kBM)),
                  static_cast<unsigned>(a.plan.splits), static_cast<unsigned>(a.B));
  const int chunk = tc_max_chunk(KP);
  const bool gw = a.gw_part != nullptr;
  if (gw) {
    // one fused sweep: the values in a single chunk of at most 48 channels
    const int64_t RT = (a.M + kBM - 1) / kBM;
    if (KP != 64 || a.CV > 48 || a.CV < 2 || a.B > 65535 || RT > 0x7fffffff)
      return cudaErrorInvalidValue;
    const dim3 gg(static_cast<unsigned>(RT), static_cast<unsigned>(a.B));
    g_tile_max_kernel<<<gg, 128, 0, s>>>(a.g, a.g_ld, a.gtmax, a.M, RT);
    pack_g_kernel<<<gg, 128, 0, s>>>(a.g, a.g_ld, a.gtmax, a.gpack, a.gscale, a.M, RT);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  for (int c0 = 0; c0 < a.CV; c0 += chunk) {
    const int cw = (a.CV - c0) < chunk ? (a.CV - c0) : chunk;
    // one value channel: fp32 records summed in registers (CP = 1)
    const bool reg1 = a.CV == 1;
    const int CP = reg1 ? 1 : tc_chunk_pad(cw);
    CUtensorMap tv;
    if (reg1) {
      const int64_t Nw = (a.N + 3) / 4 * 4;
      e = bf ? pack_records<__nv_bfloat16>(a, Nw, s) : pack_records<__half>(a, Nw, s);
      if (e != cudaSuccess) return e;
      if (!make_tmap_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.vt, Nw, 1, a.B, Nw * 4ull, Nw * 4ull,
                        kBN, 1, false))
        return cudaErrorInvalidValue;
    } else {
      e = bf ? pack_values<__nv_bfloat16>(a, c0, CP, Nst, s) : pack_values<__half>(a, c0, CP, Nst, s);
      if (e != cudaSuccess) return e;
      if (!make_tmap_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.vt, a.N, CP, a.B, Nst * 2ull,
                        CP * Nst * 2ull, 64, CP))
        return cudaErrorInvalidValue;
    }
    TcKParams kp{};
    kp.rnorm = a.rnorm;
    kp.out = a.out;
    kp.split_stride = a.split_stride;
    kp.M = a.M;
    kp.N = a.N;
    kp.ldo = a.CV;
    kp.c0 = c0;
    kp.cw = cw;
    kp.cols_per_split = a.plan.cols_per_split;
    kp.two_c = a.tau * kLog2e;
    kp.out_scale = exp2f(-kPShift);
    kp.s_ksteps = static_cast<int>((a.D + 2 + 15) / 16);
    if (gw) {
      kp.gpack = a.gpack;
      kp.gscale = a.gscale;
      kp.gw_part = a.gw_part;
      kp.rt_count = (a.M + kBM - 1) / kBM;
      e = bf ? launch_gw<1>(CP, tx, ty, tv, kp, grid, s) : launch_gw<0>(CP, tx, ty, tv, kp, grid, s);
      if (e != cudaSuccess) return e;
      continue;
    }
    if (KP == 64)
      e = bf ? launch_cp<64, 1>(CP, tx, ty, tv, kp, grid, s) : launch_cp<64, 0>(CP, tx, ty, tv, kp, grid, s);
    else if (KP == 128)
      e = bf ? launch_cp<128, 1>(CP, tx, ty, tv, kp, grid, s) : launch_cp<128, 0>(CP, tx, ty, tv, kp, grid, s);
    else
      e = bf ? launch_cp<192, 1>(CP, tx, ty, tv, kp, grid, s) : launch_cp<192, 0>(CP, tx, ty, tv, kp, grid, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t set_test_waits(uint64_t limit_ns, int stall) {
  const unsigned long long l = limit_ns;
  cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns, &l, sizeof(l));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_test_stall, &stall, sizeof(int));
  return e;
}

cudaError_t read_and_clear_device_error(int* value) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  *value = v;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  }
  return e;
}

}  // namespace gs
