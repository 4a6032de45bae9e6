// tc_f32_sm100.cu -- tensor-core Gaussian kernel sum for fp32 inputs with
// 9 <= D <= 128 on sm_100a, at fp32 accuracy: split products on tcgen05.
//
// Each fp32 operand v is split into v = hi + lo, two values of 11 significant
// bits each, and a product a b is taken as a_lo b_hi + a_hi b_lo + a_hi b_hi:
// the dropped a_lo b_lo is ~2^-22 of a b, so three MMAs give close to fp32
// products with fp32 accumulation.  This is the "memory-efficient" fp32 runs'
// arithmetic of "Fast Gauss Sums via Flash Attention" (Figures 4 and 5), done
// with B200's tensor cores.  The similarity tile x.y^T splits into fp16 parts
// (kind::f16, 16 per K step: half the MMAs of tf32 parts, which carry the same
// 11 bits), the coordinates scaled by a power of two per batch so that fp16's
// range holds them (split_exp); the value product P.v on the tensor cores
// splits P 2^14 and v 2^e (e per batch and channel) into fp16 parts as well.
//
// The exponent.  With c = tau/2 * log2 e and the points centred at z, the mean
// of a strided sample of the batch's column points (x' = x - z, y' = y - z:
// every |x - y| is unchanged, and the norms stay at the scale of the cloud of
// columns, so the expanded form below loses little to cancellation for the
// rows near them),
//     exp(-tau/2 |x_i - y_j|^2) = 2^(2c x'_i.y'_j + r_i + q_j),
//     r_i = -c |x'_i|^2,  q_j = -c |y'_j|^2
// (the norm factors of Algorithm 1 on the same page).  P_ij = ex2(fma(S, 2c, r_i) + q_j)
// with S from the split MMAs; P is split into fp16 hi/lo parts again for P.v.
//
// CTA = one 128-row tile, 2 + 4 NWG warps:
//   warp 0      TMA producer: the x' rows once (unless they sit in TMEM), then a
//               ring of stages: y' tile, the column records lane by lane (q_j,
//               then values or log2 values), and for tensor-core values the
//               split v^T tile
//   warp 1      TMEM owner + single-thread MMA issuer
//   warps 2..   NWG exp warpgroups (three with register values, two with
//               tensor-core values); warpgroup h takes column tiles h, h + NWG, ...
// The warpgroups hold the same rows (TMEM lanes), so each keeps its own
// partial result and warpgroup 0 combines them at the end.  Per column tile
// t of warpgroup h:
//   S_h  = x'.y'(t)^T                 3 fp16 MMAs per K step of 16 into one
//                                     accumulator (A from TMEM when it has room,
//                                     else from shared memory)
//   P_h  = ex2(fma(S_h, 2c, r) + q)   tcgen05.ld -> MUFU
// then either (register values, <= 3 channels, and the log-sum-exp)
//   row sums += P_h . v in registers, exact fp32 FMAs (or a running maximum and
//   shifted sum for the log-sum-exp)
// or (tensor-core values, 4 .. 64 channels per pass)
//   P_h 2^14 -> fp16 hi/lo -> tcgen05.st;  O_h += P_h . v(t), 3 fp16 MMAs per
//   K step of 16 (A = P from TMEM); the scales are undone on output.
// fp16 / bf16 inputs (log-sum-exp) are exact in their own format: unsplit
// rows of the input values, one kind::f16 MMA (fp16 or bf16 encoding) per K
// step of 16 (template SPLIT = false).
// Every mbarrier wait is bounded (2 s); on expiry the kernel raises its device
// error word, lets the other warps leave, frees TMEM and returns.
#include <cuda.h>

#include <cmath>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"
#include "values.cuh"

namespace gs {

__device__ int g_device_error_f32;
// The bounded waits' limit, and a stall mode that makes them run out on
// purpose (0: off; 1: the MMA issuer issues nothing; 2: the exp warps do
// nothing): test hooks, set by gs_test_set_waits.
__device__ unsigned long long g_wait_limit_ns_f32 = 2000000000ull;
__device__ int g_test_stall_f32;

namespace {

constexpr int kBM = 128;        // rows per CTA (one MMA tile)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kAtom = kBM * 128;   // one 128-row x 32-float (128-byte) swizzle atom

struct F32KParams {
  const float* xpack;   // [B, M, 2 K'] packed rows (copied into TMEM when it has room)
  const float* rnorm;   // [B, M]
  float* out;           // sums; log-sum-exp: the shifts m (log2 units)
  float* out_l;         // log-sum-exp: the scaled sums l (sum = 2^m l)
  int64_t split_stride;
  int64_t M, N;
  int64_t ldo;
  int c0, cw;
  int64_t cols_per_split;
  int ksteps;           // K'/16: 32-byte K steps of the hi (and of the lo) half
  int atoms;            // 128-byte atoms of a packed row actually loaded (<= KA)
  int Bsz;              // batch count (the lo half of v sits at batch index B + b)
  int bn;               // tile width the TMA boxes were made for
  int split;            // 1: fp16 rows [hi | lo]; 0: rows are the fp16 / bf16 inputs themselves
  int afmt;             // unsplit rows: 0 fp16, 1 bf16 (the MMA's operand encoding)
  float two_c;
  const int* amax;      // split rows: per batch, the bits of max |v'| (sets the power-of-two scale)
  const int* vmax;      // tensor-core values: per (batch, channel of the chunk), the bits of max |v|
};

// KA: 128-byte atoms per packed row [hi K' | lo K'] the operands may hold.
// MODE 1 or 3: the values (at most MODE channels) ride with the column norms
// and P.v is summed in registers (exact fp32 products); MODE 16, 32 or 64:
// P.v on the tensor cores for a chunk of MODE channels.
template <int KA, int MODE>
struct F32Cfg {
  static constexpr bool REG = MODE <= 3;
  // exp warpgroups, each taking every NWG-th column tile of the CTA's rows.
  // Register values: three (S of all three fits TMEM, and a third warp per
  // sub-partition hides more of the exponent chain's latency); tensor-core
  // values: two (S, P and O per warpgroup).  Plus a producer and an MMA warp.
  static constexpr int NWG = REG ? 3 : 2;
  static constexpr int THREADS = 64 + 128 * NWG;
  static constexpr int CP = REG ? 16 : MODE;
  static constexpr int CPA = (CP + 31) / 32 * 32;
  static constexpr int qw_bytes(int bn) { return bn * 16 <= 1024 ? 1024 : bn * 16; }
  // v^T in fp16 [hi | lo] parts: 64 columns per 128-byte atom row
  static constexpr int va(int bn) { return bn < 64 ? 1 : bn / 64; }
  static constexpr int v_bytes(int bn) { return REG ? 0 : 2 * va(bn) * CP * 128; }
  // Register values: the column records sit in a ring of their own (two slots
  // per exp warpgroup), so that a y' stage is free once the similarity MMAs
  // have read it, while the exp warps still read the tile's records
  // (b64_d128_f32 +9..16% at two stages).  Tensor-core values: one stage holds
  // y', the records and v^T, freed by the P.v MMAs.
  static constexpr int NR = REG ? 2 * NWG : 0;
  static constexpr int stage_bytes(int bn) {
    return KA * bn * 128 + (NR > 0 ? 0 : qw_bytes(bn)) + v_bytes(bn);
  }
  static constexpr int rec_bytes(int bn) { return NR * qw_bytes(bn); }
  // tensor-core values: each warpgroup's running fp32 sums of its drained O
  // groups, [warpgroup][channel][row] (a thread's own row: conflict-free)
  static constexpr int ORUN_BYTES = REG ? 0 : 2 * kBM * CP * 4;
  static constexpr int BUDGET = 214 * 1024;
  // TMEM columns of the accumulators: one S per warpgroup (every small
  // product first, while the sum is small, then the large ones: each addition
  // is rounded against the magnitude of what it adds to); with tensor-core
  // values P (fp16 hi/lo pairs) is written over its own S columns, and each
  // warpgroup has an O of two halves of CP columns: O_big (P_hi v_hi + P_lo
  // v_hi) and O_small (P_hi v_lo), added in the epilogue.
  static constexpr int tmem_acc(int bn) { return REG ? NWG * bn : 2 * bn + 4 * CPA; }
  // The x' rows (2 K' <= 32 KA columns) sit in TMEM as the A operand of the
  // similarity MMAs when the accumulators leave room, else in shared memory.
  static constexpr bool xt(int bn) { return tmem_acc(bn) + 32 * KA <= 512; }
  static constexpr int x_bytes(int bn) { return xt(bn) ? 0 : KA * kAtom; }
  static constexpr bool fits(int bn) {
    return tmem_acc(bn) <= 512 &&
           (BUDGET - x_bytes(bn) - rec_bytes(bn) - ORUN_BYTES) / stage_bytes(bn) >= 2;
  }
  // Column tile.  An M = 128, K = 16 MMA costs the same at N = 32 and 64 and a
  // sixth more at 128 (measured on B200: 55.6, 55.6 and 64.9 cycles), and a
  // tile's commits are paid once, so the widest tile that fits is the cheapest
  // per pair; three register channels use 32 columns (registers).
  static constexpr int BN = MODE == 3 ? 32 : (fits(128) ? 128 : (fits(64) ? 64 : 32));
  static constexpr bool XT = xt(BN);
  static constexpr int X_BYTES = x_bytes(BN);
  static constexpr int QW_BYTES = qw_bytes(BN);
  static constexpr int Y_BYTES = KA * BN * 128;
  static constexpr int V_ATOM = CP * 128;               // CP rows x 64 fp16 columns
  static constexpr int VA = va(BN);                     // v^T atoms per part and stage
  static constexpr int V_BYTES = v_bytes(BN);
  static constexpr int STAGE = stage_bytes(BN);
  static constexpr int REC_BYTES = rec_bytes(BN);
  static constexpr int NST_FIT = (BUDGET - X_BYTES - REC_BYTES - ORUN_BYTES) / STAGE;
  static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
  static constexpr int NBARS = 2 * NST + 2 + 4 * NWG + 2 * NR;
  static constexpr int RED_BYTES = (NWG - 1) * kBM * 32;   // warpgroups 1.. partial sums (m, l)
  static constexpr int SMEM_RAW =
      1024 + X_BYTES + NST * STAGE + REC_BYTES + ORUN_BYTES + 8 * NBARS + 16 + RED_BYTES;
  // at least ~120 KB: one CTA per SM, so the 512-column TMEM allocation never waits
  static constexpr int SMEM = SMEM_RAW < 122880 ? 122880 : SMEM_RAW;
  // TMEM columns.  Register values: S0 | S1 | S2 | x'.  Tensor-core values:
  // S0 | S1 | O0 | O1 | x', O_h as [O_big (CP) | O_small (CP)] in 2 CPA columns;
  // P_h over S_h: the 32-column chunk c of S holds, once read, the fp16 pairs of
  // its P_hi in columns [32 c, 32 c + 16) and of its P_lo in [32 c + 16, 32 c + 32).
  __host__ __device__ static constexpr uint32_t col_s(int h) { return h * BN; }
  // P_hi of K step ks (16 S columns; its P_lo 16 columns on)
  __host__ __device__ static constexpr uint32_t col_p(int h, int ks) {
    return h * BN + (ks >> 1) * 32 + (ks & 1) * 8;
  }
  __host__ __device__ static constexpr uint32_t col_o(int h) { return 2 * BN + 2 * CPA * h; }
  static constexpr uint32_t COL_X = tmem_acc(BN);
  static_assert(NST >= 2, "shared memory budget");
  static_assert(tmem_acc(BN) + (XT ? 32 * KA : 0) <= 512, "TMEM budget");
  static_assert(REG || (CP % 16 == 0 && CP >= 16 && CP <= 64), "value chunk");
  // P_hi [v_hi ; v_lo] reads the hi and lo value atoms of 64 columns as one
  // operand of 2 CP rows: a stage keeps them adjacent, atom a's hi then lo
  static_assert(REG || (VA >= 1 && BN == 64 * VA), "value atoms of a stage");
  static_assert(SMEM_RAW <= 227 * 1024, "shared memory per CTA");
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
        atomicOr(&g_device_error_f32, 1);
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
      atomicOr(&g_device_error_f32, 4);
      return;
    }
  }
}

// The 16 bits of an fp16 / bf16 value (unsplit rows; fp32 inputs never take them).
__device__ __forceinline__ uint16_t raw16(__half v) { return __half_as_ushort(v); }
__device__ __forceinline__ uint16_t raw16(__nv_bfloat16 v) { return __bfloat16_as_ushort(v); }
__device__ __forceinline__ uint16_t raw16(float v) { return __half_as_ushort(__float2half_rn(v)); }

// Split rows hold v' 2^e in fp16 hi + lo parts, e per batch from the bits of
// max |v'| over its x' and y' rows: the largest scaled value lies in
// [2^14, 2^15), clear of fp16's overflow, and the lo parts keep their 11 bits
// down to values 2^-14 (below that their absolute error stays under 2^-25,
// i.e. 2^-39 of the largest).  e is clamped to [-40, 60]; S from scaled rows
// is 2^(2e) S, undone in the exponent's constant.
__device__ __forceinline__ int split_exp(int amax_bits) {
  if (amax_bits <= 0) return 0;   // all points at the centre
  const int e = 14 - (((amax_bits >> 23) & 0xff) - 127);
  return e < -40 ? -40 : (e > 60 ? 60 : e);
}
// 2^k for an integer -126 <= k <= 127, exactly.
__device__ __forceinline__ float pow2_int(int k) { return __int_as_float((k + 127) << 23); }
// Tensor-core values: P is multiplied by 2^14 before its fp16 split, which
// keeps every P at or above 2^-28 in fp16's normal range.
constexpr float kPScale = 16384.f;
// Tensor-core values: column tiles a warpgroup's O accumulator sums before the
// exp warps add it into fp32 registers and the P.v MMAs start it afresh.  The
// tensor core rounds each MMA's addition into its fp32 accumulator, and over the
// ~2000 additions of a 65536-column split that drift reached 7.6e-5 of the sum
// (B = 4, N = 65536, 32 channels); 16 tiles (64 additions) keep it near 2e-6.
constexpr int kOGroup = 16;

// Named barrier of every exp warp of the CTA (warps 2.., nthreads = 128 per
// exp warpgroup).
__device__ __forceinline__ void exp_warps_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// LSE (register values, one channel): per row, the log-sum-exp of
// t_ij + log2 w_j as a running maximum m and a sum l of 2^(t - m), updated per
// 32-column chunk (the maximum of the chunk first, then its shifted sum), so
// that no value under- or overflows.
// SPLIT: rows [hi | lo] and three products per K step (fp32 inputs), or the
// exact fp16 / bf16 input rows and the large product alone.
template <int KA, int MODE, bool LSE, bool SPLIT>
__global__ void __launch_bounds__(F32Cfg<KA, MODE>::THREADS, 1)
    tc_f32_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                  const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmV,
                  const F32KParams p) {
  using Cfg = F32Cfg<KA, MODE>;
  constexpr bool REG = Cfg::REG;
  static_assert(REG || !LSE, "log-sum-exp runs on the register path");
  constexpr int kAtomElems = 64;   // 16-bit packed-row elements per 128-byte atom
  constexpr int CP = Cfg::CP;
  constexpr int NST = Cfg::NST;
  constexpr int BN = Cfg::BN;
  if (p.bn != BN || p.split != (SPLIT ? 1 : 0)) {   // boxes made for another instantiation
    if (threadIdx.x == 0) atomicOr(&g_device_error_f32, 2);
    return;
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sX = smem;
  uint8_t* sStage = smem + Cfg::X_BYTES;
  uint8_t* sRec = sStage + NST * Cfg::STAGE;   // register values: the records ring
  float* sOrun = reinterpret_cast<float*>(sRec + Cfg::REC_BYTES);   // tensor-core values
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRec + Cfg::REC_BYTES + Cfg::ORUN_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float4* red = reinterpret_cast<float4*>(tmem_slot + 4);   // 16-byte aligned

  const uint32_t bar0 = smem_u32(bars);
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (NST + s); };
  const uint32_t bar_x = bar0 + 8u * (2 * NST);
  constexpr int NWG = Cfg::NWG;
  auto bar_s = [&](int h) { return bar0 + 8u * (2 * NST + 1 + h); };             // S_h ready
  auto bar_f = [&](int h) { return bar0 + 8u * (2 * NST + 1 + NWG + h); };       // S_h read out
  auto bar_p = [&](int h) { return bar0 + 8u * (2 * NST + 1 + 2 * NWG + h); };   // P_h written
  // O_h complete after the last tile of a group of kOGroup (tensor-core values)
  auto bar_q = [&](int h) { return bar0 + 8u * (2 * NST + 1 + 3 * NWG + h); };
  const uint32_t bar_o = bar0 + 8u * (2 * NST + 1 + 4 * NWG);
  constexpr int NR = Cfg::NR;
  constexpr bool RSEP = NR > 0;          // the records in a ring of their own (register values)
  constexpr int NRM = RSEP ? NR : 1;     // (slot arithmetic)
  auto bar_rfull = [&](int r) { return bar0 + 8u * (2 * NST + 2 + 4 * NWG + r); };        // landed
  auto bar_rempty = [&](int r) { return bar0 + 8u * (2 * NST + 2 + 4 * NWG + NR + r); };  // read

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = blockIdx.z;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kBM;
  const int64_t jbeg = static_cast<int64_t>(blockIdx.y) * p.cols_per_split;
  const int64_t jend = min(p.N, jbeg + p.cols_per_split);
  const int T = (jend > jbeg) ? static_cast<int>((jend - jbeg + BN - 1) / BN) : 0;
  const uint64_t wlim = g_wait_limit_ns_f32;
  const int stall = g_test_stall_f32;
  int issued = 0;   // producer lane: column tiles whose loads were issued

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full(s), 1);
      // a stage is released by the MMAs that read it last: the similarity
      // (register values) or P.v (tensor-core values)
      mbar_init(bar_empty(s), 1);
    }
    // a records slot: loaded with its tile's y', released by the 128 exp
    // threads of the warpgroup that summed the tile
    for (int r = 0; r < NR; ++r) {
      mbar_init(bar_rfull(r), 1);
      mbar_init(bar_rempty(r), 4 * 32);
    }
    // x' ready: the TMA load (shared memory), or the 128 threads of exp
    // warpgroup 0 that copy the rows into TMEM
    mbar_init(bar_x, Cfg::XT ? 4 * 32 : 1);
    for (int h = 0; h < NWG; ++h) {
      mbar_init(bar_s(h), 1);
      mbar_init(bar_f(h), 4 * 32);
      mbar_init(bar_p(h), 4 * 32);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmY);
      tma_prefetch_desc(&tmQ);
      if constexpr (!REG) tma_prefetch_desc(&tmV);
      if constexpr (!Cfg::XT) {
        tma_prefetch_desc(&tmX);
        mbar_arrive_expect_tx(bar_x, p.atoms * kAtom);
        for (int a = 0; a < p.atoms; ++a)
          tma_load_3d(smem_u32(sX + a * kAtom), &tmX, bar_x, a * kAtomElems, static_cast<int>(row0),
                      static_cast<int>(b));
      }
      const uint32_t stage_tx = p.atoms * BN * 128 + (RSEP ? 0 : BN * 16) + Cfg::V_BYTES;
      for (int t = 0; t < T; ++t) {
        const int st = t % NST;
        const int rs = RSEP ? t % NRM : 0;
        // both slots of tile t free before either load: "issued" then counts the
        // tiles whose loads (all of them) are in flight
        if (t >= NST && !wait_bar(bar_empty(st), ((t / NST) - 1) & 1, abort_flag, wlim)) break;
        if (RSEP && t >= NR && !wait_bar(bar_rempty(rs), ((t / NRM) - 1) & 1, abort_flag, wlim))
          break;
        uint8_t* sy = sStage + st * Cfg::STAGE;
        uint8_t* sq = RSEP ? sRec + rs * Cfg::QW_BYTES : sy + Cfg::Y_BYTES;
        uint8_t* sv = sq + Cfg::QW_BYTES;
        const int j0 = static_cast<int>(jbeg + static_cast<int64_t>(t) * BN);
        mbar_arrive_expect_tx(bar_full(st), stage_tx);
        for (int a = 0; a < p.atoms; ++a)
          tma_load_3d(smem_u32(sy + a * BN * 128), &tmY, bar_full(st), a * kAtomElems, j0,
                      static_cast<int>(b));
        const uint32_t bar_q_in = RSEP ? bar_rfull(rs) : bar_full(st);
        if constexpr (RSEP) mbar_arrive_expect_tx(bar_q_in, BN * 16);
        tma_load_3d(smem_u32(sq), &tmQ, bar_q_in, j0, 0, static_cast<int>(b));
        if constexpr (!REG) {
          for (int hl = 0; hl < 2; ++hl)
            for (int a = 0; a < Cfg::VA; ++a)
              tma_load_3d(smem_u32(sv + (2 * a + hl) * Cfg::V_ATOM), &tmV, bar_full(st),
                          j0 + a * 64, 0, static_cast<int>(hl * p.Bsz + b));
        }
        issued = t + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kind::f16, 16 per K step: fp16 hi / lo parts, or the unsplit fp16 / bf16 rows
      const uint32_t idS = idesc_f16(SPLIT ? 0 : p.afmt, kBM, BN);
      const uint32_t idO = idesc_f16(0, kBM, CP);   // P.v: fp16 parts of P 2^14 and v 2^e
      const int ks_lo = p.ksteps;   // the lo half of a split row starts K' columns on
      const int ksteps = p.ksteps;
      // K step ks (8 floats = 32 bytes) of a packed row block whose atoms are
      // atom_bytes apart, from the descriptor of the block's start: the
      // descriptors of the operand regions are built once, and each operand's is
      // one add away (the issuing thread's time goes to MMAs, not to masks)
      const uint64_t dX = desc_k_sw128(smem_u32(sX));
      const uint64_t dStage = desc_k_sw128(smem_u32(sStage));
      auto kdesc = [](uint64_t dbase, int atom_bytes, int ks) {
        const int off = ks * 32;
        return desc_advance(dbase, static_cast<uint32_t>((off >> 7) * atom_bytes + (off & 127)));
      };
      // S = x'.y'^T for warpgroup h, one accumulator: every small product
      // (lo.hi, hi.lo) of every K step first, while the sum is small, then the
      // large ones -- each addition is rounded against the magnitude of what it
      // adds to.  (On B200 a chain of kind::f16 MMAs into one accumulator issues
      // as fast as independent ones, so a second accumulator would buy nothing.)
      auto issue_S = [&](int h, int st) {
        const uint64_t sy = desc_advance(dStage, static_cast<uint32_t>(st * Cfg::STAGE));
        const uint32_t db = tmem + Cfg::col_s(h);
        auto mma = [&](uint32_t d, int ka, uint64_t bdesc, uint32_t acc) {
          if constexpr (Cfg::XT)
            mma_ts(d, tmem + Cfg::COL_X + ka * 8, bdesc, idS, acc);
          else
            mma_ss(d, kdesc(dX, kAtom, ka), bdesc, idS, acc);
        };
        // (exact 16-bit operands, SPLIT false: the large products alone).  The K
        // step count is a template constant of each branch of the switch below:
        // fully unrolled, the address arithmetic of every MMA is laid out ahead of
        // the MMAs instead of between them on the one issuing thread (measured: a
        // run-time loop here cost about twice the MMAs themselves)
        auto steps = [&](auto kn) {
          constexpr int KN = decltype(kn)::value;
          if constexpr (SPLIT) {
#pragma unroll
            for (int ks = 0; ks < KN; ++ks) {
              mma(db, ks + ks_lo, kdesc(sy, BN * 128, ks), ks > 0 ? 1u : 0u);
              mma(db, ks, kdesc(sy, BN * 128, ks + ks_lo), 1u);
            }
          }
#pragma unroll
          for (int ks = 0; ks < KN; ++ks)
            mma(db, ks, kdesc(sy, BN * 128, ks), (SPLIT || ks > 0) ? 1u : 0u);
        };
        // K steps a packed row can hold: split rows [hi K' | lo K'] fill 2 K' <= 64 KA
        // columns, unsplit rows K' <= 64 KA
        constexpr int KSMAX = SPLIT ? 2 * KA : 4 * KA;
        switch (ksteps) {
          case 1: steps(std::integral_constant<int, 1>{}); break;
          case 2: if constexpr (KSMAX >= 2) steps(std::integral_constant<int, 2>{}); break;
          case 3: if constexpr (KSMAX >= 3) steps(std::integral_constant<int, 3>{}); break;
          case 4: if constexpr (KSMAX >= 4) steps(std::integral_constant<int, 4>{}); break;
          case 5: if constexpr (KSMAX >= 5) steps(std::integral_constant<int, 5>{}); break;
          case 6: if constexpr (KSMAX >= 6) steps(std::integral_constant<int, 6>{}); break;
          case 7: if constexpr (KSMAX >= 7) steps(std::integral_constant<int, 7>{}); break;
          default: if constexpr (KSMAX >= 8) steps(std::integral_constant<int, 8>{}); break;
        }
      };
      // O_h += P_hi [v_hi ; v_lo] (one MMA of N = 2 CP: O_big and O_small at
      // once, as cheap as one of N = CP) and P_lo v_hi into O_big: two MMAs a
      // K step where the three products of N = CP took three.
      const uint32_t idO2 = idesc_f16(0, kBM, 2 * CP);
      auto issue_O = [&](int h, int st, bool acc_prev) {
        const uint64_t sv = desc_advance(
            dStage, static_cast<uint32_t>(st * Cfg::STAGE + Cfg::Y_BYTES + Cfg::QW_BYTES));
        const uint32_t d = tmem + Cfg::col_o(h);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {   // K steps of 16 columns
          // atom ks / 4: rows 0 .. CP-1 the hi atom, CP .. 2 CP-1 the lo atom
          // right after it; 32 bytes a K step within the atom
          const uint64_t bhl = desc_advance(
              sv, static_cast<uint32_t>((ks >> 2) * 2 * Cfg::V_ATOM + (ks & 3) * 32));
          const uint32_t phi = tmem + Cfg::col_p(h, ks);
          const uint32_t plo = phi + 16;
          mma_ts(d, phi, bhl, idO2, (acc_prev || ks > 0) ? 1u : 0u);
          mma_ts(d, plo, bhl, idO, 1u);
        }
      };
      bool ok = wait_bar(bar_x, 0, abort_flag, wlim) && stall != 1;
      tc_fence_after();
      for (int h = 0; ok && h < NWG && h < T; ++h) {
        ok = wait_bar(bar_full(h), 0, abort_flag, wlim);
        if (ok) {
          tc_fence_after();
          issue_S(h, h);
          mma_commit(bar_s(h));
          if constexpr (RSEP) mma_commit(bar_empty(h % NST));
        }
      }
      // Register values: S_h(t + NWG) may overwrite S_h once warpgroup h has
      // read S_h(t).  Tensor-core values: P_h(t) lives in S_h's columns, so
      // S_h(t + 2) follows O_h(t), the MMA that reads it (the tensor core runs
      // one thread's MMAs in order).
      constexpr bool kSFirst = REG;
      auto next_S = [&](int h, int k, int t2) {
        if (REG && !wait_bar(bar_f(h), k & 1, abort_flag, wlim)) return false;
        if (!wait_bar(bar_full(t2 % NST), (t2 / NST) & 1, abort_flag, wlim)) return false;
        tc_fence_after();
        issue_S(h, t2 % NST);
        mma_commit(bar_s(h));
        if constexpr (RSEP) mma_commit(bar_empty(t2 % NST));
        return true;
      };
      for (int k = 0; ok && NWG * k < T; ++k) {
        for (int h = 0; h < NWG; ++h) {
          const int t = NWG * k + h;
          if (t >= T) break;
          const int t2 = t + NWG;
          if (kSFirst && t2 < T && !(ok = next_S(h, k, t2))) break;
          if constexpr (!REG) {
            if (!(ok = wait_bar(bar_p(h), k & 1, abort_flag, wlim))) break;
            tc_fence_after();
            issue_O(h, t % NST, k % kOGroup != 0);
            if ((k + 1) % kOGroup == 0) mma_commit(bar_q(h));   // (the group's drain waits on it)
            mma_commit(bar_empty(t % NST));
            if (!kSFirst && t2 < T && !(ok = next_S(h, k, t2))) break;
          }
        }
      }
      mma_commit(bar_o);   // also the drain point for whatever was issued
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ exp warpgroups
    const int h = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int64_t i = row0 + row;
    const bool valid = i < p.M;
    const float r = valid ? p.rnorm[b * p.M + i] : 0.f;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    // the exponent's constant, with the split rows' scale 2^(2e) undone
    const float two_c =
        SPLIT ? p.two_c * pow2_int(-split_exp(p.amax[b])) * pow2_int(-split_exp(p.amax[b])) : p.two_c;
    const uint64_t two_c2 = pk2(two_c, two_c);
    const uint64_t r2 = pk2(r, r);
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f;   // register values: running row sums (l for LSE)
    float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY;   // LSE: running maxima
    if constexpr (Cfg::XT) {
      if (h == 0) {
        // this thread's packed row (zeros past M) into its TMEM lane
        const int rowf = (SPLIT ? 2 : 1) * p.ksteps * 8;
        const float4* src = reinterpret_cast<const float4*>(p.xpack + (b * p.M + i) * rowf);
        for (int c = 0; c < (rowf + 15) / 16; ++c) {   // (rowf is a multiple of 8)
          uint32_t v[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const bool in = valid && c * 16 + 4 * u < rowf;
            const float4 f = in ? src[c * 4 + u] : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * u + 0] = __float_as_uint(f.x);
            v[4 * u + 1] = __float_as_uint(f.y);
            v[4 * u + 2] = __float_as_uint(f.z);
            v[4 * u + 3] = __float_as_uint(f.w);
          }
          tmem_st16(tmem + lane_base + Cfg::COL_X + c * 16, v);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_x);
      }
    }
    bool ok = true;
    if (stall == 2) {   // test hook: wait on a barrier nobody arrives on, until the limit
      wait_bar(bar_p(h), 0, abort_flag, wlim);
      ok = false;
    }
    int k = 0;
    // tensor-core values: this warpgroup's O summed over the drained tile groups,
    // this thread's row of it in shared memory (channel c at orun[c * kBM])
    float* orun = sOrun + h * CP * kBM + row;
    if constexpr (!REG) {
#pragma unroll 4
      for (int c = 0; c < CP; ++c) orun[c * kBM] = 0.f;
    }
    const uint32_t tOh = tmem + lane_base + Cfg::col_o(h);
    // O_h (big + small) added into orun, 16 channels at a time
    auto add_o = [&]() {
#pragma unroll 1
      for (int ch = 0; ch < (REG ? 0 : CP / 16); ++ch) {
        uint32_t vb[16], vs[16];
        tmem_ld16(tOh + ch * 16, vb);
        tmem_ld16(tOh + CP + ch * 16, vs);
        tmem_wait_ld();
        reg_fence16(vb);
        reg_fence16(vs);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          orun[(ch * 16 + q) * kBM] += __uint_as_float(vb[q]) + __uint_as_float(vs[q]);
      }
    };
    for (int t = h; ok && t < T; t += NWG, ++k) {
      const int st = t % NST;
      if constexpr (!REG) {
        if (k > 0 && k % kOGroup == 0) {
          // O_h has summed kOGroup tiles: once their P.v MMAs are done, into the
          // fp32 sums in shared memory; tile k's P.v MMAs then start O_h afresh
          ok = __all_sync(0xffffffffu,
                          wait_bar(bar_q(h), ((k / kOGroup) - 1) & 1, abort_flag, wlim));
          if (!ok) break;
          tc_fence_after();
          add_o();
        }
      }
      ok = wait_bar(bar_s(h), k & 1, abort_flag, wlim) &&   // norms and values landed
           (RSEP ? wait_bar(bar_rfull(t % NRM), (t / NRM) & 1, abort_flag, wlim)
                : wait_bar(bar_full(st), (t / NST) & 1, abort_flag, wlim));
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + Cfg::col_s(h);
      // the column records, lane by lane: q_j at qrec[j], value c at qrec[(1 + c) BN + j]
      const float* qrec = reinterpret_cast<const float*>(
          RSEP ? sRec + (t % NRM) * Cfg::QW_BYTES : sStage + st * Cfg::STAGE + Cfg::Y_BYTES);
      if constexpr (REG) {
        // S, 32 columns at a time: the loads of chunk ch + 1 are in flight
        // while chunk ch is exponentiated; once the last chunk is in registers
        // the TMEM columns may be reused.  P.v in registers, a partial sum per
        // tile (two-level accumulation).
        constexpr int NCH = BN / 32;
        uint32_t cb[32];
        tmem_ld32(tS, cb);
        tmem_wait_ld();
        reg_fence32(cb);
        // P.v partial sums of this tile, even and odd columns packed
        uint64_t s0 = 0ull, s1 = 0ull, s2 = 0ull;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          if constexpr (!LSE) {
            // t = S 2c + r + q_j, two columns per packed operation
            uint64_t cur2[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              cur2[e] = fma2(pk2(__uint_as_float(cb[2 * e]), __uint_as_float(cb[2 * e + 1])), two_c2, r2);
            if (ch + 1 < NCH) {
              tmem_ld32(tS + (ch + 1) * 32, cb);
            } else {
              tc_fence_before();
              mbar_arrive(bar_f(h));
            }
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const int j = ch * 32 + 4 * e4;
              const float4 qv = *reinterpret_cast<const float4*>(qrec + j);
              const float4 w0 = *reinterpret_cast<const float4*>(qrec + BN + j);
              float4 w1, w2;
              if constexpr (MODE == 3) {
                w1 = *reinterpret_cast<const float4*>(qrec + 2 * BN + j);
                w2 = *reinterpret_cast<const float4*>(qrec + 3 * BN + j);
              }
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                float t0, t1;
                upk2(add2(cur2[2 * e4 + hh], hh ? pk2(qv.z, qv.w) : pk2(qv.x, qv.y)), t0, t1);
                const uint64_t pe = pk2(ex2(t0), ex2(t1));
                s0 = fma2(pe, hh ? pk2(w0.z, w0.w) : pk2(w0.x, w0.y), s0);
                if constexpr (MODE == 3) {
                  s1 = fma2(pe, hh ? pk2(w1.z, w1.w) : pk2(w1.x, w1.y), s1);
                  s2 = fma2(pe, hh ? pk2(w2.z, w2.w) : pk2(w2.x, w2.y), s2);
                }
              }
            }
          } else {
            float cur[32];
#pragma unroll
            for (int e = 0; e < 32; ++e)
              cur[e] = fmaf(__uint_as_float(cb[e]), two_c, r);
            if (ch + 1 < NCH) {
              tmem_ld32(tS + (ch + 1) * 32, cb);
            } else {
              tc_fence_before();
              mbar_arrive(bar_f(h));
            }
            // lanes 1.. of the records hold log2 w: u = t + log2 w per channel
            auto lse_channel = [&](int lanec, float& m, float& l) {
              const float* lw = qrec + lanec * BN + ch * 32;
              float cm = -INFINITY;
#pragma unroll
              for (int e = 0; e < 32; ++e) cm = fmaxf(cm, cur[e] + lw[e]);
              const float mn = fmaxf(m, cm);
              if (mn != -INFINITY) {
                float cs = 0.f;
#pragma unroll
                for (int e = 0; e < 32; ++e) cs += ex2(cur[e] + lw[e] - mn);
                l = fmaf(l, ex2(m - mn), cs);   // m = -inf: l = 0 and ex2(-inf) = 0
                m = mn;
              }
            };
#pragma unroll
            for (int e = 0; e < 32; ++e) cur[e] += qrec[ch * 32 + e];
            lse_channel(1, mx0, acc0);
            if constexpr (MODE > 1) {
              lse_channel(2, mx1, acc1);
              lse_channel(3, mx2, acc2);
            }
          }
          if (ch + 1 < NCH) {
            tmem_wait_ld();
            reg_fence32(cb);
          }
        }
        if constexpr (!LSE) {   // (log-sum-exp: the running (m, l) are mx*, acc*)
          float lo, hi;
          upk2(s0, lo, hi);
          acc0 += lo + hi;
          if constexpr (MODE == 3) {
            upk2(s1, lo, hi);
            acc1 += lo + hi;
            upk2(s2, lo, hi);
            acc2 += lo + hi;
          }
        }
        mbar_arrive(bar_rempty(t % NRM));   // this thread is done with the records
      } else {
        // S chunk by chunk, 32 columns: each chunk's P goes over the chunk's
        // own S columns once they are read.  (S_h(t) was written after O_h(t-2)
        // had read P_h(t-2) from these columns: the MMAs run in order.)
#pragma unroll
        for (int ch = 0; ch < BN / 32; ++ch) {
          uint32_t sv[32];
          tmem_ld32(tS + ch * 32, sv);
          tmem_wait_ld();
          reg_fence32(sv);
          // P 2^14 in fp16 hi + lo parts, two columns per 32-bit TMEM word:
          // every P keeps an absolute error under 2^-39 (relative 2^-22 from
          // P = 2^-3 up)
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = ch * 32 + 2 * e;
            float t0, t1;
            upk2(add2(fma2(pk2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                           two_c2, r2),
                      *reinterpret_cast<const uint64_t*>(qrec + c)),
                 t0, t1);
            const float u0 = ex2(t0) * kPScale, u1 = ex2(t1) * kPScale;
            const __half2 h2 = __floats2half2_rn(u0, u1);
            const float2 hf = __half22float2(h2);
            const __half2 l2 = __floats2half2_rn(u0 - hf.x, u1 - hf.y);
            hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
            lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          tmem_st16(tS + ch * 32, hi);
          tmem_st16(tS + ch * 32 + 16, lo);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p(h));
      }
    }
    if constexpr (REG) {
      // warpgroups 1.. hand their row sums (or their (m, l)) to warpgroup 0,
      // which adds them in warpgroup order; every exp warp reaches the barrier
      if (h > 0) {
        red[2 * ((h - 1) * kBM + row)] = make_float4(acc0, acc1, acc2, 0.f);
        red[2 * ((h - 1) * kBM + row) + 1] = make_float4(mx0, mx1, mx2, 0.f);
      }
      exp_warps_sync(NWG * 128);
      if (h == 0 && valid && ok && !*abort_flag) {
        const int64_t at = static_cast<int64_t>(blockIdx.y) * p.split_stride +
                           (b * p.M + i) * p.ldo + p.c0;
#pragma unroll
        for (int g = 1; g < NWG; ++g) {
          const float4 o = red[2 * ((g - 1) * kBM + row)];
          if constexpr (!LSE) {
            acc0 += o.x;
            acc1 += o.y;
            acc2 += o.z;
          } else {
            const float4 om = red[2 * ((g - 1) * kBM + row) + 1];
            // (m, l) merged with (m1, l1): the larger shift, both sums rescaled to it
            auto merge = [&](float& m0, float& l0, float m1, float l1) {
              const float m = fmaxf(m0, m1);
              float l = 0.f;
              if (m != -INFINITY) l = l0 * ex2(m0 - m) + l1 * ex2(m1 - m);
              m0 = m;
              l0 = l;
            };
            merge(mx0, acc0, om.x, o.x);
            merge(mx1, acc1, om.y, o.y);
            merge(mx2, acc2, om.z, o.z);
          }
        }
        if constexpr (!LSE) {
          float* orow = p.out + at;
          orow[0] = acc0;
          if (p.cw > 1) orow[1] = acc1;
          if (p.cw > 2) orow[2] = acc2;
        } else {
          p.out[at] = mx0;
          p.out_l[at] = acc0;
          if (p.cw > 1) { p.out[at + 1] = mx1; p.out_l[at + 1] = acc1; }
          if (p.cw > 2) { p.out[at + 2] = mx2; p.out_l[at + 2] = acc2; }
        }
      }
    } else {
      if (ok) ok = wait_bar(bar_o, 0, abort_flag, wlim);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      // Each warpgroup's total: the drained groups plus the open one still in O_h
      // (none when the warpgroup had no tile); then warpgroup 0 adds warpgroup 1's
      // (both warpgroups reach the barrier)
      const int kh = T > h ? (T - h + NWG - 1) / NWG : 0;   // column tiles of warpgroup h
      if (ok && kh > 0) add_o();
      exp_warps_sync(NWG * 128);
      if (ok && h == 0 && valid) {
        float* orow = p.out + static_cast<int64_t>(blockIdx.y) * p.split_stride +
                      (b * p.M + i) * p.ldo + p.c0;
        const float* orun1 = sOrun + CP * kBM + row;
        for (int c = 0; c < p.cw; ++c)   // undo P's 2^14 and the channel's 2^e, exactly
          orow[c] = (orun[c * kBM] + orun1[c * kBM]) *
                    pow2_int(-14 - split_exp(p.vmax[b * CP + c]));
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
    if constexpr (RSEP)
      for (int t = issued > NR ? issued - NR : 0; t < issued; ++t)
        drain_bar(bar_rfull(t % NRM), (t / NRM) & 1, wlim);
    if constexpr (!Cfg::XT) drain_bar(bar_x, 0, wlim);
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
// z[b, :] = the mean of the column points y[b, s * stride, :], s < S, with
// S = min(N, 1024) and stride = N / S (any centre is exact; a sample mean
// costs little and is not thrown off by one outlying point).  Fixed summation
// order: warp w of the block takes samples w, w + 8, ...; lanes take features.
__global__ void column_mean_kernel(const float* __restrict__ y, float* __restrict__ z, int64_t N,
                                   int D) {
  __shared__ float part[8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t b = blockIdx.x;
  const int k = blockIdx.y * 32 + lane;
  const int64_t S = N < 1024 ? N : 1024;
  const int64_t stride = S > 0 ? N / S : 1;
  float acc = 0.f;
  if (k < D)
    for (int64_t q = w; q < S; q += 8) acc += y[(b * N + q * stride) * D + k];
  part[w][lane] = acc;
  __syncthreads();
  if (w == 0 && k < D) {
    float t = 0.f;
    for (int q = 0; q < 8; ++q) t += part[q][lane];
    z[b * D + k] = S > 0 ? t / static_cast<float>(S) : 0.f;
  }
}

// Per batch, the bits of max |v_k - z_k| over the rows of x and y (non-negative
// floats order like their bit patterns): the split rows' scale.  Grid
// (B, blocks) of 256 threads; a group of `grp` lanes (a power of two, 4
// features a lane, D <= 128) reads one row, so a warp reads 32 / grp rows at
// once; amax zeroed before.
__global__ void centred_maxabs_kernel(const float* __restrict__ x, const float* __restrict__ y,
                                      const float* __restrict__ zc, int* __restrict__ amax,
                                      int64_t M, int64_t N, int D, int grp) {
  const int64_t b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rpw = 32 / grp, lig = lane & (grp - 1), sub = lane / grp;
  const int k0 = 4 * lig;
  float z[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) z[u] = (k0 + u < D) ? zc[b * D + k0 + u] : 0.f;
  float m = 0.f;
  for (int64_t r0 = (static_cast<int64_t>(blockIdx.y) * 8 + warp) * rpw; r0 < M + N;
       r0 += static_cast<int64_t>(gridDim.y) * 8 * rpw) {
    const int64_t r = r0 + sub;
    if (r >= M + N) continue;
    const float* v = r < M ? x + (b * M + r) * D : y + (b * N + (r - M)) * D;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (k0 + u < D) m = fmaxf(m, fabsf(v[k0 + u] - z[u]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if (lane == 0) wm[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wm[w]);
    atomicMax(amax + b, __float_as_int(m));
  }
}

// Packed operand rows of the centred points v' = v - z, z = zc[b, :]: fp16
// [hi (K') | lo (K')] of v' 2^e (split_exp), and the norm term -c |v'|^2 from
// v' itself in fp32: for the row side into
// norm[b * R + r]; for the column side (records) into lane 0 of the column's
// record, norm[4 b Rpad + r] (lanes 1-3, Rpad floats apart, zeroed), with -inf
// for the padding columns r >= R.  fp16 / bf16 inputs (zc == nullptr,
// split == 0): the input values themselves, rows [v (K')] only.
struct PackSide {
  const void* src;
  float* dst;
  float* norm;
  int64_t R, Rpad;
  int records;
};

// Both sides in one launch: blockIdx.z = 0 the rows, 1 the columns; blockIdx.y
// = the batch (its centre and scale read once per block).  Split rows: a group
// of `grp` lanes (a power of two, 4 features a lane) builds one row, so a warp
// builds 32 / grp rows at once; unsplit rows (fp16 / bf16 inputs): one warp per
// row, lanes along the features.
template <typename T>
__global__ void pack_rows_f32_kernel(PackSide rows_side, PackSide cols_side,
                                     const float* __restrict__ zc, int D, int Kp, float c,
                                     int split, const int* __restrict__ amax, int grp) {
  const PackSide& ps = blockIdx.z == 0 ? rows_side : cols_side;
  const T* __restrict__ src = static_cast<const T*>(ps.src);
  const int64_t R = ps.R, Rpad = ps.Rpad;
  const int records = ps.records;
  const int lane = threadIdx.x & 31;
  const int64_t b = blockIdx.y;
  const float* z = zc ? zc + b * D : nullptr;
  const int64_t gw = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  // records: lane l of column rr at norm[(4 b + l) Rpad + rr]; rows: norm[b Rpad + rr]
  auto norm_at = [&](int64_t rr) { return records ? ps.norm + 4 * b * Rpad + rr : ps.norm + b * Rpad + rr; };
  if (split) {
    // fp16 [hi (K') | lo (K')] of v' 2^e: v' 2^e is exact, hi its nearest fp16,
    // lo the nearest fp16 of the (exact) remainder
    const float sc = pow2_int(split_exp(amax[b]));
    const int rpw = 32 / grp, lig = lane & (grp - 1), sub = lane / grp;
    const int k0 = 4 * lig;
    for (int64_t r0 = gw * rpw; r0 < Rpad; r0 += nw * rpw) {
      const int64_t rr = r0 + sub;
      const bool row = rr < R;
      const T* v = src + (b * R + (row ? rr : 0)) * D;
      float d[4], sq = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + u;
        d[u] = (row && k < D) ? vf(v[k]) - z[k] : 0.f;
        sq = fmaf(d[u], d[u], sq);
      }
      for (int o = grp / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (rr >= Rpad) continue;
      float* nrm = norm_at(rr);
      if (!row) {
        if (lig == 0) {
          nrm[0] = -INFINITY;   // padding columns: kernel value 0
          if (records) nrm[Rpad] = nrm[2 * Rpad] = nrm[3 * Rpad] = 0.f;
        }
        continue;
      }
      if (k0 < Kp) {
        __half hi[4], lo[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float x = d[u] * sc;
          hi[u] = __float2half_rn(x);
          lo[u] = __float2half_rn(x - __half2float(hi[u]));
        }
        __half* out = reinterpret_cast<__half*>(ps.dst) + (b * R + rr) * (2 * static_cast<int64_t>(Kp)) + k0;
        *reinterpret_cast<uint2*>(out) = make_uint2(
            static_cast<uint32_t>(__half_as_ushort(hi[0])) | (static_cast<uint32_t>(__half_as_ushort(hi[1])) << 16),
            static_cast<uint32_t>(__half_as_ushort(hi[2])) | (static_cast<uint32_t>(__half_as_ushort(hi[3])) << 16));
        *reinterpret_cast<uint2*>(out + Kp) = make_uint2(
            static_cast<uint32_t>(__half_as_ushort(lo[0])) | (static_cast<uint32_t>(__half_as_ushort(lo[1])) << 16),
            static_cast<uint32_t>(__half_as_ushort(lo[2])) | (static_cast<uint32_t>(__half_as_ushort(lo[3])) << 16));
      }
      if (lig == 0) {
        nrm[0] = -c * sq;
        if (records) nrm[Rpad] = nrm[2 * Rpad] = nrm[3 * Rpad] = 0.f;
      }
    }
    return;
  }
  for (int64_t rr = gw; rr < Rpad; rr += nw) {
    float* nrm = norm_at(rr);
    if (rr >= R) {
      if (lane == 0) {
        nrm[0] = -INFINITY;   // padding columns: kernel value 0
        if (records) nrm[Rpad] = nrm[2 * Rpad] = nrm[3 * Rpad] = 0.f;
      }
      continue;
    }
    const T* v = src + (b * R + rr) * D;
    float sq = 0.f;
    // the fp16 / bf16 input values themselves (exact in the MMA's encoding)
    uint16_t* out = reinterpret_cast<uint16_t*>(ps.dst) + (b * R + rr) * static_cast<int64_t>(Kp);
    for (int k = lane; k < Kp; k += 32) {
      const float d = (k < D) ? vf(v[k]) : 0.f;
      sq = fmaf(d, d, sq);
      out[k] = (k < D) ? raw16(v[k]) : static_cast<uint16_t>(0);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) {
      nrm[0] = -c * sq;
      if (records) nrm[Rpad] = nrm[2 * Rpad] = nrm[3 * Rpad] = 0.f;
    }
  }
}

// Register-path values: channels [c0, c0 + cw) (cw <= 3) of the pass's values
// (values.cuh) into lanes 1.. of the records (qw[(4 b + l) Nq + j]); for the log-sum-exp, their
// base-2 logarithms.
template <typename TW, typename TY>
__global__ void pack_values_qw_kernel(const TW* __restrict__ w, const TY* __restrict__ y,
                                      const TY* __restrict__ rows, float* __restrict__ qw,
                                      int64_t B, int64_t N, int64_t Nq, int64_t Mrows, int C, int D,
                                      int c0, int cw, int log2_values, int64_t src_ld) {
  const int64_t total = B * N;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / N, j = e % N;
    for (int ch = 0; ch < cw; ++ch) {
      const float v = value_at(w, y, rows, b, e, Mrows, D, C, c0 + ch, src_ld);
      qw[(4 * b + 1 + ch) * Nq + j] = log2_values ? lg2(v) : v;
    }
  }
}

// Per (batch, channel cc of the chunk [c0, c0 + CP)), the bits of max |v| over
// the columns: the value parts' scale.  Grid (B CP, blocks) of 256 threads;
// vmax zeroed before.
__global__ void values_maxabs_kernel(const float* __restrict__ w, const float* __restrict__ y,
                                     const float* __restrict__ rows, int* __restrict__ vmax,
                                     int64_t N, int64_t Mrows, int C, int D, int CV, int c0, int CP,
                                     int64_t src_ld) {
  const int64_t bc = blockIdx.x;
  const int cc = static_cast<int>(bc % CP);
  const int64_t b = bc / CP;
  const int ch = c0 + cc;
  float m = 0.f;
  if (ch < CV) {
    for (int64_t j = blockIdx.y * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < N;
         j += static_cast<int64_t>(gridDim.y) * blockDim.x)
      m = fmaxf(m, fabsf(value_at(w, y, rows, b, b * N + j, Mrows, D, C, ch, src_ld)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int v = 1; v < 8; ++v) m = fmaxf(m, wm[v]);
    if (m > 0.f) atomicMax(vmax + bc, __float_as_int(m));
  }
}

// Value matrix v^T in fp16 parts of v 2^e (e per batch and channel, from vmax):
// hi at [b][CP][Nst], lo at [B + b][CP][Nst], for channels [c0, c0 + CP) of the
// pass's values (values.cuh); zeros past CV.
__global__ void pack_values_f32_split_kernel(const float* __restrict__ w,
                                             const float* __restrict__ y,
                                             const float* __restrict__ rows,
                                             __half* __restrict__ vt, const int* __restrict__ vmax,
                                             int64_t B, int64_t N, int64_t Nst, int64_t Mrows, int C,
                                             int D, int CV, int c0, int CP, int64_t src_ld) {
  const int64_t total = B * CP * N;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = e % N;
    const int64_t bc = e / N;
    const int cc = static_cast<int>(bc % CP);
    const int64_t b = bc / CP;
    const int ch = c0 + cc;
    const float v = (ch < CV) ? value_at(w, y, rows, b, b * N + j, Mrows, D, C, ch, src_ld) : 0.f;
    const float u = v * pow2_int(split_exp(vmax[b * CP + cc]));
    const __half hi = __float2half_rn(u);
    vt[(b * CP + cc) * Nst + j] = hi;
    vt[((B + b) * CP + cc) * Nst + j] = __float2half_rn(u - __half2float(hi));
  }
}

// Exponent shift of a pass (log2 units): rows -- norm[b * R + r] -- or columns
// -- the records' lane 0, norm[4 b Nq + r], r < R -- gain scale * src[(b * R + r) * ld + c].
__global__ void add_shift_kernel(float* __restrict__ norm, int64_t bstride, const float* __restrict__ src,
                                 int64_t ld, int c, float scale, int64_t B, int64_t R) {
  const int64_t total = B * R;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / R, r = e % R;
    norm[b * bstride + r] += scale * src[e * ld + c];
  }
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148 * 32) b = 148 * 32;
  return static_cast<int>(b);
}

struct TileMaps {
  CUtensorMap x, y, q, v;
};

template <int KA, int MODE, bool LSE = false, bool SPLIT = true>
cudaError_t launch_kernel(const TileMaps& m, const F32KParams& kp, dim3 grid, cudaStream_t s) {
  using Cfg = F32Cfg<KA, MODE>;
  auto fn = tc_f32_kernel<KA, MODE, LSE, SPLIT>;
  static bool attr_done = false;   // idempotent; a benign race at worst repeats the call
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  fn<<<grid, Cfg::THREADS, Cfg::SMEM, s>>>(m.x, m.y, m.q, m.v, kp);
  return cudaGetLastError();
}

template <int KA>
cudaError_t launch_mode(int mode, bool lse, const TileMaps& m, const F32KParams& kp, dim3 grid,
                        cudaStream_t s) {
  if (lse)   // one channel per pass
    return kp.split ? launch_kernel<KA, 1, true, true>(m, kp, grid, s)
                    : launch_kernel<KA, 1, true, false>(m, kp, grid, s);
  if (!kp.split) return cudaErrorInvalidValue;   // unsplit rows: log-sum-exp only
  switch (mode) {
    case 1: return launch_kernel<KA, 1>(m, kp, grid, s);
    case 3: return launch_kernel<KA, 3>(m, kp, grid, s);
    case 16: return launch_kernel<KA, 16>(m, kp, grid, s);
    case 32: return launch_kernel<KA, 32>(m, kp, grid, s);
    default: return launch_kernel<KA, 64>(m, kp, grid, s);
  }
}

// Shared-memory atoms the kernel is compiled for, covering `atoms`.
// (D <= 128: a split row [hi K' | lo K'] holds at most four 128-byte atoms)
int ka_for(int atoms) { return atoms <= 1 ? 1 : (atoms <= 2 ? 2 : 4); }

// Tile width of instantiation (KA, mode): the host sizes the TMA boxes with it.
template <int KA>
int tile_cols_ka(int mode) {
  switch (mode) {
    case 1: return F32Cfg<KA, 1>::BN;
    case 3: return F32Cfg<KA, 3>::BN;
    case 16: return F32Cfg<KA, 16>::BN;
    case 32: return F32Cfg<KA, 32>::BN;
    default: return F32Cfg<KA, 64>::BN;
  }
}


}  // namespace

F32Plan f32_plan(int64_t B, int64_t M, int64_t N, int64_t D, int sm_count, bool split) {
  F32Plan p{};
  p.split = split;
  // 16-bit rows, K' = D rounded up to 16 (kind::f16 K steps): fp16 [hi | lo]
  // (split) or the fp16 / bf16 input values (unsplit)
  p.Kp = static_cast<int>((D + 15) / 16 * 16);
  p.atoms = ((split ? 2 : 1) * p.Kp + 63) / 64;
  p.max_chunk = 64;
  // a split is a whole number of 128-column blocks (every tile width divides
  // it, so no tile straddles two splits)
  const int64_t U = B * ((M + kBM - 1) / kBM);
  const int64_t ntj = (N + 127) / 128;
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
  const int64_t per = (ntj + best - 1) / best;
  p.cols_per_split = (per < 1 ? 1 : per) * 128;
  p.splits = static_cast<int>((N + p.cols_per_split - 1) / p.cols_per_split);
  if (p.splits < 1) p.splits = 1;
  return p;
}

int f32_chunk_pad(int cw) { return cw <= 16 ? 16 : (cw <= 32 ? 32 : 64); }

int f32_tile_cols(int KA, int mode) {
  switch (KA) {
    case 1: return tile_cols_ka<1>(mode);
    case 2: return tile_cols_ka<2>(mode);
    default: return tile_cols_ka<4>(mode);
  }
}

// Packed rows of x and y (and, for fp32, the column centre first).
// The per-batch max words sit right after the column centres, then the
// per-(batch, channel) max words of a tensor-core value chunk (the workspace
// layouts reserve B (D + 1) floats, and B (D + 1 + 64) where chunks run).
int* f32_amax(const F32Args& a) { return reinterpret_cast<int*>(a.zc + a.B * a.D); }
int* f32_vmax(const F32Args& a) { return reinterpret_cast<int*>(a.zc + a.B * (a.D + 1)); }

template <typename T>
void pack_operands_f32(const F32Args& a, int64_t Nq, float c, cudaStream_t s) {
  const T* x = static_cast<const T*>(a.x);
  const T* y = static_cast<const T*>(a.y);
  const int split = a.plan.split ? 1 : 0;
  const float* zc = nullptr;
  int* amax = nullptr;
  if constexpr (std::is_same<T, float>::value) {
    if (split) {
      column_mean_kernel<<<dim3(static_cast<unsigned>(a.B), static_cast<unsigned>((a.D + 31) / 32)),
                           256, 0, s>>>(y, a.zc, a.N, a.D);
      zc = a.zc;
      amax = f32_amax(a);
      cudaMemsetAsync(amax, 0, static_cast<size_t>(a.B) * sizeof(int), s);
      int grp = 4;   // lanes per row: the power of two covering D / 4 features' lanes
      while (grp * 4 < a.D) grp *= 2;
      const int64_t per_block = 8 * (32 / grp);   // rows per block and pass
      int64_t blocks = (a.M + a.N + per_block - 1) / per_block;
      const int64_t cap = (148 * 16 + a.B - 1) / a.B;
      if (blocks > cap) blocks = cap;
      if (blocks > 65535) blocks = 65535;
      centred_maxabs_kernel<<<dim3(static_cast<unsigned>(a.B), static_cast<unsigned>(blocks)), 256, 0,
                              s>>>(x, y, a.zc, amax, a.M, a.N, a.D, grp);
    }
  }
  // one warp per row, 8 rows per 256-thread block; about 148 x 32 blocks in all
  const PackSide rs{x, a.xpack, a.rnorm, a.M, a.M, 0};
  const PackSide cs{y, a.ypack, a.qw, a.N, Nq, 1};
  const int64_t rmax = a.M > Nq ? a.M : Nq;
  int64_t bx = (rmax + 7) / 8;
  const int64_t cap = (148 * 16 + a.B - 1) / a.B;
  if (bx > cap) bx = cap;
  if (bx < 1) bx = 1;
  int grp = 4;   // lanes per split row: the power of two covering Kp / 4 features' lanes
  while (grp * 4 < a.plan.Kp) grp *= 2;
  pack_rows_f32_kernel<T><<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(a.B), 2), 256, 0, s>>>(
      rs, cs, zc, a.D, a.plan.Kp, c, split, amax, grp);
}

template <typename T>
void pack_qw_values(const F32Args& a, int64_t Nq, int c0, int cw, cudaStream_t s) {
  const T* x = static_cast<const T*>(a.x);
  const T* y = static_cast<const T*>(a.y);
  pack_values_qw_kernel<T, T><<<grid_for(a.B * a.N, 256), 256, 0, s>>>(
      static_cast<const T*>(a.w), y, x, a.qw, a.B, a.N, Nq, a.M, a.C, a.D, c0, cw, a.lse ? 1 : 0,
      a.src_ld > 0 ? a.src_ld : a.C);
}

cudaError_t launch_tc_f32_sum(const F32Args& a, cudaStream_t s) {
  if (a.B == 0 || a.M == 0) return cudaSuccess;
  const int Kp = a.plan.Kp;
  const float c = 0.5f * a.tau * kLog2e;
  const int64_t Nq = (a.N + 127) / 128 * 128;
  // register values for at most 3 channels per pass; the log-sum-exp one
  // channel per pass; fp16 / bf16 inputs (unsplit rows) take the register path only
  const bool reg = a.lse || a.CV <= 3;
  if (a.dt != GS_F32 && (!reg || a.plan.split)) return cudaErrorInvalidValue;
  if (a.dt == GS_F32)
    pack_operands_f32<float>(a, Nq, c, s);
  else if (a.dt == GS_F16)
    pack_operands_f32<__half>(a, Nq, c, s);
  else
    pack_operands_f32<__nv_bfloat16>(a, Nq, c, s);
  if (a.shift_mode == 1)
    add_shift_kernel<<<grid_for(a.B * a.M, 256), 256, 0, s>>>(a.rnorm, a.M, a.shift_src, a.shift_ld,
                                                             a.shift_c, a.shift_scale, a.B, a.M);
  else if (a.shift_mode == 2)
    add_shift_kernel<<<grid_for(a.B * a.N, 256), 256, 0, s>>>(a.qw, 4 * Nq, a.shift_src, a.shift_ld,
                                                             a.shift_c, a.shift_scale, a.B, a.N);
  else if (a.shift_mode != 0)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float* x = static_cast<const float*>(a.x);   // fp32 only below (tensor-core values)
  const float* y = static_cast<const float*>(a.y);
  TileMaps m;
  // 16-bit packed rows, 64 per 128-byte atom: split fp16 [hi | lo], or the
  // fp16 / bf16 inputs unsplit
  const bool sp = a.plan.split;
  const CUtensorMapDataType rdt = (!sp && a.dt == GS_BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint64_t rowe = (sp ? 2ull : 1ull) * Kp;   // elements per packed row
  const uint64_t rowb = rowe * 2ull;                // bytes per packed row
  const int atom_e = 64;
  if (!make_tmap_3d(&m.x, rdt, a.xpack, rowe, a.M, a.B, rowb, a.M * rowb, atom_e, kBM))
    return cudaErrorInvalidValue;
  const int KA = ka_for(a.plan.atoms);
  const int64_t Nst = (a.N + 7) / 8 * 8;   // fp16 rows of v^T: 16-byte multiples
  const dim3 grid(static_cast<unsigned>((a.M + kBM - 1) / kBM), static_cast<unsigned>(a.plan.splits),
                  static_cast<unsigned>(a.B));
  const int chunk = a.lse ? 1 : (reg ? 3 : a.plan.max_chunk);
  for (int c0 = 0; c0 < a.CV; c0 += chunk) {
    const int cw = (a.CV - c0) < chunk ? (a.CV - c0) : chunk;
    const int mode = reg ? (cw == 1 ? 1 : 3) : f32_chunk_pad(cw);
    if (reg) {
      if (a.dt == GS_F32)
        pack_qw_values<float>(a, Nq, c0, cw, s);
      else if (a.dt == GS_F16)
        pack_qw_values<__half>(a, Nq, c0, cw, s);
      else
        pack_qw_values<__nv_bfloat16>(a, Nq, c0, cw, s);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    const int BN = f32_tile_cols(KA, mode);
    if (BN != 32 && BN != 64 && BN != 128) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&m.y, rdt, a.ypack, rowe, a.N, a.B, rowb, a.N * rowb, atom_e, BN) ||
        !make_tmap_3d(&m.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.qw, Nq, 4, a.B, Nq * 4ull,
                      Nq * 16ull, BN, 4, false))
      return cudaErrorInvalidValue;
    if (reg) {
      m.v = m.q;   // unused
    } else {
      const int CP = mode;
      const int64_t total = a.B * CP * a.N;
      int* vmax = f32_vmax(a);
      e = cudaMemsetAsync(vmax, 0, static_cast<size_t>(a.B) * CP * sizeof(int), s);
      if (e != cudaSuccess) return e;
      {
        int64_t nb = (a.N + 255) / 256;
        const int64_t cap = (148 * 16 + a.B * CP - 1) / (a.B * CP);
        if (nb > cap) nb = cap;
        if (nb > 65535) nb = 65535;
        values_maxabs_kernel<<<dim3(static_cast<unsigned>(a.B * CP), static_cast<unsigned>(nb)), 256, 0,
                               s>>>(static_cast<const float*>(a.w), y, x, vmax, a.N, a.M, a.C, a.D,
                                    a.CV, c0, CP, a.src_ld > 0 ? a.src_ld : a.C);
      }
      pack_values_f32_split_kernel<<<grid_for(total, 256), 256, 0, s>>>(
          static_cast<const float*>(a.w), y, x, reinterpret_cast<__half*>(a.vt), vmax, a.B, a.N, Nst,
          a.M, a.C, a.D, a.CV, c0, CP, a.src_ld > 0 ? a.src_ld : a.C);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      if (!make_tmap_3d(&m.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.vt, a.N, CP, 2 * a.B, Nst * 2ull,
                        CP * Nst * 2ull, 64, CP))
        return cudaErrorInvalidValue;
    }
    F32KParams kp{};
    kp.xpack = a.xpack;
    kp.rnorm = a.rnorm;
    kp.out = a.out;
    kp.out_l = a.out_l;
    kp.split_stride = a.split_stride;
    kp.M = a.M;
    kp.N = a.N;
    kp.ldo = a.CV;
    kp.c0 = c0;
    kp.cw = cw;
    kp.cols_per_split = a.plan.cols_per_split;
    kp.ksteps = Kp / 16;
    kp.afmt = a.dt == GS_BF16 ? 1 : 0;
    kp.atoms = a.plan.atoms;
    kp.Bsz = static_cast<int>(a.B);
    kp.bn = BN;
    kp.split = a.plan.split ? 1 : 0;
    kp.two_c = a.tau * kLog2e;
    kp.amax = sp ? f32_amax(a) : nullptr;
    kp.vmax = reg ? nullptr : f32_vmax(a);
    switch (KA) {
      case 1: e = launch_mode<1>(mode, a.lse, m, kp, grid, s); break;
      case 2: e = launch_mode<2>(mode, a.lse, m, kp, grid, s); break;
      default: e = launch_mode<4>(mode, a.lse, m, kp, grid, s); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t set_test_waits_f32(uint64_t limit_ns, int stall) {
  const unsigned long long l = limit_ns;
  cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns_f32, &l, sizeof(l));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_test_stall_f32, &stall, sizeof(int));
  return e;
}

cudaError_t read_and_clear_device_error_f32(int* value) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error_f32, sizeof(int));
  if (e != cudaSuccess) return e;
  *value = v;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error_f32, &zero, sizeof(int));
  }
  return e;
}

}  // namespace gs
