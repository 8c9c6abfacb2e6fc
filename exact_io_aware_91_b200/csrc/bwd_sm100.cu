// Backward pass of exact attention on sm_100a, recomputing the probabilities
// from the saved per-row LSE instead of storing them ("Flash Attention
// uitgelegd: een uitgebreide gids", section "Recomputation"; "Flash Attention:
// Ako transformery ...", section 2, "Rekomputacia pri spatnom prechode").
//
// With P = exp(scale * Q K^T - LSE) (masked entries 0), the gradients of
// L = sum(O * dO) are (softmax Jacobian; derived, not printed on the pages):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dQ = scale * dS K,
//   dK = scale * dS^T Q,  with D_i = rowsum(dO * O)_i from the preprocess.
//
// Two persistent kernels (one CTA per SM taking 128-row work units from a work counter,
// heaviest first within groups of heads), every tensor-core product an M=128, N=128 (or
// N=d) tcgen05.mma (smaller N runs the tensor core well below its peak on sm_100a).
// Grouped-query heads and the sliding window only change which units and steps exist and
// which entries are masked.  Warp 0 streams tiles with TMA, warp 1 issues the MMAs
// (warp-convergent, one elected lane), warps 4-7 and 8-11 are two compute
// warpgroups that split every step's 128 columns in halves (one thread per TMEM
// lane = tile row, 64 columns each).
//   * dK/dV kernel (128 keys per CTA, K and V resident; 128-query steps of Q and
//     dO from two-deep rings): S^T = K Q^T and dP^T = V dO^T land in TMEM; the
//     warpgroups write P^T and dS^T back into the same TMEM columns as fp16,
//     where they feed dV += P^T dO and dK += dS^T Q directly.  MMA order per step
//     i: dV(i), S^T(i+1), dK(i), dP^T(i+1), so the elementwise work of one step
//     runs while the tensor core finishes the previous one.
//   * dQ kernel (128 queries per CTA, Q and dO resident; 128-key steps, three K
//     buffers and two V buffers): S double-buffered in TMEM; order per step j:
//     dQ(j) += dS(j) K_j, dP(j+1), S(j+2).
// All products run in fp16 with fp32 accumulation on copies of the bf16 inputs made by the
// preprocess, each exactly the input times a power of two 2^e chosen per tensor (e = 0 in
// the common case; see bwd_pre.cu); the kernels read the exponents, fold those of Q and K
// into the softmax scale and undo the others in the epilogues.  Gradients are fp32.
#include <type_traits>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kThreads = 384;
// registers per thread: 168 at launch (65536 / 384, rounded down to a multiple of 8);
// warpgroup 0 (TMA, MMA) drops to 64 and the two compute warpgroups rise to 216
constexpr uint32_t kRegsLaunch = 168, kRegsLow = 64, kRegsHigh = 216;
static_assert(kRegsLow + 2 * kRegsHigh <= 3 * kRegsLaunch, "register split exceeds the launch budget");

constexpr int kBox = 128 * 128;  // one 64-column x 128-row fp16 box (16 KB)
#ifndef FA_DKDV_EXP_FMA_PER16
#define FA_DKDV_EXP_FMA_PER16 8
#endif
// exponentials out of every 16 of the dK/dV kernel's P^T that run on the FMA pipe (multiple of 4)
constexpr int kDkdvExpFmaPer16 = FA_DKDV_EXP_FMA_PER16;
static_assert(kDkdvExpFmaPer16 % 4 == 0 && kDkdvExpFmaPer16 >= 0 && kDkdvExpFmaPer16 <= 16, "groups of four");

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
}

// SS product D (+)= A * B^T over K = Dh, both operands 128-row tiles of
// 64-column boxes; the descriptors are prebuilt, each MMA adds a constant offset.
template <int Dh>
__device__ __forceinline__ void issue_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t issue) {
#pragma unroll
  for (int k = 0; k < Dh / 16; ++k) {
    const uint32_t off = (k >> 2) * kBox + (k & 3) * 32;
    mma_ss(d_tmem, sdesc_add(a_desc, off), sdesc_add(b_desc, off), idesc, k > 0 ? 1u : 0u, issue);
  }
}

// TS product D (+)= A[tmem] * B over K = 128 rows of B (MN-major descriptor prebuilt).
// The fp16 A operand sits in two 32-column halves of a 128-column TMEM region:
// rows 0..63 of K at columns [0, 32), rows 64..127 at columns [64, 96) -- where
// the two compute warpgroups wrote them.
__device__ __forceinline__ void issue_ts_split(uint32_t d_tmem, uint32_t a_region, uint64_t b_desc, uint32_t idesc,
                                               bool acc, uint32_t issue) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t a = a_region + (k < 4 ? 8 * k : 64 + 8 * (k - 4));
    mma_ts(d_tmem, a, sdesc_add(b_desc, k * 2048), idesc, (acc || k > 0) ? 1u : 0u, issue);
  }
}

// Half of the TS product above: part 0 takes K rows {0..31, 64..95} (the first 32 columns
// each compute warpgroup writes), part 1 the rest.  `first` marks the product's first MMA
// (which overwrites D).
__device__ __forceinline__ void issue_ts_split_part(uint32_t d_tmem, uint32_t a_region, uint64_t b_desc,
                                                    uint32_t idesc, bool first, int part, uint32_t issue) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = (i & 1) + 2 * part + 4 * (i >> 1);  // part 0: 0 1 4 5, part 1: 2 3 6 7
    const uint32_t a = a_region + (k < 4 ? 8 * k : 64 + 8 * (k - 4));
    mma_ts(d_tmem, a, sdesc_add(b_desc, k * 2048), idesc, (first && i == 0) ? 0u : 1u, issue);
  }
}

// 2^E as a product of two floats, each a power of two within the normal range, so that
// x * mult * f.a * f.b scales x by mult * 2^E exactly (up to the final rounding) for the
// exponent sums of the copies (|E| <= 252); both are 1 in the common case E = 0.
struct Pow2 {
  float a, b;
};
__device__ __forceinline__ Pow2 pow2_factors(int E) {
  const int e1 = E < -126 ? -126 : (E > 126 ? 126 : E);
  int e2 = E - e1;
  e2 = e2 < -126 ? -126 : (e2 > 126 ? 126 : e2);
  return Pow2{__int_as_float((e1 + 127) << 23), __int_as_float((e2 + 127) << 23)};
}

// Coalesced store of a warp's rows: lane l holds NC fp32 values of row `row0 + l` (times
// `mult` and the factors f) to be written at dst_base + (row0 + l) * ld (in floats); see
// warp_store_rows_128b.
template <int NC>
__device__ __forceinline__ void warp_store_rows_f32(const float (&v)[NC], float* dst_base, size_t ld, int row0,
                                                    int n_rows, float mult, Pow2 f) {
  static_assert(NC % 32 == 0, "32-column chunks");
  auto sc = [&](float x) { return __float_as_uint(x * mult * f.a * f.b); };
#pragma unroll
  for (int ch = 0; ch < NC / 32; ++ch) {
    uint4 a[8];
#pragma unroll
    for (int m = 0; m < 8; ++m)
      a[m] = make_uint4(sc(v[32 * ch + 4 * m]), sc(v[32 * ch + 4 * m + 1]), sc(v[32 * ch + 4 * m + 2]),
                        sc(v[32 * ch + 4 * m + 3]));
    warp_store_rows_128b(a, reinterpret_cast<uint8_t*>(dst_base + 32 * ch), ld * sizeof(float), row0, n_rows);
  }
}

// Load 64 fp32 columns of this thread's TMEM lane (two 32-column loads, one wait; the
// destination registers are read only after the wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t u0[32], u1[32];
  tmem_ld32(taddr, u0);
  tmem_ld32(taddr + 32, u1);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    v[c] = __uint_as_float(u0[c]);
    v[32 + c] = __uint_as_float(u1[c]);
  }
}

constexpr int kSmemMax = 232448;  // dynamic shared memory of one CTA on sm_100
// The kernels declare their shared memory 1024-byte aligned and allocate at most kSmemMax; this
// checks that the aligned base leaves room for the layout (it always does with an aligned start).
template <typename L>
__device__ __forceinline__ bool smem_base_fits(uint32_t raw, uint32_t base) {
  return base - raw + (uint32_t)L::BYTES <= (uint32_t)L::SMEM_ALLOC;
}

// ============================================================================ dK / dV
template <int D>
struct DkdvLayout {
  static constexpr int KCH = D / 64;
  static constexpr int TILE = KCH * kBox;  // one 128 x D fp16 tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;        // two Q buffers
  static constexpr int OFF_DO = 4 * TILE;       // two dO buffers
  static constexpr int OFF_LD = 6 * TILE;       // two (lse2[128], delta[128]) pairs, 1 KB each
  static constexpr int OFF_STG = OFF_LD + 2048;  // epilogue: a 32-row x 128-byte box per compute warp
  static constexpr int OFF_BAR = OFF_STG + 8 * 4096;
  static constexpr int BAR_KV = 0;        // a unit's K, V landed
  static constexpr int BAR_Q_FULL = 1;    // [2]
  static constexpr int BAR_Q_EMPTY = 3;   // [2]
  static constexpr int BAR_DO_FULL = 5;   // [2]
  static constexpr int BAR_DO_EMPTY = 7;  // [2]
  static constexpr int BAR_S = 9;
  static constexpr int BAR_DP = 10;
  static constexpr int BAR_P_READY = 11;
  static constexpr int BAR_DS_READY = 12;
  static constexpr int BAR_ACC = 13;      // a unit's dV, dK complete in TMEM
  static constexpr int BAR_DONE = 14;
  static constexpr int BAR_P_HALF = 15;   // first 32 of each warpgroup's 64 P^T columns written
  static constexpr int BAR_KV_EMPTY = 16; // the MMAs reading a unit's K and V have completed
  static constexpr int BAR_ACC_FREE = 17; // the epilogue has read a unit's dV, dK out of TMEM
  static constexpr int BAR_UNIT_FULL = 18;   // [2]
  static constexpr int BAR_UNIT_EMPTY = 20;  // [2]
  static constexpr int NBAR = 22;
  static constexpr int OFF_UNIT = OFF_BAR + NBAR * 8;  // int[2]
  static constexpr int OFF_TMEM_SLOT = OFF_UNIT + 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int BYTES = OFF_ABORT + 8;
  static constexpr int SMEM_ALLOC = BYTES + 1024 <= kSmemMax ? BYTES + 1024 : kSmemMax;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;
};
static_assert(DkdvLayout<128>::BYTES <= kSmemMax, "dK/dV kernel exceeds the shared memory of a CTA");

// Persistent dK/dV kernel: one CTA per SM takes work units (key/value head, 128-key tile,
// share of the group's query heads) one after another from a work counter in the workspace
// (zeroed by the preprocess), in the order of unit_order; the producer warp takes each
// index and publishes it to the other roles through a two-slot ring in shared memory (an
// index >= the unit count means "no more work").  The next unit's K/V loads and first
// S^T, dP^T products overlap the previous unit's last steps and epilogue.  Ring positions
// (Q, dO, row statistics) and the per-step barriers count steps across units; the
// per-unit barriers (KV, KV_EMPTY, ACC, ACC_FREE) count units.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                             const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             const __grid_constant__ CUtensorMap tm_dv, const __grid_constant__ CUtensorMap tm_dk,
                             const BwdParams p) {
  using L = DkdvLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if (!smem_base_fits<L>(raw, base)) {  // cannot happen with a 1024-aligned start; report, do nothing
    if (threadIdx.x == 0) atomicExch(p.err, kDevRange);
    return;
  }
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // fa_bwd_ws: the forward's V copy now holds 2^exps[V] V (the fix-up converted it again if
  // the exponent changed); record that in the forward's workspace
  if (p.v_exp_fwd != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *p.v_exp_fwd = p.exps[kExpV];

  // heaviest first within groups of heads (see unit_order): under the causal mask the
  // first key tiles of a head meet the most query tiles
  const int n_kt = (p.N + 127) / 128;
  const int BH_kv = p.BH / p.H * p.H_kv;
  const int n_units = n_kt * BH_kv * p.kv_split;
  const int g_per = p.H / p.H_kv / p.kv_split;  // query heads per unit
  struct Unit {
    int bh, j, sp, i_start, n_q, n_it;
  };
  auto unit_of = [&](int u) -> Unit {
    Unit x;
    int rank;  // rank of (key tile, split) within the key/value head
    unit_order(u, n_kt * p.kv_split, BH_kv, p.head_group_kv, x.bh, rank);
    x.j = rank / p.kv_split;   // key tile
    x.sp = rank % p.kv_split;  // which share of the group's query heads
    // query tiles that see some key of this tile (causal mask, sliding window)
    x.i_start = query_lo(x.j * 128, p.causal, p.win_right) / 128;
    x.n_q = query_hi(min(x.j * 128 + 127, p.N - 1), p.N, p.win_left) / 128 - x.i_start + 1;  // >= 1
    x.n_it = g_per * x.n_q;    // steps: query head q_head_of(bh, sp * g_per + it / n_q), tile i_start + it % n_q
    return x;
  };
  int* unit_ring = reinterpret_cast<int*>(gbase + L::OFF_UNIT);
  auto next_unit = [&](int k, bool& ok) -> int {  // index of this CTA's k-th unit
    const int slot = k & 1;
    ok = mbar_wait(bar(L::BAR_UNIT_FULL + slot), (k >> 1) & 1, wctx);
    return ok ? *reinterpret_cast<volatile int*>(unit_ring + slot) : n_units;
  };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::BAR_KV), 1);
    mbar_init(bar(L::BAR_KV_EMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::BAR_Q_FULL + s), 1);
      mbar_init(bar(L::BAR_Q_EMPTY + s), 1);
      mbar_init(bar(L::BAR_DO_FULL + s), 1);
      mbar_init(bar(L::BAR_DO_EMPTY + s), 1);
      mbar_init(bar(L::BAR_UNIT_FULL + s), 1);
      mbar_init(bar(L::BAR_UNIT_EMPTY + s), 1 + 256);
    }
    mbar_init(bar(L::BAR_S), 1);
    mbar_init(bar(L::BAR_DP), 1);
    mbar_init(bar(L::BAR_P_READY), 256);
    mbar_init(bar(L::BAR_P_HALF), 256);
    mbar_init(bar(L::BAR_DS_READY), 256);
    mbar_init(bar(L::BAR_ACC), 1);
    mbar_init(bar(L::BAR_ACC_FREE), 256);
    mbar_init(bar(L::BAR_DONE), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::OFF_TMEM_SLOT, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::OFF_TMEM_SLOT);

  if (warp == 0) {
    // ===================================================== TMA producer + work distribution
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    int T = 0;         // Q / dO tiles issued (ring position, across units)
    int kv_issued = 0;
    bool ok = true;
    for (int uc = 0;; ++uc) {
      // the ring slot is free once every consumer has read unit uc - 2
      if (uc >= 2 && !(ok = mbar_wait(bar(L::BAR_UNIT_EMPTY + (uc & 1)), ((uc - 2) >> 1) & 1, wctx))) break;
      int u = 0;
      if (lane == 0) u = (int)atomicAdd(p.dkdv_counter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (lane == 0) {
        unit_ring[uc & 1] = u < n_units ? u : n_units;
        mbar_arrive(bar(L::BAR_UNIT_FULL + (uc & 1)));
      }
      __syncwarp();
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      // K, V of this unit replace the previous unit's once its last S^T, dP^T completed
      if (uc > 0 && !(ok = mbar_wait(bar(L::BAR_KV_EMPTY), (uc - 1) & 1, wctx))) break;
      mbar_arrive_expect_tx(bar(L::BAR_KV), 2 * L::TILE, leader);
      for (int c = 0; c < L::KCH; ++c) {
        tma_load_3d(base + L::OFF_K + c * kBox, &tm_k, c * 64, x.j * 128, x.bh, bar(L::BAR_KV), leader);
        tma_load_3d(base + L::OFF_V + c * kBox, &tm_v, c * 64, x.j * 128, x.bh, bar(L::BAR_KV), leader);
      }
      ++kv_issued;
      for (int it = 0; it < x.n_it; ++it, ++T) {
        const int s = T & 1;
        const uint32_t ph = ((T >> 1) & 1) ^ 1u;
        const int i = x.i_start + it % x.n_q;
        const int bhq = q_head_of(x.bh, x.sp * g_per + it / x.n_q, p.H, p.H_kv);
        if (!(ok = mbar_wait(bar(L::BAR_Q_EMPTY + s), ph, wctx))) break;
        const uint32_t fq = bar(L::BAR_Q_FULL + s);
        mbar_arrive_expect_tx(fq, L::TILE + 1024, leader);
        for (int c = 0; c < L::KCH; ++c)
          tma_load_3d(base + L::OFF_Q + s * L::TILE + c * kBox, &tm_q, c * 64, i * 128, bhq, fq, leader);
        const size_t roff = (size_t)bhq * p.Np + (size_t)i * 128;
        bulk_load(base + L::OFF_LD + s * 1024, p.lse2 + roff, 512, fq, leader);
        bulk_load(base + L::OFF_LD + s * 1024 + 512, p.delta + roff, 512, fq, leader);
        if (!(ok = mbar_wait(bar(L::BAR_DO_EMPTY + s), ph, wctx))) {
          ++T;  // this step's Q tile was issued
          break;
        }
        const uint32_t fd = bar(L::BAR_DO_FULL + s);
        mbar_arrive_expect_tx(fd, L::TILE, leader);
        for (int c = 0; c < L::KCH; ++c)
          tma_load_3d(base + L::OFF_DO + s * L::TILE + c * kBox, &tm_do, c * 64, i * 128, bhq, fd, leader);
      }
      if (!ok) break;
    }
    // drain: every issued copy has landed before the CTA may exit
    if (kv_issued > 0) drain_wait(bar(L::BAR_KV), (kv_issued - 1) & 1);
    for (int t = (T > 2 ? T - 2 : 0); t < T; ++t) {
      drain_wait(bar(L::BAR_Q_FULL + (t & 1)), (t >> 1) & 1);
      drain_wait(bar(L::BAR_DO_FULL + (t & 1)), (t >> 1) & 1);
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    constexpr uint32_t idesc_s = make_idesc(128, 128, false, false, false);  // M=128 keys, N=128 queries
    constexpr uint32_t idesc_g = make_idesc(128, D, false, false, true);     // N=D, B MN-major
    const uint64_t dK = make_sdesc_sw128(base + L::OFF_K, 16, 1024);
    const uint64_t dV = make_sdesc_sw128(base + L::OFF_V, 16, 1024);
    const uint64_t dQk = make_sdesc_sw128(base + L::OFF_Q, 16, 1024);      // Q as K-major B
    const uint64_t dDOk = make_sdesc_sw128(base + L::OFF_DO, 16, 1024);    // dO as K-major B
    const uint64_t dQmn = make_sdesc_sw128(base + L::OFF_Q, kBox, 1024);   // Q as MN-major B
    const uint64_t dDOmn = make_sdesc_sw128(base + L::OFF_DO, kBox, 1024); // dO as MN-major B
    // S^T(t) = K Q_t^T and dP^T(t) = V dO_t^T for global step t
    auto issue_s = [&](int t) -> bool {
      if (!mbar_wait(bar(L::BAR_Q_FULL + (t & 1)), (t >> 1) & 1, wctx)) return false;
      tc_fence_after();
      issue_ss<D>(tmem + L::T_S, dK, sdesc_add(dQk, (t & 1) * L::TILE), idesc_s, leader);
      mma_commit(bar(L::BAR_S), leader);
      return true;
    };
    auto issue_dp = [&](int t) -> bool {
      if (!mbar_wait(bar(L::BAR_DO_FULL + (t & 1)), (t >> 1) & 1, wctx)) return false;
      tc_fence_after();
      issue_ss<D>(tmem + L::T_DP, dV, sdesc_add(dDOk, (t & 1) * L::TILE), idesc_s, leader);
      mma_commit(bar(L::BAR_DP), leader);
      return true;
    };
    int T0 = 0;  // global step index of the current unit's step 0
    bool ok = true;
    for (int uc = 0; ok; ++uc) {
      const int u = next_unit(uc, ok);
      if (lane == 0) mbar_arrive(bar(L::BAR_UNIT_EMPTY + (uc & 1)));
      if (!ok || u >= n_units) break;
      const int n = unit_of(u).n_it;
      if (!(ok = mbar_wait(bar(L::BAR_KV), uc & 1, wctx))) break;
      tc_fence_after();
      if (!(ok = issue_s(T0))) break;
      if (!(ok = issue_dp(T0))) break;
      if (n == 1) mma_commit(bar(L::BAR_KV_EMPTY), leader);  // last S^T, dP^T of the unit issued
      for (int it = 0; it < n && ok; ++it) {
        const int t = T0 + it;
        const int s = t & 1;
        const uint32_t so = s * L::TILE;
        // dV += P^T dO in two halves: the first starts while the second half of P^T is computed;
        // the unit's first product overwrites the accumulators, which the previous unit's
        // epilogue must have read out of TMEM
        if (!(ok = mbar_wait(bar(L::BAR_P_HALF), t & 1, wctx))) break;
        tc_fence_after();
        if (it == 0 && uc > 0) {
          if (!(ok = mbar_wait(bar(L::BAR_ACC_FREE), (uc - 1) & 1, wctx))) break;
          tc_fence_after();
        }
        issue_ts_split_part(tmem + L::T_DV, tmem + L::T_S, sdesc_add(dDOmn, so), idesc_g, it == 0, 0, leader);
        if (!(ok = mbar_wait(bar(L::BAR_P_READY), t & 1, wctx))) break;
        tc_fence_after();
        issue_ts_split_part(tmem + L::T_DV, tmem + L::T_S, sdesc_add(dDOmn, so), idesc_g, false, 1, leader);
        mma_commit(bar(L::BAR_DO_EMPTY + s), leader);
        if (it + 1 < n && !(ok = issue_s(t + 1))) break;
        if (!(ok = mbar_wait(bar(L::BAR_DS_READY), t & 1, wctx))) break;
        tc_fence_after();
        issue_ts_split(tmem + L::T_DK, tmem + L::T_DP, sdesc_add(dQmn, so), idesc_g, it > 0, leader);  // dK += dS^T Q
        mma_commit(bar(L::BAR_Q_EMPTY + s), leader);
        if (it + 1 < n) {
          if (!(ok = issue_dp(t + 1))) break;
          if (it + 2 == n) mma_commit(bar(L::BAR_KV_EMPTY), leader);  // last S^T, dP^T of the unit issued
        }
      }
      if (!ok) break;
      mma_commit(bar(L::BAR_ACC), leader);
      T0 += n;
    }
    mma_commit(bar(L::BAR_DONE), leader);
    drain_wait(bar(L::BAR_DONE), 0);
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle
  } else {
    // ===================================================== compute warpgroups
    regs_inc<kRegsHigh>();
    const int w = (warp - 4) >> 2;   // query columns [64 w, 64 w + 64) of every step
    const int wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;  // key row inside the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::T_S + 64 * w;
    const uint32_t tDP = tmem + lane_off + L::T_DP + 64 * w;
    // the copies are Q 2^eq, K 2^ek, V 2^ev, dO 2^edo: S^T carries 2^(eq+ek), dP^T and D (and so
    // the fp16 dS^T) 2^(ev+edo), dV's accumulator 2^edo, dK's 2^(ev+edo+eq)
    const float sl2 = ldexpf(p.scale_log2, -(p.exps[kExpQ] + p.exps[kExpK]));
    const uint64_t sl2x2 = f2pack(sl2, sl2);
    bool ok = true;
    int T0 = 0;
    int u = next_unit(0, ok);
    mbar_arrive(bar(L::BAR_UNIT_EMPTY + 0));
    for (int uc = 0; ok && u < n_units; ++uc) {
      int j, i_start, n_q, n_it;
      {
        const Unit x = unit_of(u);
        j = x.j;
        i_start = x.i_start;
        n_q = x.n_q;
        n_it = x.n_it;
      }
      const int key = j * 128 + row;
      const int q_vis_lo = query_lo(key, p.causal, p.win_right);
      const int q_vis_hi = query_hi(key, p.N, p.win_left);
      // queries that every key of the tile sees: both bounds grow with the key
      const int all_lo = query_lo(min(j * 128 + 127, p.N - 1), p.causal, p.win_right);
      const int all_hi = query_hi(j * 128, p.N, p.win_left);
      for (int it = 0; it < n_it; ++it) {
        const int T = T0 + it;
        const int i = i_start + it % n_q;  // query tile of this step
        const float* lse2 = reinterpret_cast<const float*>(gbase + L::OFF_LD + (T & 1) * 1024) + 64 * w;
        const float* delta = lse2 + 128;
        const int q0 = i * 128 + 64 * w;  // first query of this warpgroup's columns
        // ---- P^T = 2^(S^T * scale * log2(e) - lse2), written back over S^T as fp16
        if (!(ok = mbar_wait(bar(L::BAR_S), T & 1, wctx))) break;
        tc_fence_after();
        float pr[64];
        tmem_ld64(tS, pr);
        // the same for every thread of the CTA: tiles inside every key's visible query range
        // take the loop without compares; the others mask column c unless c_lo <= c <= c_hi
        // (this key's visible queries; padded queries have P = 0)
        auto probs = [&](auto masked) {
          const int c_lo = q_vis_lo - q0, c_hi = q_vis_hi - q0;
#pragma unroll
          for (int g = 0; g < 64; g += 16) {
            uint32_t pk[8];
#pragma unroll
            for (int c = g; c < g + 16; c += 4) {
              const float4 L4 = *reinterpret_cast<const float4*>(lse2 + c);
              float t0, t1, t2, t3;
              f2unpack(ffma2(f2pack(pr[c], pr[c + 1]), sl2x2, f2pack(-L4.x, -L4.y)), t0, t1);
              f2unpack(ffma2(f2pack(pr[c + 2], pr[c + 3]), sl2x2, f2pack(-L4.z, -L4.w)), t2, t3);
              if ((c - g) < kDkdvExpFmaPer16) {
                // both warpgroups run this phase at once, so the MUFU unit is the limit: part of
                // the exponentials go to the FMA pipe
                exp2_fma_pipe(t0, t1);
                exp2_fma_pipe(t2, t3);
                pr[c] = t0;
                pr[c + 1] = t1;
                pr[c + 2] = t2;
                pr[c + 3] = t3;
              } else {
                pr[c] = ex2_approx(t0);
                pr[c + 1] = ex2_approx(t1);
                pr[c + 2] = ex2_approx(t2);
                pr[c + 3] = ex2_approx(t3);
              }
              if constexpr (decltype(masked)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (c + e < c_lo || c + e > c_hi) pr[c + e] = 0.f;
              }
              pk[(c - g) / 2] = pack_f16(pr[c], pr[c + 1]);
              pk[(c - g) / 2 + 1] = pack_f16(pr[c + 2], pr[c + 3]);
            }
            tmem_st8(tS + g / 2, pk);
            if (g == 16) {  // columns 0..31 of this warpgroup done: the first half of dV may start
              tmem_wait_st();
              tc_fence_before();
              mbar_arrive(bar(L::BAR_P_HALF));
            }
          }
        };
        if (q0 < all_lo || q0 + 63 > all_hi)
          probs(std::true_type{});
        else
          probs(std::false_type{});
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::BAR_P_READY));
        // ---- dS^T = P^T * (dP^T - D), written back over dP^T as fp16
        if (!(ok = mbar_wait(bar(L::BAR_DP), T & 1, wctx))) break;
        tc_fence_after();
        float dp[64];
        tmem_ld64(tDP, dp);
#pragma unroll
        for (int g = 0; g < 64; g += 16) {
          uint32_t pk[8];
#pragma unroll
          for (int c = g; c < g + 16; c += 4) {
            const float4 D4 = *reinterpret_cast<const float4*>(delta + c);
            float d0, d1, d2, d3;
            f2unpack(fmul2(f2pack(pr[c], pr[c + 1]), fsub2(f2pack(dp[c], dp[c + 1]), f2pack(D4.x, D4.y))), d0, d1);
            f2unpack(fmul2(f2pack(pr[c + 2], pr[c + 3]), fsub2(f2pack(dp[c + 2], dp[c + 3]), f2pack(D4.z, D4.w))), d2,
                     d3);
            pk[(c - g) / 2] = pack_f16(d0, d1);
            pk[(c - g) / 2 + 1] = pack_f16(d2, d3);
          }
          tmem_st8(tDP + g / 2, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::BAR_DS_READY));
      }
      if (!ok) break;
      if (!(ok = mbar_wait(bar(L::BAR_ACC), uc & 1, wctx))) break;
      tc_fence_after();
      // with the group split over several CTAs each writes its partial sums for the reduction
      // (the host points tm_dv / tm_dk at the partial buffers then)
      const Unit x = unit_of(u);
      const int head = p.kv_split == 1 ? x.bh : x.sp * BH_kv + x.bh;
      // warpgroup 0 writes dV, warpgroup 1 writes scale * dK (rows past N are padding and are
      // clipped by the bulk store), 64 columns at a time through this warp's 32-row x 128-byte
      // staging box, one bulk tensor store per 32 columns; once the last columns are loaded
      // the next unit may overwrite the accumulators
      const uint32_t t_acc = tmem + lane_off + (w == 0 ? L::T_DV : L::T_DK);
      const Pow2 out_f = pow2_factors(w == 0 ? -p.exps[kExpDO] : -(p.exps[kExpV] + p.exps[kExpDO] + p.exps[kExpQ]));
      const float mult = w == 0 ? 1.0f : p.scale;
      auto sc = [&](float v) { return __float_as_uint(v * mult * out_f.a * out_f.b); };
      const uint32_t stg = base + L::OFF_STG + (uint32_t)(warp - 4) * 4096u;
      const CUtensorMap* m_out = w == 0 ? &tm_dv : &tm_dk;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        float acc[64];
        tmem_ld64(t_acc + 64 * c, acc);
        if (c == D / 64 - 1) {
          tc_fence_before();
          mbar_arrive(bar(L::BAR_ACC_FREE));
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (lane == 0) bulk_wait_group_read0();  // the box's previous store has read it
          __syncwarp();
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float* a = acc + 32 * h + 4 * q4;
            const uint32_t addr = stg + sw128_offset(lane, q4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(sc(a[0])), "r"(sc(a[1])),
                         "r"(sc(a[2])), "r"(sc(a[3]))
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(m_out, 64 * c + 32 * h, j * 128 + wq * 32, head, stg);
            bulk_commit_group();
          }
        }
      }
      T0 += n_it;
      u = next_unit(uc + 1, ok);
      mbar_arrive(bar(L::BAR_UNIT_EMPTY + ((uc + 1) & 1)));
    }
    if (lane == 0) bulk_wait_group0();  // this warp's bulk stores are complete
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ============================================================================ dQ
template <int D>
struct DqLayout {
  static constexpr int KCH = D / 64;
  static constexpr int TILE = KCH * kBox;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_K = 2 * TILE;  // three K buffers
  static constexpr int OFF_V = 5 * TILE;  // two V buffers
  static constexpr int OFF_BAR = 7 * TILE;
  static constexpr int BAR_Q = 0;        // Q and dO of a unit landed
  static constexpr int BAR_K_FULL = 1;   // [3]
  static constexpr int BAR_K_EMPTY = 4;  // [3]
  static constexpr int BAR_V_FULL = 7;   // [2]
  static constexpr int BAR_V_EMPTY = 9;  // [2]
  static constexpr int BAR_S = 11;       // [2]
  static constexpr int BAR_DP = 13;
  static constexpr int BAR_DS = 14;      // [2]
  static constexpr int BAR_ACC = 16;     // a unit's dQ complete in TMEM
  static constexpr int BAR_DONE = 17;
  static constexpr int BAR_Q_EMPTY = 18; // the MMAs reading a unit's Q and dO have completed
  static constexpr int BAR_DQ_FREE = 19; // the epilogue has read a unit's dQ out of TMEM
  static constexpr int BAR_UNIT_FULL = 20;   // [2] next work unit index published
  static constexpr int BAR_UNIT_EMPTY = 22;  // [2] ... and read by the MMA warp and both warpgroups
  static constexpr int BAR_DP_LOADED = 24;   // the step's dP is in the compute warps' registers
  static constexpr int NBAR = 25;
  static constexpr int OFF_UNIT = OFF_BAR + NBAR * 8;  // int[2]: work unit ring
  static constexpr int OFF_TMEM_SLOT = OFF_UNIT + 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM_ALLOC = OFF_ABORT + 8 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 256, T_DQ = 384;  // S buffer b at T_S + 128 b
};

// Persistent dQ kernel: one CTA per SM takes work units one after another, so that one
// unit's epilogue and the next unit's loads and first MMAs overlap instead of paying a CTA
// launch, barrier and TMEM set-up and a pipeline fill per unit.  Units are handed out
// dynamically in the order of unit_order (heaviest first within L2-sized head groups): the
// producer warp takes the next index from a global counter (zeroed by the preprocess
// kernel) and publishes it to the other roles through a two-slot ring in shared memory;
// an index >= the unit count means "no more work".  Ring positions (K, V, S, dS, dP) count
// steps across units; per-unit barriers (Q, Q_EMPTY, ACC, DQ_FREE) count units.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const BwdParams p) {
  // exponentials out of every 16 of P that run on the FMA pipe (even): a quarter measured
  // 1.3-2 % faster than none on B200 (N = 8192 / 2048), a half slower
#ifndef FA_DQ_EXP_FMA_PER16
#define FA_DQ_EXP_FMA_PER16 4
#endif
  constexpr int kDqExpFmaPer16 = FA_DQ_EXP_FMA_PER16;
  static_assert(kDqExpFmaPer16 % 2 == 0 && kDqExpFmaPer16 >= 0 && kDqExpFmaPer16 <= 16, "pairs");
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heaviest first within groups of heads (see unit_order): under the causal mask the
  // last query tiles of a head meet the most key tiles
  const int nq = (p.N + 127) / 128;
  const int n_units = nq * p.BH;
  struct Unit {
    int bh, bh_kv, qt, jlo, n_it;
  };
  auto unit_of = [&](int u) -> Unit {
    Unit x;
    int rank;
    unit_order(u, nq, p.BH, p.head_group, x.bh, rank);
    x.bh_kv = kv_head_of(x.bh, p.H, p.H_kv);  // the key/value head this query head reads
    x.qt = p.causal ? (nq - 1 - rank) : rank;
    // key tiles this query tile sees (causal mask, sliding window): 128-key steps
    x.jlo = key_lo(x.qt * 128, p.N, p.win_left) / 128;
    x.n_it = key_hi(x.qt * 128 + 127, p.N, p.causal, p.win_right) / 128 - x.jlo + 1;
    return x;
  };

  int* unit_ring = reinterpret_cast<int*>(gbase + L::OFF_UNIT);
  // index of the k-th unit of this CTA (all roles call it in the same order, k = 0, 1, ...)
  auto next_unit = [&](int k, bool& ok) -> int {
    const int slot = k & 1;
    ok = mbar_wait(bar(L::BAR_UNIT_FULL + slot), (k >> 1) & 1, wctx);
    const int u = ok ? *reinterpret_cast<volatile int*>(unit_ring + slot) : n_units;
    return u;
  };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::BAR_Q), 1);
    mbar_init(bar(L::BAR_Q_EMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::BAR_UNIT_FULL + s), 1);
      mbar_init(bar(L::BAR_UNIT_EMPTY + s), 1 + 256);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar(L::BAR_K_FULL + s), 1);
      mbar_init(bar(L::BAR_K_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::BAR_V_FULL + s), 1);
      mbar_init(bar(L::BAR_V_EMPTY + s), 1);
      mbar_init(bar(L::BAR_S + s), 1);
      mbar_init(bar(L::BAR_DS + s), 256);
    }
    mbar_init(bar(L::BAR_DP), 1);
    mbar_init(bar(L::BAR_DP_LOADED), 256);
    mbar_init(bar(L::BAR_ACC), 1);
    mbar_init(bar(L::BAR_DQ_FREE), 256);
    mbar_init(bar(L::BAR_DONE), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::OFF_TMEM_SLOT, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::OFF_TMEM_SLOT);

  if (warp == 0) {
    // ===================================================== TMA producer
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    int T = 0;   // K/V tiles issued (ring position, across units)
    int uc = 0;  // units started
    int q_issued = 0;
    bool ok = true;
    for (;; ++uc) {
      // take the next unit and publish it (slot free once every consumer read unit uc - 2)
      if (uc >= 2 && !(ok = mbar_wait(bar(L::BAR_UNIT_EMPTY + (uc & 1)), ((uc - 2) >> 1) & 1, wctx))) break;
      int u = 0;
      if (lane == 0) u = (int)atomicAdd(p.dq_counter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (lane == 0) {
        unit_ring[uc & 1] = u < n_units ? u : n_units;
        mbar_arrive(bar(L::BAR_UNIT_FULL + (uc & 1)));
      }
      __syncwarp();
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      // Q, dO of this unit overwrite the previous unit's once its last S and dP MMAs are done
      if (uc > 0 && !(ok = mbar_wait(bar(L::BAR_Q_EMPTY), (uc - 1) & 1, wctx))) break;
      mbar_arrive_expect_tx(bar(L::BAR_Q), 2 * L::TILE, leader);
      for (int c = 0; c < L::KCH; ++c) {
        tma_load_3d(base + L::OFF_Q + c * kBox, &tm_q, c * 64, x.qt * 128, x.bh, bar(L::BAR_Q), leader);
        tma_load_3d(base + L::OFF_DO + c * kBox, &tm_do, c * 64, x.qt * 128, x.bh, bar(L::BAR_Q), leader);
      }
      ++q_issued;
      for (int it = 0; it < x.n_it; ++it, ++T) {
        const int sk = T % 3, sv = T & 1;
        if (!(ok = mbar_wait(bar(L::BAR_K_EMPTY + sk), ((T / 3) & 1) ^ 1u, wctx))) break;
        mbar_arrive_expect_tx(bar(L::BAR_K_FULL + sk), L::TILE, leader);
        for (int c = 0; c < L::KCH; ++c)
          tma_load_3d(base + L::OFF_K + sk * L::TILE + c * kBox, &tm_k, c * 64, (x.jlo + it) * 128, x.bh_kv,
                      bar(L::BAR_K_FULL + sk), leader);
        if (!(ok = mbar_wait(bar(L::BAR_V_EMPTY + sv), ((T >> 1) & 1) ^ 1u, wctx))) {
          ++T;  // the K tile of this step was issued
          break;
        }
        mbar_arrive_expect_tx(bar(L::BAR_V_FULL + sv), L::TILE, leader);
        for (int c = 0; c < L::KCH; ++c)
          tma_load_3d(base + L::OFF_V + sv * L::TILE + c * kBox, &tm_v, c * 64, (x.jlo + it) * 128, x.bh_kv,
                      bar(L::BAR_V_FULL + sv), leader);
      }
    }
    // drain: every issued copy has landed before the CTA may exit
    if (q_issued > 0) drain_wait(bar(L::BAR_Q), (q_issued - 1) & 1);
    for (int t = (T > 3 ? T - 3 : 0); t < T; ++t) drain_wait(bar(L::BAR_K_FULL + t % 3), (t / 3) & 1);
    for (int t = (T > 2 ? T - 2 : 0); t < T; ++t) drain_wait(bar(L::BAR_V_FULL + (t & 1)), (t >> 1) & 1);
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    constexpr uint32_t idesc_s = make_idesc(128, 128, false, false, false);  // M=128 queries, N=128 keys
    constexpr uint32_t idesc_g = make_idesc(128, D, false, false, true);
    const uint64_t dQd = make_sdesc_sw128(base + L::OFF_Q, 16, 1024);
    const uint64_t dDO = make_sdesc_sw128(base + L::OFF_DO, 16, 1024);
    const uint64_t dKk = make_sdesc_sw128(base + L::OFF_K, 16, 1024);      // K as K-major B
    const uint64_t dVk = make_sdesc_sw128(base + L::OFF_V, 16, 1024);      // V as K-major B
    const uint64_t dKmn = make_sdesc_sw128(base + L::OFF_K, kBox, 1024);   // K as MN-major B
    int T0 = 0;  // global step index of the current unit's step 0
    // S(t) = Q K_t^T into S buffer t & 1 (t global)
    auto issue_s = [&](int t) -> bool {
      if (!mbar_wait(bar(L::BAR_K_FULL + t % 3), (t / 3) & 1, wctx)) return false;
      tc_fence_after();
      issue_ss<D>(tmem + L::T_S + 128 * (t & 1), dQd, sdesc_add(dKk, (t % 3) * L::TILE), idesc_s, leader);
      mma_commit(bar(L::BAR_S + (t & 1)), leader);
      return true;
    };
    // dP(t) = dO V_t^T
    auto issue_dp = [&](int t) -> bool {
      if (!mbar_wait(bar(L::BAR_V_FULL + (t & 1)), (t >> 1) & 1, wctx)) return false;
      tc_fence_after();
      issue_ss<D>(tmem + L::T_DP, dDO, sdesc_add(dVk, (t & 1) * L::TILE), idesc_s, leader);
      mma_commit(bar(L::BAR_DP), leader);
      mma_commit(bar(L::BAR_V_EMPTY + (t & 1)), leader);
      return true;
    };
    bool ok = true;
    for (int uc = 0;; ++uc) {
      const int u = next_unit(uc, ok);
      if (lane == 0) mbar_arrive(bar(L::BAR_UNIT_EMPTY + (uc & 1)));
      if (!ok || u >= n_units) break;
      const int n = unit_of(u).n_it;
      if (!(ok = mbar_wait(bar(L::BAR_Q), uc & 1, wctx))) break;
      tc_fence_after();
      if (!(ok = issue_s(T0))) break;
      if (!(ok = issue_dp(T0))) break;
      if (n > 1 && !(ok = issue_s(T0 + 1))) break;
      // the last MMAs that read this unit's Q / dO: S(n-1) and dP(n-1)
      if (n == 1) mma_commit(bar(L::BAR_Q_EMPTY), leader);
      for (int it = 0; it < n && ok; ++it) {
        const int t = T0 + it;
        const int b = t & 1;
        // dP(t + 1) as soon as the compute warps hold dP(t) in registers (dS goes over S)
        if (it + 1 < n) {
          if (!(ok = mbar_wait(bar(L::BAR_DP_LOADED), t & 1, wctx))) break;
          if (!(ok = issue_dp(t + 1))) break;
        }
        if (!(ok = mbar_wait(bar(L::BAR_DS + b), (t >> 1) & 1, wctx))) break;
        tc_fence_after();
        // the first dQ MMA of a unit overwrites the accumulator: the previous unit's epilogue
        // must have read it out of TMEM
        if (it == 0 && uc > 0) {
          if (!(ok = mbar_wait(bar(L::BAR_DQ_FREE), (uc - 1) & 1, wctx))) break;
          tc_fence_after();
        }
        issue_ts_split(tmem + L::T_DQ, tmem + L::T_S + 128 * b, sdesc_add(dKmn, (t % 3) * L::TILE), idesc_g, it > 0,
                       leader);  // dQ += dS K
        mma_commit(bar(L::BAR_K_EMPTY + t % 3), leader);
        if (it + 2 < n && !(ok = issue_s(t + 2))) break;
        if (it + 2 == n) mma_commit(bar(L::BAR_Q_EMPTY), leader);  // S(n-1), dP(n-1) issued
      }
      if (ok) mma_commit(bar(L::BAR_ACC), leader);
      T0 += n;
    }
    mma_commit(bar(L::BAR_DONE), leader);
    drain_wait(bar(L::BAR_DONE), 0);
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle
  } else {
    // ===================================================== compute warpgroups
    regs_inc<kRegsHigh>();
    const int w = (warp - 4) >> 2;   // key columns [64 w, 64 w + 64) of every step
    const int wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    // copies Q 2^eq, K 2^ek, V 2^ev, dO 2^edo: S carries 2^(eq+ek), dP and D (and the fp16 dS)
    // 2^(ev+edo), dQ's accumulator 2^(ev+edo+ek)
    const float sl2 = ldexpf(p.scale_log2, -(p.exps[kExpQ] + p.exps[kExpK]));
    const uint64_t sl2x2 = f2pack(sl2, sl2);
    bool ok = true;
    int T0 = 0;
    // this row's lse2 and delta, loaded one unit ahead (during the previous unit's epilogue)
    float lse2 = 0.f, delta = 0.f;
    int u = next_unit(0, ok);
    mbar_arrive(bar(L::BAR_UNIT_EMPTY + 0));
    if (ok && u < n_units) {
      const Unit x0 = unit_of(u);
      const size_t prow = (size_t)x0.bh * p.Np + x0.qt * 128 + row;  // < BH * Np (Np is a multiple of 128)
      lse2 = p.lse2[prow];
      delta = p.delta[prow];
    }
    for (int uc = 0; ok && u < n_units; ++uc) {
      const Unit x = unit_of(u);
      const int r = x.qt * 128 + row;  // query index
      const int k_vis_lo = key_lo(r, p.N, p.win_left);  // visible keys of this row
      const int k_vis_hi = key_hi(r, p.N, p.causal, p.win_right);
      // keys that every row of the tile sees: both bounds grow with the row
      const int all_lo = key_lo(min(x.qt * 128 + 127, p.N - 1), p.N, p.win_left);
      const int all_hi = key_hi(x.qt * 128, p.N, p.causal, p.win_right);
      const uint64_t nl2 = f2pack(-lse2, -lse2), dd = f2pack(delta, delta);
      for (int it = 0; it < x.n_it; ++it) {
        const int t = T0 + it;
        const int b = t & 1;
        const uint32_t tS = tmem + lane_off + L::T_S + 128 * b + 64 * w;
        const int k0 = (x.jlo + it) * 128 + 64 * w;  // first key of this warpgroup's columns
        if (!(ok = mbar_wait(bar(L::BAR_S + b), (t >> 1) & 1, wctx))) break;
        tc_fence_after();
        float pr[64];
        tmem_ld64(tS, pr);
        // the same for every thread of the CTA: tiles inside every row's visible range take
        // the loop without compares; the others mask column c unless c_lo <= c <= c_hi
        auto probs = [&](auto masked) {
          const int c_lo = k_vis_lo - k0, c_hi = k_vis_hi - k0;
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float t0, t1;
            f2unpack(ffma2(f2pack(pr[c], pr[c + 1]), sl2x2, nl2), t0, t1);
            if ((c & 15) < kDqExpFmaPer16) {  // part of the exponentials on the FMA pipe
              exp2_fma_pipe(t0, t1);
              pr[c] = t0;
              pr[c + 1] = t1;
            } else {
              pr[c] = ex2_approx(t0);
              pr[c + 1] = ex2_approx(t1);
            }
            if constexpr (decltype(masked)::value) {
              if (c < c_lo || c > c_hi) pr[c] = 0.f;
              if (c + 1 < c_lo || c + 1 > c_hi) pr[c + 1] = 0.f;
            }
          }
        };
        if (k0 < all_lo || k0 + 63 > all_hi)
          probs(std::true_type{});
        else
          probs(std::false_type{});
        if (!(ok = mbar_wait(bar(L::BAR_DP), t & 1, wctx))) break;
        tc_fence_after();
        float dp[64];
        tmem_ld64(tmem + lane_off + L::T_DP + 64 * w, dp);
        tc_fence_before();
        mbar_arrive(bar(L::BAR_DP_LOADED));  // dP(t + 1) may overwrite dP
#pragma unroll
        for (int g = 0; g < 64; g += 16) {
          uint32_t pk[8];
#pragma unroll
          for (int c = g; c < g + 16; c += 2) {
            float d0, d1;
            f2unpack(fmul2(f2pack(pr[c], pr[c + 1]), fsub2(f2pack(dp[c], dp[c + 1]), dd)), d0, d1);
            pk[(c - g) / 2] = pack_f16(d0, d1);
          }
          tmem_st8(tS + g / 2, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::BAR_DS + b));
      }
      if (!ok) break;
      if (!(ok = mbar_wait(bar(L::BAR_ACC), uc & 1, wctx))) break;
      tc_fence_after();
      // each warpgroup writes half of the columns of scale * dQ: read them out of TMEM,
      // release the accumulator to the next unit, then store
      float acc[D / 2];
      if constexpr (D == 128) {
        tmem_ld64(tmem + lane_off + L::T_DQ + w * 64, acc);
      } else {
        uint32_t uu[32];
        tmem_ld32(tmem + lane_off + L::T_DQ + w * 32, uu);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) acc[c] = __uint_as_float(uu[c]);
      }
      tc_fence_before();
      mbar_arrive(bar(L::BAR_DQ_FREE));
      const int u_next = next_unit(uc + 1, ok);  // published long before: the producer runs ahead
      mbar_arrive(bar(L::BAR_UNIT_EMPTY + ((uc + 1) & 1)));
      if (ok && u_next < n_units) {  // prefetch the next unit's row statistics
        const Unit xn = unit_of(u_next);
        const size_t prow = (size_t)xn.bh * p.Np + xn.qt * 128 + row;
        lse2 = p.lse2[prow];
        delta = p.delta[prow];
      }
      // this warp's 32 query rows, columns [w D/2, (w + 1) D/2) of scale * dQ
      const Pow2 out_f = pow2_factors(-(p.exps[kExpV] + p.exps[kExpDO] + p.exps[kExpK]));
      warp_store_rows_f32<D / 2>(acc, p.dq + (size_t)x.bh * p.N * D + w * (D / 2), D, x.qt * 128 + wq * 32, p.N,
                                 p.scale, out_f);
      T0 += x.n_it;
      u = u_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ============================================================================ head dim 256
// At d = 256 the accumulators do not fit next to S^T and dP^T in tensor memory (dV and dK of
// a 128-key tile take 256 columns each), and the tiles do not fit in shared memory (K, V, Q
// and dO of 128 rows take 64 KB each).  The two kernels below therefore:
//   * dK/dV: two kernels, one per gradient, each accumulating it over the full d in 256 TMEM
//     columns; a work unit is (key/value head, 128-key tile, share of the group's query heads).
//     The dV kernel computes S^T = K Q^T (double-buffered: two 128-column buffers) and
//     dV += P^T dO; the dK kernel S^T, dP^T = V dO^T and dK += dS^T Q.  Per (key tile, query
//     tile) pair that is 5 products of 128 x 128 x 256 (S^T in both kernels) where one unit
//     accumulating half of both gradients needs 6 (S^T and dP^T once per half).  K (and V in the
//     dK kernel) stay resident (64 KB each); Q and dO stream as 128-column halves (32 KB)
//     through a FIFO of 3 slots, 5 in the dV kernel (V's space), in the order the products take
//     them (the dK kernel loads Q a second time for dK), so the FIFO releases slots in the
//     order it fills them.
//   * dQ: Q and dO stay resident; S is single-buffered (S, dP 128 columns, dQ 256); K and V
//     stream as halves through the same kind of FIFO, K's halves a second time for dQ += dS K.
// Both are persistent like the d = 128 kernels; every other step (recomputed probabilities,
// masks, grouped heads, windows, work order, coalesced epilogues) is the same.
constexpr int kHalf = 2 * kBox;  // 128 rows x 128 fp16 columns (two 64-column boxes), 32 KB
constexpr int kWSlots = 3;       // FIFO slots of one half each

// SS product D (+)= A * B^T over K = 128 (one half of d): `first` marks the first product into D.
__device__ __forceinline__ void issue_ss_half(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              bool first, uint32_t issue) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t off = (k >> 2) * kBox + (k & 3) * 32;
    mma_ss(d_tmem, sdesc_add(a_desc, off), sdesc_add(b_desc, off), idesc, (first && k == 0) ? 0u : 1u, issue);
  }
}

// One gradient per kernel: KIND 0 = dV, KIND 1 = dK (units of the other kind run in the other
// launch).  A dV unit needs K but not V, so its Q / dO ring takes V's 64 KB as two more slots.
template <int KIND>
struct DkdvWLayout {
  static constexpr int SLOTS = KIND == 0 ? 5 : 3;  // FIFO slots of one half each
  static constexpr int OFF_K = 0;                      // K: two halves
  static constexpr int OFF_V = 2 * kHalf;              // V: two halves (dK), ring slots 3-4 (dV)
  static constexpr int OFF_RING = 4 * kHalf;           // ring slots 0-2
  static constexpr int OFF_LD = OFF_RING + 3 * kHalf;  // two (lse2[128], delta[128]) pairs, 1 KB each
  static constexpr int OFF_BAR = OFF_LD + 2048;
  static constexpr int BAR_KV = 0;          // a unit's K (and V) landed
  static constexpr int BAR_KV_EMPTY = 1;    // the MMAs reading a unit's K and V have completed
  static constexpr int BAR_SLOT_FULL = 2;                  // [SLOTS]
  static constexpr int BAR_SLOT_EMPTY = 2 + SLOTS;         // [SLOTS]
  static constexpr int BAR_LD_EMPTY = 2 + 2 * SLOTS;       // [2] the step whose LSE / D a buffer holds is finished
  static constexpr int BAR_S = BAR_LD_EMPTY + 2;           // [2] S^T of a step complete in buffer b (dV: two buffers)
  static constexpr int BAR_DP = BAR_S + 2;                 // dP^T complete (dK)
  static constexpr int BAR_S_LOADED = BAR_DP + 1;          // the compute warps hold S^T in registers (dK)
  static constexpr int BAR_P_HALF = BAR_S_LOADED + 1;      // [2] the first half of P^T is in buffer b (dV)
  static constexpr int BAR_P_READY = BAR_P_HALF + 2;       // [2] all of P^T is in buffer b (dV)
  static constexpr int BAR_DS_READY = BAR_P_READY + 2;     // dS^T is in TMEM over dP^T (dK)
  static constexpr int BAR_ACC = BAR_DS_READY + 1;
  static constexpr int BAR_ACC_FREE = BAR_ACC + 1;
  static constexpr int BAR_UNIT_FULL = BAR_ACC_FREE + 1;   // [2]
  static constexpr int BAR_UNIT_EMPTY = BAR_UNIT_FULL + 2; // [2]
  static constexpr int BAR_DONE = BAR_UNIT_EMPTY + 2;
  static constexpr int NBAR = BAR_DONE + 1;
  static constexpr int OFF_UNIT = OFF_BAR + NBAR * 8;  // int[2]
  static constexpr int OFF_TMEM_SLOT = OFF_UNIT + 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int BYTES = OFF_ABORT + 8;
  // the base is rounded up to 1024 bytes inside the allocation; the kernel checks that the
  // rounding fits (it does for a 1024-aligned start, which the declaration asks for)
  static constexpr int SMEM_ALLOC = BYTES + 1024 <= kSmemMax ? BYTES + 1024 : kSmemMax;
  static constexpr uint32_t TMEM_COLS = 512;
  // dV: S^T buffers at 0 and 128; dK: S^T at 0, dP^T at 128; the gradient (256 columns) at 256
  static constexpr uint32_t T_S = 0, T_DP = 128, T_ACC = 256;
  // byte offset of ring slot st from the shared-memory base
  __device__ static uint32_t slot_off(int st) {
    return (KIND == 0 && st >= 3) ? (uint32_t)(OFF_V + (st - 3) * kHalf) : (uint32_t)(OFF_RING + st * kHalf);
  }
};
static_assert(DkdvWLayout<0>::BYTES <= kSmemMax && DkdvWLayout<1>::BYTES <= kSmemMax,
              "d = 256 dK/dV kernels exceed the shared memory of a CTA");


template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dkdv_d256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            const BwdParams p) {
  using L = DkdvWLayout<KIND>;
  constexpr int D = 256;
  constexpr int SL = L::SLOTS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if (!smem_base_fits<L>(raw, base)) {  // cannot happen with a 1024-aligned start; report, do nothing
    if (threadIdx.x == 0) atomicExch(p.err, kDevRange);
    return;
  }
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (KIND == 1 && p.v_exp_fwd != nullptr && blockIdx.x == 0 && threadIdx.x == 0)
    *p.v_exp_fwd = p.exps[kExpV];  // as above

  const int n_kt = (p.N + 127) / 128;
  const int BH_kv = p.BH / p.H * p.H_kv;
  const int per_head = n_kt * p.kv_split;  // (key tile, split) per key/value head
  const int n_units = per_head * BH_kv;
  const int g_per = p.H / p.H_kv / p.kv_split;
  struct Unit {
    int bh, j, sp, i_start, n_q, n_it;
  };
  auto unit_of = [&](int u) -> Unit {
    Unit x;
    int rank;
    unit_order(u, per_head, BH_kv, p.head_group_kv, x.bh, rank);
    x.j = rank / p.kv_split;  // heaviest (first) key tiles first
    x.sp = rank % p.kv_split;
    x.i_start = query_lo(x.j * 128, p.causal, p.win_right) / 128;
    x.n_q = query_hi(min(x.j * 128 + 127, p.N - 1), p.N, p.win_left) / 128 - x.i_start + 1;
    x.n_it = g_per * x.n_q;
    return x;
  };
  int* unit_ring = reinterpret_cast<int*>(gbase + L::OFF_UNIT);
  auto next_unit = [&](int k, bool& ok) -> int {
    const int slot = k & 1;
    ok = mbar_wait(bar(L::BAR_UNIT_FULL + slot), (k >> 1) & 1, wctx);
    return ok ? *reinterpret_cast<volatile int*>(unit_ring + slot) : n_units;
  };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::BAR_KV), 1);
    mbar_init(bar(L::BAR_KV_EMPTY), 1);
    for (int s = 0; s < SL; ++s) {
      mbar_init(bar(L::BAR_SLOT_FULL + s), 1);
      mbar_init(bar(L::BAR_SLOT_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::BAR_LD_EMPTY + s), 1);
      mbar_init(bar(L::BAR_S + s), 1);
      mbar_init(bar(L::BAR_P_HALF + s), 256);
      mbar_init(bar(L::BAR_P_READY + s), 256);
      mbar_init(bar(L::BAR_UNIT_FULL + s), 1);
      mbar_init(bar(L::BAR_UNIT_EMPTY + s), 1 + 256);
    }
    mbar_init(bar(L::BAR_DP), 1);
    mbar_init(bar(L::BAR_S_LOADED), 256);
    mbar_init(bar(L::BAR_DS_READY), 256);
    mbar_init(bar(L::BAR_ACC), 1);
    mbar_init(bar(L::BAR_ACC_FREE), 256);
    mbar_init(bar(L::BAR_DONE), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::OFF_TMEM_SLOT, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::OFF_TMEM_SLOT);

  // The FIFO order of a unit with n steps (Xk(t) = half k of X for step t), which the producer
  // fills and the MMA warp drains:
  //   dV: Q0(0) Q1(0) [Q0(1) Q1(1)], then for it = 0..n-1: dO0(it) dO1(it) [Q0(it+2) Q1(it+2)]
  //   dK: Q0(0) Q1(0) dO0(0) dO1(0), then for it = 0..n-1:
  //       [Q0(it+1) Q1(it+1)] Q0(it) Q1(it) [dO0(it+1) dO1(it+1)]
  // (bracketed parts only while those steps exist).  The dK products take Q(it) one half at a
  // time, so each product holds at most one slot and the loads run ahead of the products.
  if (warp == 0) {
    // ===================================================== TMA producer + work distribution
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_k);
    if (KIND == 1) prefetch_tmap(&tm_v);
    int F = 0;  // halves put in the FIFO so far (all units)
    int T = 0;  // steps of the previous units
    int kv_issued = 0;
    bool ok = true;
    // half `half` of Q (which = 0) or dO (which = 1) for the unit step `it`; with_ld: also the
    // step's LSE * log2(e) and D rows (global step t) into their buffer
    auto load_half = [&](const Unit& x, int which, int half, int it, bool with_ld) -> bool {
      const int st = F % SL;
      if (!mbar_wait(bar(L::BAR_SLOT_EMPTY + st), ((F / SL) & 1) ^ 1u, wctx)) return false;
      const int t = T + it;
      const int i = x.i_start + it % x.n_q;
      const int bhq = q_head_of(x.bh, x.sp * g_per + it / x.n_q, p.H, p.H_kv);
      if (with_ld && t >= 2 && !mbar_wait(bar(L::BAR_LD_EMPTY + (t & 1)), ((t >> 1) - 1) & 1, wctx)) return false;
      const uint32_t fb = bar(L::BAR_SLOT_FULL + st);
      mbar_arrive_expect_tx(fb, kHalf + (with_ld ? 1024 : 0), leader);
      const CUtensorMap* m = which ? &tm_do : &tm_q;
      const uint32_t dst = base + L::slot_off(st);
      for (int b = 0; b < 2; ++b) tma_load_3d(dst + b * kBox, m, half * 128 + b * 64, i * 128, bhq, fb, leader);
      if (with_ld) {
        const size_t roff = (size_t)bhq * p.Np + (size_t)i * 128;
        bulk_load(base + L::OFF_LD + (t & 1) * 1024, p.lse2 + roff, 512, fb, leader);
        bulk_load(base + L::OFF_LD + (t & 1) * 1024 + 512, p.delta + roff, 512, fb, leader);
      }
      ++F;
      return true;
    };
    auto load_both = [&](const Unit& x, int which, int it) -> bool {  // both halves; Q's first carries LSE / D
      return load_half(x, which, 0, it, which == 0) && load_half(x, which, 1, it, false);
    };
    for (int uc = 0;; ++uc) {
      if (uc >= 2 && !(ok = mbar_wait(bar(L::BAR_UNIT_EMPTY + (uc & 1)), ((uc - 2) >> 1) & 1, wctx))) break;
      int u = 0;
      if (lane == 0) u = (int)atomicAdd(KIND == 0 ? p.dkdv_counter : p.dk_counter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (lane == 0) {
        unit_ring[uc & 1] = u < n_units ? u : n_units;
        mbar_arrive(bar(L::BAR_UNIT_FULL + (uc & 1)));
      }
      __syncwarp();
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      if (uc > 0 && !(ok = mbar_wait(bar(L::BAR_KV_EMPTY), (uc - 1) & 1, wctx))) break;
      mbar_arrive_expect_tx(bar(L::BAR_KV), (KIND == 1 ? 4 : 2) * kHalf, leader);
      for (int c = 0; c < 4; ++c) {
        const uint32_t off = (c >> 1) * kHalf + (c & 1) * kBox;
        tma_load_3d(base + L::OFF_K + off, &tm_k, c * 64, x.j * 128, x.bh, bar(L::BAR_KV), leader);
        if (KIND == 1) tma_load_3d(base + L::OFF_V + off, &tm_v, c * 64, x.j * 128, x.bh, bar(L::BAR_KV), leader);
      }
      ++kv_issued;
      const int n = x.n_it;
      if (KIND == 0) {
        ok = load_both(x, 0, 0) && (n < 2 || load_both(x, 0, 1));
        for (int it = 0; it < n && ok; ++it) ok = load_both(x, 1, it) && (it + 2 >= n || load_both(x, 0, it + 2));
      } else {
        ok = load_both(x, 0, 0) && load_both(x, 1, 0);
        for (int it = 0; it < n && ok; ++it)
          ok = (it + 1 >= n || load_both(x, 0, it + 1)) && load_half(x, 0, 0, it, false) &&
               load_half(x, 0, 1, it, false) && (it + 1 >= n || load_both(x, 1, it + 1));
      }
      if (!ok) break;
      T += n;
    }
    // drain: every issued copy has landed before the CTA may exit
    if (kv_issued > 0) drain_wait(bar(L::BAR_KV), (kv_issued - 1) & 1);
    for (int f = (F > SL ? F - SL : 0); f < F; ++f) drain_wait(bar(L::BAR_SLOT_FULL + f % SL), (f / SL) & 1);
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    constexpr uint32_t idesc_s = make_idesc(128, 128, false, false, false);  // M=128 keys, N=128 queries
    constexpr uint32_t idesc_g = make_idesc(128, 128, false, false, true);   // N=128 (a d-half), B MN-major
    const uint64_t dKs[2] = {make_sdesc_sw128(base + L::OFF_K, 16, 1024),
                             make_sdesc_sw128(base + L::OFF_K + kHalf, 16, 1024)};
    const uint64_t dVs[2] = {make_sdesc_sw128(base + L::OFF_V, 16, 1024),
                             make_sdesc_sw128(base + L::OFF_V + kHalf, 16, 1024)};
    int C = 0;  // halves taken from the FIFO so far
    bool ok = true;
    auto take = [&]() -> int {
      const int st = C % SL;
      ok = mbar_wait(bar(L::BAR_SLOT_FULL + st), (C / SL) & 1, wctx);
      ++C;
      if (ok) tc_fence_after();
      return st;
    };
    // S^T = K Q^T (or dP^T = V dO^T) over both d-halves, each half taken from the FIFO
    auto issue_full = [&](uint32_t d_tmem, const uint64_t (&a)[2], uint32_t done_bar) -> bool {
      for (int hh = 0; hh < 2; ++hh) {
        const int st = take();
        if (!ok) return false;
        issue_ss_half(d_tmem, a[hh], make_sdesc_sw128(base + L::slot_off(st), 16, 1024), idesc_s, hh == 0, leader);
        mma_commit(bar(L::BAR_SLOT_EMPTY + st), leader);
      }
      mma_commit(done_bar, leader);
      return true;
    };
    // a slot's half as the MN-major B operand of a gradient product
    auto mn_desc = [&](int st) -> uint64_t { return make_sdesc_sw128(base + L::slot_off(st), kBox, 1024); };
    int T0 = 0;
    int nP[2] = {0, 0};    // dV: steps that used S^T buffer b so far (P_HALF / P_READY phases)
    int nSL = 0, nDS = 0;  // dK: S_LOADED and DS_READY phases so far
    for (int uc = 0; ok; ++uc) {
      const int u = next_unit(uc, ok);
      if (lane == 0) mbar_arrive(bar(L::BAR_UNIT_EMPTY + (uc & 1)));
      if (!ok || u >= n_units) break;
      const int n = unit_of(u).n_it;
      if (!(ok = mbar_wait(bar(L::BAR_KV), uc & 1, wctx))) break;
      tc_fence_after();
      // the unit's first product into the accumulator overwrites it: the previous unit's
      // epilogue must have read it
      auto acc_free = [&](int it) -> bool {
        if (it > 0 || uc == 0) return true;
        if (!mbar_wait(bar(L::BAR_ACC_FREE), (uc - 1) & 1, wctx)) return false;
        tc_fence_after();
        return true;
      };
      if constexpr (KIND == 0) {
        // ---- dV: S^T double-buffered, dV (256 columns) += P^T dO in two d-halves
        if (!(ok = issue_full(tmem + L::T_S, dKs, bar(L::BAR_S)))) break;
        if (n > 1 && !(ok = issue_full(tmem + L::T_S + 128, dKs, bar(L::BAR_S + 1)))) break;
        if (n <= 2) mma_commit(bar(L::BAR_KV_EMPTY), leader);  // the unit's last S^T issued
        for (int it = 0; it < n && ok; ++it) {
          const int t = T0 + it, b = it & 1;
          const uint32_t tP = tmem + L::T_S + 128 * b;
          const int st0 = take();
          if (!ok) break;
          const int st1 = take();
          if (!ok) break;
          if (!(ok = mbar_wait(bar(L::BAR_P_HALF + b), nP[b] & 1, wctx))) break;
          tc_fence_after();
          if (!(ok = acc_free(it))) break;
          // the first half of P^T (query columns {0..31, 64..95}) while the second is computed
          issue_ts_split_part(tmem + L::T_ACC, tP, mn_desc(st0), idesc_g, it == 0, 0, leader);
          issue_ts_split_part(tmem + L::T_ACC + 128, tP, mn_desc(st1), idesc_g, it == 0, 0, leader);
          if (!(ok = mbar_wait(bar(L::BAR_P_READY + b), nP[b] & 1, wctx))) break;
          tc_fence_after();
          ++nP[b];
          issue_ts_split_part(tmem + L::T_ACC, tP, mn_desc(st0), idesc_g, false, 1, leader);
          issue_ts_split_part(tmem + L::T_ACC + 128, tP, mn_desc(st1), idesc_g, false, 1, leader);
          mma_commit(bar(L::BAR_SLOT_EMPTY + st0), leader);
          mma_commit(bar(L::BAR_SLOT_EMPTY + st1), leader);
          mma_commit(bar(L::BAR_LD_EMPTY + (t & 1)), leader);  // step t's LSE / D buffer is free after this
          if (it + 2 < n) {  // S^T(it + 2) into this step's buffer, after the products reading its P^T
            if (!(ok = issue_full(tP, dKs, bar(L::BAR_S + b)))) break;
            if (it + 3 == n) mma_commit(bar(L::BAR_KV_EMPTY), leader);
          }
        }
      } else {
        // ---- dK: S^T, dP^T; dK (256 columns) += dS^T Q in two d-halves, one Q half at a time
        if (!(ok = issue_full(tmem + L::T_S, dKs, bar(L::BAR_S)))) break;
        if (!(ok = issue_full(tmem + L::T_DP, dVs, bar(L::BAR_DP)))) break;
        if (n == 1) mma_commit(bar(L::BAR_KV_EMPTY), leader);
        for (int it = 0; it < n && ok; ++it) {
          const int t = T0 + it;
          if (it + 1 < n) {  // S^T(it + 1) once the compute warps hold S^T(it) in registers
            if (!(ok = mbar_wait(bar(L::BAR_S_LOADED), nSL & 1, wctx))) break;
            tc_fence_after();
            ++nSL;
            if (!(ok = issue_full(tmem + L::T_S, dKs, bar(L::BAR_S)))) break;
          }
          if (!(ok = mbar_wait(bar(L::BAR_DS_READY), nDS & 1, wctx))) break;
          tc_fence_after();
          ++nDS;
          if (!(ok = acc_free(it))) break;
          for (int hh = 0; hh < 2; ++hh) {
            const int st = take();
            if (!ok) break;
            issue_ts_split(tmem + L::T_ACC + 128 * hh, tmem + L::T_DP, mn_desc(st), idesc_g, it > 0, leader);
            mma_commit(bar(L::BAR_SLOT_EMPTY + st), leader);
          }
          if (!ok) break;
          mma_commit(bar(L::BAR_LD_EMPTY + (t & 1)), leader);
          if (it + 1 < n) {  // dP^T(it + 1) after the products reading dS^T(it)
            if (!(ok = issue_full(tmem + L::T_DP, dVs, bar(L::BAR_DP)))) break;
            if (it + 2 == n) mma_commit(bar(L::BAR_KV_EMPTY), leader);  // the unit's last S^T, dP^T issued
          }
        }
      }
      if (!ok) break;
      mma_commit(bar(L::BAR_ACC), leader);
      T0 += n;
    }
    mma_commit(bar(L::BAR_DONE), leader);
    drain_wait(bar(L::BAR_DONE), 0);
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle
  } else {
    // ===================================================== compute warpgroups
    regs_inc<kRegsHigh>();
    const int w = (warp - 4) >> 2;   // query columns [64 w, 64 w + 64) of every step
    const int wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;  // key row inside the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tDP = tmem + lane_off + L::T_DP + 64 * w;
    const float sl2 = ldexpf(p.scale_log2, -(p.exps[kExpQ] + p.exps[kExpK]));
    const uint64_t sl2x2 = f2pack(sl2, sl2);
    bool ok = true;
    int T0 = 0;
    int nS[2] = {0, 0}, nDP = 0;  // completions of S^T buffer b and of dP^T waited for so far
    int u = next_unit(0, ok);
    mbar_arrive(bar(L::BAR_UNIT_EMPTY + 0));
    for (int uc = 0; ok && u < n_units; ++uc) {
      const Unit x = unit_of(u);
      const int j = x.j, i_start = x.i_start, n_q = x.n_q, n_it = x.n_it;
      const int key = j * 128 + row;
      const int q_vis_lo = query_lo(key, p.causal, p.win_right);
      const int q_vis_hi = query_hi(key, p.N, p.win_left);
      const int all_lo = query_lo(min(j * 128 + 127, p.N - 1), p.causal, p.win_right);
      const int all_hi = query_hi(j * 128, p.N, p.win_left);
      for (int it = 0; it < n_it; ++it) {
        const int T = T0 + it;
        const int i = i_start + it % n_q;
        const float* lse2 = reinterpret_cast<const float*>(gbase + L::OFF_LD + (T & 1) * 1024) + 64 * w;
        const float* delta = lse2 + 128;
        const int q0 = i * 128 + 64 * w;
        const int b = KIND == 1 ? 0 : (it & 1);  // S^T buffer of this step
        const uint32_t tS = tmem + lane_off + L::T_S + 128 * b + 64 * w;
        if (!(ok = mbar_wait(bar(L::BAR_S + b), nS[b] & 1, wctx))) break;
        tc_fence_after();
        ++nS[b];
        float pr[64];
        tmem_ld64(tS, pr);
        if (KIND == 1 && it + 1 < n_it) {  // S^T is in registers: the next S^T may overwrite it
          tc_fence_before();
          mbar_arrive(bar(L::BAR_S_LOADED));
        }
        // P^T = 2^(S^T scale log2(e) - LSE log2(e)); for dV written to TMEM over S^T as fp16 in
        // two halves (the first announced on P_HALF), for dK kept in registers
        auto probs = [&](auto masked) {
          const int c_lo = q_vis_lo - q0, c_hi = q_vis_hi - q0;
#pragma unroll
          for (int g = 0; g < 64; g += 16) {
            uint32_t pk[8];
#pragma unroll
            for (int c = g; c < g + 16; c += 4) {
              const float4 L4 = *reinterpret_cast<const float4*>(lse2 + c);
              float t0, t1, t2, t3;
              f2unpack(ffma2(f2pack(pr[c], pr[c + 1]), sl2x2, f2pack(-L4.x, -L4.y)), t0, t1);
              f2unpack(ffma2(f2pack(pr[c + 2], pr[c + 3]), sl2x2, f2pack(-L4.z, -L4.w)), t2, t3);
              if ((c - g) < kDkdvExpFmaPer16) {
                exp2_fma_pipe(t0, t1);
                exp2_fma_pipe(t2, t3);
                pr[c] = t0;
                pr[c + 1] = t1;
                pr[c + 2] = t2;
                pr[c + 3] = t3;
              } else {
                pr[c] = ex2_approx(t0);
                pr[c + 1] = ex2_approx(t1);
                pr[c + 2] = ex2_approx(t2);
                pr[c + 3] = ex2_approx(t3);
              }
              if constexpr (decltype(masked)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (c + e < c_lo || c + e > c_hi) pr[c + e] = 0.f;
              }
              if constexpr (KIND == 0) {
                pk[(c - g) / 2] = pack_f16(pr[c], pr[c + 1]);
                pk[(c - g) / 2 + 1] = pack_f16(pr[c + 2], pr[c + 3]);
              }
            }
            if constexpr (KIND == 0) {
              tmem_st8(tS + g / 2, pk);
              if (g == 16) {
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(L::BAR_P_HALF + b));
              }
            }
          }
        };
        if (q0 < all_lo || q0 + 63 > all_hi)
          probs(std::true_type{});
        else
          probs(std::false_type{});
        if constexpr (KIND == 0) {
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(L::BAR_P_READY + b));
        } else {
          if (!(ok = mbar_wait(bar(L::BAR_DP), nDP & 1, wctx))) break;
          tc_fence_after();
          ++nDP;
          float dp[64];
          tmem_ld64(tDP, dp);
#pragma unroll
          for (int g = 0; g < 64; g += 16) {
            uint32_t pk[8];
#pragma unroll
            for (int c = g; c < g + 16; c += 4) {
              const float4 D4 = *reinterpret_cast<const float4*>(delta + c);
              float d0, d1, d2, d3;
              f2unpack(fmul2(f2pack(pr[c], pr[c + 1]), fsub2(f2pack(dp[c], dp[c + 1]), f2pack(D4.x, D4.y))), d0, d1);
              f2unpack(fmul2(f2pack(pr[c + 2], pr[c + 3]), fsub2(f2pack(dp[c + 2], dp[c + 3]), f2pack(D4.z, D4.w))),
                       d2, d3);
              pk[(c - g) / 2] = pack_f16(d0, d1);
              pk[(c - g) / 2 + 1] = pack_f16(d2, d3);
            }
            tmem_st8(tDP + g / 2, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(L::BAR_DS_READY));
        }
      }
      if (!ok) break;
      if (!(ok = mbar_wait(bar(L::BAR_ACC), uc & 1, wctx))) break;
      tc_fence_after();
      // warpgroup w writes columns [128 w, 128 w + 128) of the kernel's gradient: dV, or scale * dK
      const size_t head_off = p.kv_split == 1 ? (size_t)x.bh * p.N * D : ((size_t)x.sp * BH_kv + x.bh) * p.N * D;
      float* out = (p.kv_split == 1 ? (KIND == 1 ? p.dk : p.dv) : (KIND == 1 ? p.dk_part : p.dv_part)) + head_off +
                   128 * w;
      const uint32_t t_acc = tmem + lane_off + L::T_ACC + 128 * w;
      const Pow2 out_f =
          pow2_factors(KIND == 1 ? -(p.exps[kExpV] + p.exps[kExpDO] + p.exps[kExpQ]) : -p.exps[kExpDO]);
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float acc[64];
        tmem_ld64(t_acc + 64 * c, acc);
        if (c == 1) {
          tc_fence_before();
          mbar_arrive(bar(L::BAR_ACC_FREE));
        }
        warp_store_rows_f32<64>(acc, out + 64 * c, D, j * 128 + wq * 32, p.N, KIND == 1 ? p.scale : 1.0f, out_f);
      }
      T0 += n_it;
      u = next_unit(uc + 1, ok);
      mbar_arrive(bar(L::BAR_UNIT_EMPTY + ((uc + 1) & 1)));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

struct DqWLayout {
  static constexpr int OFF_Q = 0;              // Q: two halves (resident for the unit)
  static constexpr int OFF_DO = 2 * kHalf;     // dO: two halves
  static constexpr int OFF_RING = 4 * kHalf;   // kWSlots halves of K or V
  static constexpr int OFF_BAR = OFF_RING + kWSlots * kHalf;
  static constexpr int BAR_Q = 0;           // a unit's Q and dO landed
  static constexpr int BAR_Q_EMPTY = 1;     // the MMAs reading a unit's Q and dO have completed
  static constexpr int BAR_SLOT_FULL = 2;   // [kWSlots]
  static constexpr int BAR_SLOT_EMPTY = 5;  // [kWSlots]
  static constexpr int BAR_S = 8;
  static constexpr int BAR_DP = 9;
  static constexpr int BAR_DS = 10;         // dS of a step written over dP
  static constexpr int BAR_ACC = 11;
  static constexpr int BAR_DQ_FREE = 12;
  static constexpr int BAR_UNIT_FULL = 13;   // [2]
  static constexpr int BAR_UNIT_EMPTY = 15;  // [2]
  static constexpr int BAR_DONE = 17;
  static constexpr int BAR_S_LOADED = 18;    // the step's S is in the compute warps' registers
  static constexpr int NBAR = 19;
  static constexpr int OFF_UNIT = OFF_BAR + NBAR * 8;
  static constexpr int OFF_TMEM_SLOT = OFF_UNIT + 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int BYTES = OFF_ABORT + 8;
  static constexpr int SMEM_ALLOC = BYTES + 1024 <= kSmemMax ? BYTES + 1024 : kSmemMax;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256;
};
static_assert(DqWLayout::BYTES <= kSmemMax, "d = 256 dQ kernel exceeds the shared memory of a CTA");

__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dq_d256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const BwdParams p) {
  using L = DqWLayout;
  constexpr int D = 256;
#ifndef FA_DQ_EXP_FMA_PER16
#define FA_DQ_EXP_FMA_PER16 4
#endif
  constexpr int kDqExpFmaPer16 = FA_DQ_EXP_FMA_PER16;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if (!smem_base_fits<L>(raw, base)) {
    if (threadIdx.x == 0) atomicExch(p.err, kDevRange);
    return;
  }
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int nq = (p.N + 127) / 128;
  const int n_units = nq * p.BH;
  struct Unit {
    int bh, bh_kv, qt, jlo, n_it;
  };
  auto unit_of = [&](int u) -> Unit {
    Unit x;
    int rank;
    unit_order(u, nq, p.BH, p.head_group, x.bh, rank);
    x.bh_kv = kv_head_of(x.bh, p.H, p.H_kv);
    x.qt = p.causal ? (nq - 1 - rank) : rank;
    x.jlo = key_lo(x.qt * 128, p.N, p.win_left) / 128;
    x.n_it = key_hi(x.qt * 128 + 127, p.N, p.causal, p.win_right) / 128 - x.jlo + 1;
    return x;
  };
  int* unit_ring = reinterpret_cast<int*>(gbase + L::OFF_UNIT);
  auto next_unit = [&](int k, bool& ok) -> int {
    const int slot = k & 1;
    ok = mbar_wait(bar(L::BAR_UNIT_FULL + slot), (k >> 1) & 1, wctx);
    return ok ? *reinterpret_cast<volatile int*>(unit_ring + slot) : n_units;
  };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::BAR_Q), 1);
    mbar_init(bar(L::BAR_Q_EMPTY), 1);
    for (int s = 0; s < kWSlots; ++s) {
      mbar_init(bar(L::BAR_SLOT_FULL + s), 1);
      mbar_init(bar(L::BAR_SLOT_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::BAR_UNIT_FULL + s), 1);
      mbar_init(bar(L::BAR_UNIT_EMPTY + s), 1 + 256);
    }
    mbar_init(bar(L::BAR_S), 1);
    mbar_init(bar(L::BAR_DP), 1);
    mbar_init(bar(L::BAR_DS), 256);
    mbar_init(bar(L::BAR_ACC), 1);
    mbar_init(bar(L::BAR_DQ_FREE), 256);
    mbar_init(bar(L::BAR_DONE), 1);
    mbar_init(bar(L::BAR_S_LOADED), 256);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::OFF_TMEM_SLOT, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::OFF_TMEM_SLOT);

  // dS is written over dP, so S(it + 1) may overwrite S as soon as the compute warps hold S(it)
  // in registers, while dP(it + 1) follows dQ(it) (which reads dS(it)).  FIFO order of a unit
  // with n key steps: K0(0) K1(0) V0(0) V1(0), then for it = 0..n-1:
  // [K0(it+1) K1(it+1)] K0(it) K1(it) [V0(it+1) V1(it+1)]  (bracketed parts while it + 1 < n).
  if (warp == 0) {
    // ===================================================== TMA producer + work distribution
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    int F = 0, q_issued = 0;
    bool ok = true;
    auto load_half = [&](const Unit& x, int which, int half, int it) -> bool {  // half of K (0) or V (1)
      const int st = F % kWSlots;
      if (!mbar_wait(bar(L::BAR_SLOT_EMPTY + st), ((F / kWSlots) & 1) ^ 1u, wctx)) return false;
      const uint32_t fb = bar(L::BAR_SLOT_FULL + st);
      mbar_arrive_expect_tx(fb, kHalf, leader);
      const CUtensorMap* m = which ? &tm_v : &tm_k;
      const uint32_t dst = base + L::OFF_RING + st * kHalf;
      for (int b = 0; b < 2; ++b)
        tma_load_3d(dst + b * kBox, m, half * 128 + b * 64, (x.jlo + it) * 128, x.bh_kv, fb, leader);
      ++F;
      return true;
    };
    for (int uc = 0;; ++uc) {
      if (uc >= 2 && !(ok = mbar_wait(bar(L::BAR_UNIT_EMPTY + (uc & 1)), ((uc - 2) >> 1) & 1, wctx))) break;
      int u = 0;
      if (lane == 0) u = (int)atomicAdd(p.dq_counter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (lane == 0) {
        unit_ring[uc & 1] = u < n_units ? u : n_units;
        mbar_arrive(bar(L::BAR_UNIT_FULL + (uc & 1)));
      }
      __syncwarp();
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      if (uc > 0 && !(ok = mbar_wait(bar(L::BAR_Q_EMPTY), (uc - 1) & 1, wctx))) break;
      mbar_arrive_expect_tx(bar(L::BAR_Q), 4 * kHalf, leader);
      for (int c = 0; c < 4; ++c) {
        const uint32_t off = (c >> 1) * kHalf + (c & 1) * kBox;
        tma_load_3d(base + L::OFF_Q + off, &tm_q, c * 64, x.qt * 128, x.bh, bar(L::BAR_Q), leader);
        tma_load_3d(base + L::OFF_DO + off, &tm_do, c * 64, x.qt * 128, x.bh, bar(L::BAR_Q), leader);
      }
      ++q_issued;
      const int n = x.n_it;
      ok = load_half(x, 0, 0, 0) && load_half(x, 0, 1, 0) && load_half(x, 1, 0, 0) && load_half(x, 1, 1, 0);
      for (int it = 0; it < n && ok; ++it) {
        if (it + 1 < n) ok = load_half(x, 0, 0, it + 1) && load_half(x, 0, 1, it + 1);  // S(it + 1)
        ok = ok && load_half(x, 0, 0, it) && load_half(x, 0, 1, it);                    // K again, dQ(it)
        if (ok && it + 1 < n) ok = load_half(x, 1, 0, it + 1) && load_half(x, 1, 1, it + 1);  // dP(it + 1)
      }
      if (!ok) break;
    }
    if (q_issued > 0) drain_wait(bar(L::BAR_Q), (q_issued - 1) & 1);
    for (int f = (F > kWSlots ? F - kWSlots : 0); f < F; ++f)
      drain_wait(bar(L::BAR_SLOT_FULL + f % kWSlots), (f / kWSlots) & 1);
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    constexpr uint32_t idesc_s = make_idesc(128, 128, false, false, false);  // M=128 queries, N=128 keys
    constexpr uint32_t idesc_g = make_idesc(128, 128, false, false, true);   // N=128 (a d-half), B MN-major
    const uint64_t dQs[2] = {make_sdesc_sw128(base + L::OFF_Q, 16, 1024),
                             make_sdesc_sw128(base + L::OFF_Q + kHalf, 16, 1024)};
    const uint64_t dDOs[2] = {make_sdesc_sw128(base + L::OFF_DO, 16, 1024),
                              make_sdesc_sw128(base + L::OFF_DO + kHalf, 16, 1024)};
    const uint64_t dRingK = make_sdesc_sw128(base + L::OFF_RING, 16, 1024);
    const uint64_t dRingMN = make_sdesc_sw128(base + L::OFF_RING, kBox, 1024);
    int C = 0;
    bool ok = true;
    auto take = [&]() -> int {
      const int st = C % kWSlots;
      ok = mbar_wait(bar(L::BAR_SLOT_FULL + st), (C / kWSlots) & 1, wctx);
      ++C;
      if (ok) tc_fence_after();
      return st;
    };
    // S = Q K^T (dP = dO V^T) over both d-halves, each half of K (V) taken from the FIFO
    auto issue_full = [&](uint32_t d_tmem, const uint64_t (&a)[2], uint32_t done_bar) -> bool {
      for (int hh = 0; hh < 2; ++hh) {
        const int st = take();
        if (!ok) return false;
        issue_ss_half(d_tmem, a[hh], sdesc_add(dRingK, st * kHalf), idesc_s, hh == 0, leader);
        mma_commit(bar(L::BAR_SLOT_EMPTY + st), leader);
      }
      mma_commit(done_bar, leader);
      return true;
    };
    int T0 = 0;
    for (int uc = 0;; ++uc) {
      const int u = next_unit(uc, ok);
      if (lane == 0) mbar_arrive(bar(L::BAR_UNIT_EMPTY + (uc & 1)));
      if (!ok || u >= n_units) break;
      const int n = unit_of(u).n_it;
      if (!(ok = mbar_wait(bar(L::BAR_Q), uc & 1, wctx))) break;
      tc_fence_after();
      if (!(ok = issue_full(tmem + L::T_S, dQs, bar(L::BAR_S)))) break;
      if (!(ok = issue_full(tmem + L::T_DP, dDOs, bar(L::BAR_DP)))) break;
      if (n == 1) mma_commit(bar(L::BAR_Q_EMPTY), leader);
      for (int it = 0; it < n && ok; ++it) {
        const int t = T0 + it;
        if (it + 1 < n) {  // S(it + 1) once the compute warps hold S(it) in registers
          if (!(ok = mbar_wait(bar(L::BAR_S_LOADED), t & 1, wctx))) break;
          tc_fence_after();
          if (!(ok = issue_full(tmem + L::T_S, dQs, bar(L::BAR_S)))) break;
        }
        if (!(ok = mbar_wait(bar(L::BAR_DS), t & 1, wctx))) break;
        tc_fence_after();
        if (it == 0 && uc > 0) {
          if (!(ok = mbar_wait(bar(L::BAR_DQ_FREE), (uc - 1) & 1, wctx))) break;
          tc_fence_after();
        }
        for (int hh = 0; hh < 2 && ok; ++hh) {  // dQ[:, 128 hh ..] += dS K_hh
          const int st = take();
          if (!ok) break;
          issue_ts_split(tmem + L::T_DQ + 128 * hh, tmem + L::T_DP, sdesc_add(dRingMN, st * kHalf), idesc_g,
                         it > 0, leader);
          mma_commit(bar(L::BAR_SLOT_EMPTY + st), leader);
        }
        if (!ok) break;
        if (it + 1 < n) {
          if (!(ok = issue_full(tmem + L::T_DP, dDOs, bar(L::BAR_DP)))) break;  // dP(it + 1), after dQ(it)
          if (it + 2 == n) mma_commit(bar(L::BAR_Q_EMPTY), leader);
        }
      }
      if (ok) mma_commit(bar(L::BAR_ACC), leader);
      T0 += n;
    }
    mma_commit(bar(L::BAR_DONE), leader);
    drain_wait(bar(L::BAR_DONE), 0);
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle
  } else {
    // ===================================================== compute warpgroups
    regs_inc<kRegsHigh>();
    const int w = (warp - 4) >> 2;   // key columns [64 w, 64 w + 64) of every step
    const int wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::T_S + 64 * w;
    const float sl2 = ldexpf(p.scale_log2, -(p.exps[kExpQ] + p.exps[kExpK]));
    const uint64_t sl2x2 = f2pack(sl2, sl2);
    bool ok = true;
    int T0 = 0;
    float lse2 = 0.f, delta = 0.f;
    int u = next_unit(0, ok);
    mbar_arrive(bar(L::BAR_UNIT_EMPTY + 0));
    if (ok && u < n_units) {
      const Unit x0 = unit_of(u);
      const size_t prow = (size_t)x0.bh * p.Np + x0.qt * 128 + row;
      lse2 = p.lse2[prow];
      delta = p.delta[prow];
    }
    for (int uc = 0; ok && u < n_units; ++uc) {
      const Unit x = unit_of(u);
      const int r = x.qt * 128 + row;
      const int k_vis_lo = key_lo(r, p.N, p.win_left);
      const int k_vis_hi = key_hi(r, p.N, p.causal, p.win_right);
      const int all_lo = key_lo(min(x.qt * 128 + 127, p.N - 1), p.N, p.win_left);
      const int all_hi = key_hi(x.qt * 128, p.N, p.causal, p.win_right);
      const uint64_t nl2 = f2pack(-lse2, -lse2), dd = f2pack(delta, delta);
      for (int it = 0; it < x.n_it; ++it) {
        const int t = T0 + it;
        const int k0 = (x.jlo + it) * 128 + 64 * w;
        if (!(ok = mbar_wait(bar(L::BAR_S), t & 1, wctx))) break;
        tc_fence_after();
        float pr[64];
        tmem_ld64(tS, pr);
        tc_fence_before();
        mbar_arrive(bar(L::BAR_S_LOADED));  // S(it + 1) may overwrite S
        auto probs = [&](auto masked) {
          const int c_lo = k_vis_lo - k0, c_hi = k_vis_hi - k0;
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float t0, t1;
            f2unpack(ffma2(f2pack(pr[c], pr[c + 1]), sl2x2, nl2), t0, t1);
            if ((c & 15) < kDqExpFmaPer16) {
              exp2_fma_pipe(t0, t1);
              pr[c] = t0;
              pr[c + 1] = t1;
            } else {
              pr[c] = ex2_approx(t0);
              pr[c + 1] = ex2_approx(t1);
            }
            if constexpr (decltype(masked)::value) {
              if (c < c_lo || c > c_hi) pr[c] = 0.f;
              if (c + 1 < c_lo || c + 1 > c_hi) pr[c + 1] = 0.f;
            }
          }
        };
        if (k0 < all_lo || k0 + 63 > all_hi)
          probs(std::true_type{});
        else
          probs(std::false_type{});
        if (!(ok = mbar_wait(bar(L::BAR_DP), t & 1, wctx))) break;
        tc_fence_after();
        float dp[64];
        const uint32_t tDP = tmem + lane_off + L::T_DP + 64 * w;
        tmem_ld64(tDP, dp);
#pragma unroll
        for (int g = 0; g < 64; g += 16) {
          uint32_t pk[8];
#pragma unroll
          for (int c = g; c < g + 16; c += 2) {
            float d0, d1;
            f2unpack(fmul2(f2pack(pr[c], pr[c + 1]), fsub2(f2pack(dp[c], dp[c + 1]), dd)), d0, d1);
            pk[(c - g) / 2] = pack_f16(d0, d1);
          }
          tmem_st8(tDP + g / 2, pk);  // dS over dP
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::BAR_DS));
      }
      if (!ok) break;
      if (!(ok = mbar_wait(bar(L::BAR_ACC), uc & 1, wctx))) break;
      tc_fence_after();
      // each warpgroup writes 128 of the 256 columns of scale * dQ, 64 at a time
      const Pow2 out_f = pow2_factors(-(p.exps[kExpV] + p.exps[kExpDO] + p.exps[kExpK]));
      const int u_next = next_unit(uc + 1, ok);
      mbar_arrive(bar(L::BAR_UNIT_EMPTY + ((uc + 1) & 1)));
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float acc[64];
        tmem_ld64(tmem + lane_off + L::T_DQ + w * 128 + 64 * c, acc);
        if (c == 1) {
          tc_fence_before();
          mbar_arrive(bar(L::BAR_DQ_FREE));
        }
        warp_store_rows_f32<64>(acc, p.dq + (size_t)x.bh * p.N * D + w * 128 + 64 * c, D, x.qt * 128 + wq * 32,
                                p.N, p.scale, out_f);
      }
      if (ok && u_next < n_units) {  // the next unit's row statistics
        const Unit xn = unit_of(u_next);
        const size_t prow = (size_t)xn.bh * p.Np + xn.qt * 128 + row;
        lse2 = p.lse2[prow];
        delta = p.delta[prow];
      }
      T0 += x.n_it;
      u = u_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <typename Layout, typename Kern>
cudaError_t launch_one(Kern kern, dim3 grid, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                       const CUtensorMap& d, const BwdParams& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, Layout::SMEM_ALLOC, s>>>(a, b, c, d, p);
  return cudaGetLastError();
}

}  // namespace

template <int D>
cudaError_t launch_dkdv_t(dim3 grid, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                          const CUtensorMap& tv, const CUtensorMap& tdv, const CUtensorMap& tdk, const BwdParams& p,
                          cudaStream_t s) {
  using L = DkdvLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(fa_bwd_dkdv_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  fa_bwd_dkdv_sm100_kernel<D><<<grid, kThreads, L::SMEM_ALLOC, s>>>(tq, tdo, tk, tv, tdv, tdk, p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const CUtensorMap& tdv, const CUtensorMap& tdk,
                                  const BwdParams& p, int d, cudaStream_t s) {
  // persistent: one CTA per SM (at most one per unit: key tile x key/value head x group split;
  // at d = 256 the same units in each of the two kernels)
  const long long units = (long long)((p.N + 127) / 128) * (p.BH / p.H * p.H_kv) * p.kv_split;
  const dim3 grid((unsigned)(units < p.num_sms ? units : p.num_sms));
  if (d == 256) {  // the dV kernel, then the dK kernel
    const cudaError_t e = launch_one<DkdvWLayout<0>>(fa_bwd_dkdv_d256_kernel<0>, grid, tq, tdo, tk, tv, p, s);
    if (e != cudaSuccess) return e;
    return launch_one<DkdvWLayout<1>>(fa_bwd_dkdv_d256_kernel<1>, grid, tq, tdo, tk, tv, p, s);
  }
  if (d == 128) return launch_dkdv_t<128>(grid, tq, tdo, tk, tv, tdv, tdk, p, s);
  return launch_dkdv_t<64>(grid, tq, tdo, tk, tv, tdv, tdk, p, s);
}

cudaError_t launch_bwd_dq_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                const CUtensorMap& tv, const BwdParams& p, int d, cudaStream_t s) {
  // persistent: one CTA per SM (at most one per work unit)
  const long long units = (long long)((p.N + 127) / 128) * p.BH;
  const dim3 grid((unsigned)(units < p.num_sms ? units : p.num_sms));
  if (d == 256) return launch_one<DqWLayout>(fa_bwd_dq_d256_kernel, grid, tq, tdo, tk, tv, p, s);
  if (d == 128) return launch_one<DqLayout<128>>(fa_bwd_dq_sm100_kernel<128>, grid, tq, tdo, tk, tv, p, s);
  return launch_one<DqLayout<64>>(fa_bwd_dq_sm100_kernel<64>, grid, tq, tdo, tk, tv, p, s);
}

}  // namespace fa
