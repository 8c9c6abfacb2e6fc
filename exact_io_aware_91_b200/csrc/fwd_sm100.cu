// Forward pass of exact attention on sm_100a:
//   O = softmax(scale * Q K^T + causal mask) V,  LSE = ln sum_j exp(scale * S_ij)
//
// The method ("Flash Attention uitgelegd: een uitgebreide gids", sections
// "Tiling" and "Werkingsmechanisme"; "FlashAttention (EL)", sections "Tiling",
// "Online computation of Softmax" and "Fusion of operations into one CUDA
// kernel"): Q, K and V are cut into on-chip tiles, the softmax is applied
// incrementally with a running row maximum and exp-sum, and the partial output
// is rescaled as each K/V tile arrives, so the N x N score matrix never reaches
// HBM.  One fused kernel writes only O (and the per-row LSE kept for the
// backward pass).
//
// B200 design (not a translation of the pages' A100/H100 kernels):
//   * one CTA = one work unit = two 128-row query tiles of one (b, h); the two
//     tiles ping-pong on the tensor core so that the softmax of one overlaps the
//     MMAs of the other ("overlapping GEMM + softmax", page "Flash Attention:
//     Ako transformery ...", section 3, re-done for tcgen05);
//   * warp 0 streams K/V tiles with TMA into a multi-stage shared-memory ring;
//   * warp 1 issues tcgen05.mma: S_t = Q_t K_j^T into tensor memory (TMEM), and
//     O_t += P_t V_j with P_t read straight from TMEM (it overwrites S_t there);
//   * warps 2-3 convert each V tile to fp16 in shared memory (exact for bf16
//     values of normal fp16 range) so that P is rounded to fp16 (11 significant
//     bits) rather than bf16 (8) before the P V product;
//   * warpgroups 1 and 2 (one per query tile, one thread per row) run the online
//     softmax on S rows loaded from TMEM, write P back to TMEM as fp16 and, when
//     the running maximum grows by more than 2^8, rescale O in TMEM;
//   * the epilogue divides by the row sum, converts to bf16 and TMA-stores O, and
//     optionally writes the bf16 residual O_fp32 - O_bf16 so that the backward
//     pass can form rowsum(dO * O) from an fp32-accurate O.
//
// Kernels in this file:
//   fa_fwd_sm100_kernel<d>            one CTA per unit, V converted on chip (fa_fwd, fa_fwd_gqa)
//   fa_fwd_persist_sm100_kernel<d,F8> persistent, V already fp16 (fa_fwd_ws, fa_attn_fwd); with
//                                     F8 the E4M3 forward (fa_attn_fwd_fp8)
//   fa_fwd_d256_sm100_kernel          persistent, head dim 256, one query tile per unit
//   fa_fwd_v16_kernel                 V bf16 -> fp16 into the workspace (and the work counter reset)
//   fa_fwd_v16_fixup_kernel           the V copy's exponent (re-conversion when it is not 0)
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

template <int D>
struct FwdLayout {
  static constexpr int BM = 128;                 // query rows per tile
  static constexpr int BN = 128;                 // keys per K/V tile
  static constexpr int KCH = D / 64;             // 128-byte column chunks per row
  static constexpr int BOX = 128 * 128;          // one 64-column x 128-row bf16 box (16 KB)
  static constexpr int TILE = KCH * BOX;         // one 128 x D bf16 tile
  static constexpr int STAGES = (D == 128) ? 4 : 8;
  static constexpr int OFF_Q0 = 0;
  static constexpr int OFF_Q1 = TILE;
  static constexpr int OFF_KV = 2 * TILE;
  static constexpr int OFF_BAR = OFF_KV + STAGES * TILE;
  // barriers: q_full, kv_full[STAGES], kv_empty[STAGES], v_conv[STAGES], s_full[2], p_half[2],
  // p_full[2], o_full[2], mma_done, v_exp[STAGES]
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_KV_FULL = 1;
  static constexpr int BAR_KV_EMPTY = 1 + STAGES;
  static constexpr int BAR_V_CONV = 1 + 2 * STAGES;
  static constexpr int BAR_S_FULL = 1 + 3 * STAGES;
  static constexpr int BAR_P_HALF = BAR_S_FULL + 2;  // P for keys 0..63 of the tile is in TMEM
  static constexpr int BAR_P_FULL = BAR_P_HALF + 2;
  static_assert(BAR_P_FULL == BAR_P_HALF + 2, "the softmax arrives on BAR_P_HALF + t + 2 * half");
  static constexpr int BAR_O_FULL = BAR_P_FULL + 2;
  static constexpr int BAR_MMA_DONE = BAR_O_FULL + 2;
  static constexpr int BAR_V_EXP = BAR_MMA_DONE + 1;  // [STAGES] the V tile's copy exponent is published
  static constexpr int BAR_V_AMAX = BAR_V_EXP + STAGES;  // [2] both converter warps' tile maxima written
  static constexpr int NBAR = BAR_V_AMAX + 2;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NBAR * 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int OFF_VEXP = OFF_ABORT + 8;       // int[STAGES]: exponent of the V tile in each stage
  static constexpr int OFF_VAMAX = OFF_VEXP + 4 * STAGES;  // uint32[2][2]: the two converter warps' maxima
  static constexpr int BYTES = OFF_VAMAX + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;  // slack to align the base to 1024 bytes
  static constexpr uint32_t TMEM_COLS = 512;       // S0, S1 (128 each), O0, O1 (D each)
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O0 = 256, T_O1 = 256 + D;
};

constexpr int kThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 2-3 V to fp16, warps 4-7 / 8-11 softmax
// registers per thread: 168 at launch (65536 / 384, rounded down to a multiple of 8);
// warpgroup 0 (TMA, MMA, V conversion) drops to 64, the softmax warpgroups rise to 216
constexpr uint32_t kRegsLaunch = 168, kRegsLow = 64, kRegsHigh = 216;
static_assert(kRegsLow + 2 * kRegsHigh <= 3 * kRegsLaunch, "register split exceeds the launch budget");
constexpr int kConvThreads = 64;
// A quarter of the softmax exponentials run on the FMA pipe (degree-3 polynomial, see
// exp2_fma_pipe): measured on B200 with the fp16-V forward, 2 of 8 gives -6 % at N = 8192
// (4 of 8 is slower again: the single softmax warp per sub-partition becomes issue-bound).
#ifndef FA_EXP_FMA_PER8
#define FA_EXP_FMA_PER8 2
#endif
// The 8-bit forward's products take half the tensor-core time, so the exponentials (16 per
// clock per SM on the MUFU) are its bound: it moves a larger share to the FMA pipe.
#ifndef FA_EXP_FMA_PER8_F8
#define FA_EXP_FMA_PER8_F8 2
#endif
// The persistent forward hands P to the tensor core in this many parts per 128-key step
// (2 or 4): the last part's share of P V is what the next S product of the tile waits for.
#ifndef FA_FWD_PARTS
#define FA_FWD_PARTS 2
#endif
constexpr int kFwdParts = FA_FWD_PARTS;
// element pairs out of every 8 whose exponentials run on the FMA pipe (even, 0..8)
constexpr int kExpFmaPer8 = FA_EXP_FMA_PER8;

constexpr int kExpFmaPer8F8 = FA_EXP_FMA_PER8_F8;
static_assert(kExpFmaPer8 % 2 == 0 && kExpFmaPer8 >= 0 && kExpFmaPer8 <= 8, "pairs are taken two at a time");
static_assert(kExpFmaPer8F8 % 2 == 0 && kExpFmaPer8F8 >= 0 && kExpFmaPer8F8 <= 8, "pairs are taken two at a time");
static_assert(FwdLayout<128>::STAGES % 2 == 0 && FwdLayout<64>::STAGES % 2 == 0,
              "K and V tiles must alternate over fixed ring stages");

// Bounded wait used while draining copies on the way out: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// One online-softmax step of a query tile (one thread per row): S_j from TMEM, mask,
// running maximum (kept while within 2^8 of the true one), O rescaled in TMEM when the
// maximum moves, P = 2^(scale*log2(e)*S - m) written back over S as fp16 in two halves
// (the tensor core starts on the first half's P V while the second half is computed).
// With F8, P is written as E4M3 (four per TMEM column, 16 columns per half) for the 8-bit
// P V product; the row sum uses the fp32 values before rounding.  bar_o_ready (non-zero)
// is waited on, with parity o_ready_parity, before a rescale of O: for a kernel whose
// previous P V into O may still be running when this step starts.
// TILE_EXP: the V tile of this step is an fp16 copy V_j 2^v (v <= 0, published in *vexp_slot
// once bar_vexp completes with parity vexp_parity); the step then writes P' = P 2^-v, so that
// P' V_j 2^v = P V_j, and adds 2^v sum(P') to the row sum.  P' must stay within fp16 (P'
// <= 2^15): the running maximum may then lag the true one by at most min(8, 15 + v).
// A tile whose P sum exceeds what valid scores allow (a non-finite input, or a score beyond
// the fp32 range) is recorded as kDevRange in the error word.
// Returns false if a bounded wait gave up.
template <int D, bool F8 = false, bool TILE_EXP = false, int PARTS = 2>
__device__ __forceinline__ bool fwd_softmax_step(const FwdParams& p, uint32_t tS, uint32_t tO, uint32_t bar_s_full,
                                                 uint32_t s_parity, uint32_t bar_p_half, uint32_t bar_p_full, int j,
                                                 bool first, int q_base, int r, float& m, float& l,
                                                 const WaitCtx& wctx, uint32_t bar_o_ready = 0,
                                                 uint32_t o_ready_parity = 0, uint32_t bar_vexp = 0,
                                                 uint32_t vexp_parity = 0, const int* vexp_slot = nullptr) {
  const float sl2 = p.scale_log2;
  if (!mbar_wait(bar_s_full, s_parity, wctx)) return false;
  tc_fence_after();
  float x[128];
  {
    uint32_t u[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, u[c]);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < 32; ++i) x[32 * c + i] = __uint_as_float(u[c][i]);
  }
  // keys kb .. kb + 127 against this row's visible range (causal mask, sliding window, N);
  // with a window a row can have no visible key in a tile of its warpgroup's range.  The
  // test is on the range every row of the tile sees (both bounds grow with the row), the
  // same for the whole warpgroup, so tiles inside it skip the per-element compares.
  const int kb = j * 128;
  const int all_lo = key_lo(min(q_base + 127, p.N - 1), p.N, p.win_left);
  const int all_hi = key_hi(q_base, p.N, p.causal, p.win_right);
  if (kb < all_lo || kb + 127 > all_hi) {
    const int lo = key_lo(r, p.N, p.win_left), hi = key_hi(r, p.N, p.causal, p.win_right);
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if (kb + c < lo || kb + c > hi) x[c] = -INFINITY;
  }
  // row max: a tree of 3-input maxima (depth 4)
  float a_[43], b_[15];
#pragma unroll
  for (int i = 0; i < 42; ++i) a_[i] = max3f(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
  a_[42] = fmaxf(x[126], x[127]);
#pragma unroll
  for (int i = 0; i < 14; ++i) b_[i] = max3f(a_[3 * i], a_[3 * i + 1], a_[3 * i + 2]);
  b_[14] = a_[42];
  const float mx = max3f(max3f(max3f(b_[0], b_[1], b_[2]), max3f(b_[3], b_[4], b_[5]), max3f(b_[6], b_[7], b_[8])),
                         max3f(b_[9], b_[10], b_[11]), max3f(b_[12], b_[13], b_[14]));
  const float m_new = fmaxf(m, mx * sl2);
  int v = 0;  // exponent of this step's V tile copy (TILE_EXP)
  if constexpr (TILE_EXP) {
    if (!mbar_wait(bar_vexp, vexp_parity, wctx)) return false;
    v = *reinterpret_cast<const volatile int*>(vexp_slot);
  }
  // keep a stale maximum while it is within 2^8 of the true one: exact in the end
  // because O / l and the LSE use the same maximum
  const float lag = TILE_EXP ? (float)min(8, 15 + v) : 8.0f;
  const float m_use = (m_new - m > lag) ? m_new : m;
  const float alpha = (m_use == m) ? 1.0f : ex2_approx(m - m_use);  // 0 on the first tile
  float neg_m = m_use == -INFINITY ? 0.0f : -m_use;  // no visible key yet: every P is 0
  if constexpr (TILE_EXP) neg_m -= (float)v;         // P' = P 2^-v
  if (!first && __any_sync(0xffffffffu, alpha != 1.0f)) {
    // rescale O before this tile's P V starts; either the previous O += P V of this tile
    // completed before S_j did (issued before it by the same thread, in-order tensor pipe),
    // or the caller names the barrier its completion arrives on
    if (bar_o_ready != 0 && !mbar_wait(bar_o_ready, o_ready_parity, wctx)) return false;
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t u[32];
      tmem_ld32(tO + 32 * c, u);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
      tmem_st32(tO + 32 * c, u);
    }
  }
  uint64_t sa = 0, sb = 0;  // packed fp32 partial row sums (0.0f, 0.0f)
  // P goes to TMEM in PARTS parts of 128 / PARTS keys; part h is announced on bar_p_half +
  // 16 h (with two parts: bar_p_half, then bar_p_full), so its share of P V can start while
  // the next part is computed
  static_assert(PARTS == 2 || PARTS == 4, "two halves or four quarters of the 128 keys");
  constexpr int PER = 128 / PARTS;  // keys per part
#pragma unroll
  for (int h = 0; h < PARTS; ++h) {
    uint32_t pk[PER / 2];
#pragma unroll
    for (int i = 0; i < PER / 2; i += 2) {
      float* e = &x[PER * h + 2 * i];
      fma2(e[0], e[1], sl2, neg_m);
      fma2(e[2], e[3], sl2, neg_m);
      // kExpFmaPer8 (kExpFmaPer8F8) of every 8 element pairs take 2^x on the FMA pipe, the
      // rest on MUFU
      constexpr int fma_per8 = F8 ? kExpFmaPer8F8 : kExpFmaPer8;
      if ((i & 7) < 2 * (fma_per8 / 2)) {
        exp2_fma_pipe(e[0], e[1]);
        exp2_fma_pipe(e[2], e[3]);
      } else {
        e[0] = ex2_approx(e[0]);
        e[1] = ex2_approx(e[1]);
        e[2] = ex2_approx(e[2]);
        e[3] = ex2_approx(e[3]);
      }
      if constexpr (F8) {
        pk[i / 2] = pack_e4m3x4(e[0], e[1], e[2], e[3]);
      } else {
        pk[i] = pack_f16(e[0], e[1]);
        pk[i + 1] = pack_f16(e[2], e[3]);
      }
      asm("add.rn.f32x2 %0, %0, %1;" : "+l"(sa) : "l"(f2pack(e[0], e[1])));
      asm("add.rn.f32x2 %0, %0, %1;" : "+l"(sb) : "l"(f2pack(e[2], e[3])));
    }
    if constexpr (F8 && PER == 64)
      tmem_st16(tS + 16 * h, pk);
    else if constexpr (F8)
      tmem_st8(tS + 8 * h, pk);
    else if constexpr (PER == 64)
      tmem_st32(tS + 32 * h, reinterpret_cast<const uint32_t(&)[32]>(pk));
    else
      tmem_st16(tS + 16 * h, pk);
    // this part of P (and any rescale of O) visible to the tensor core: its share of P V
    // can start while the next part is computed
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(PARTS == 2 ? (h == 0 ? bar_p_half : bar_p_full) : bar_p_half + 16u * h);
  }
  float s0, s1, s2, s3;
  f2unpack(sa, s0, s1);
  f2unpack(sb, s2, s3);
  const float tile_sum = (s0 + s1) + (s2 + s3);
  // a valid row's P (P') are each <= 2^15 (<= 2^8 unless TILE_EXP), so the tile's sum is <= 2^22:
  // a larger, infinite or NaN sum means a non-finite score (a non-finite input or a score beyond
  // the fp32 range: the row maximum is then +inf or ignores NaN elements)
  if (!(tile_sum <= 8388608.0f)) atomicExch(p.err, kDevRange);
  if constexpr (TILE_EXP)
    l = fmaf(l, alpha, tile_sum * __int_as_float((127 + v) << 23));  // 2^v sum(P')
  else
    l = fmaf(l, alpha, tile_sum);
  m = m_use;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        const FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: heaviest first within groups of heads (see unit_order); under the
  // causal mask the last query tiles of a head carry the most work
  int bh, rank;
  unit_order((int)blockIdx.x, p.n_pairs, p.BH, p.head_group, bh, rank);
  const int pair = p.causal ? (p.n_pairs - 1 - rank) : rank;
  const int bh_kv = kv_head_of(bh, p.H, p.H_kv);  // the key/value head this query head reads
  const int q_base0 = pair * 256;
  const int q_base1 = q_base0 + 128;
  const int n_kv = (p.N + 127) / 128;
  const int n0 = p.causal ? min(n_kv, q_base0 / 128 + 1) : n_kv;
  const int n1 = p.causal ? min(n_kv, q_base1 / 128 + 1) : n_kv;  // n1 >= n0

  // ---- setup
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::BAR_Q), 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::BAR_KV_FULL + s), 1);
      mbar_init(bar(L::BAR_KV_EMPTY + s), 1);
      mbar_init(bar(L::BAR_V_CONV + s), kConvThreads);
      mbar_init(bar(L::BAR_V_EXP + s), kConvThreads);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::BAR_S_FULL + t), 1);
      mbar_init(bar(L::BAR_P_HALF + t), 128);
      mbar_init(bar(L::BAR_P_FULL + t), 128);
      mbar_init(bar(L::BAR_O_FULL + t), 1);
    }
    mbar_init(bar(L::BAR_MMA_DONE), 1);
    mbar_init(bar(L::BAR_V_AMAX + 0), kConvThreads);
    mbar_init(bar(L::BAR_V_AMAX + 1), kConvThreads);
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
    {
      const uint32_t leader = elect_one();  // the lane that issues async instructions
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_o);
      mbar_arrive_expect_tx(bar(L::BAR_Q), 2 * L::TILE, leader);
      for (int c = 0; c < L::KCH; ++c) {
        tma_load_3d(base + L::OFF_Q0 + c * L::BOX, &tm_q, c * 64, q_base0, bh, bar(L::BAR_Q), leader);
        tma_load_3d(base + L::OFF_Q1 + c * L::BOX, &tm_q, c * 64, q_base1, bh, bar(L::BAR_Q), leader);
      }
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n1 && ok; ++j) {
        for (int which = 0; which < 2 && ok; ++which) {
          const int st = issued % L::STAGES;
          const uint32_t ph = (issued / L::STAGES) & 1;
          ok = mbar_wait(bar(L::BAR_KV_EMPTY + st), ph ^ 1u, wctx);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::BAR_KV_FULL + st), L::TILE, leader);
          const CUtensorMap* m = which ? &tm_v : &tm_k;
          for (int c = 0; c < L::KCH; ++c)
            tma_load_3d(base + L::OFF_KV + st * L::TILE + c * L::BOX, m, c * 64, j * 128, bh_kv,
                        bar(L::BAR_KV_FULL + st), leader);
          ++issued;
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      drain_wait(bar(L::BAR_Q), 0);
      const int first = issued > L::STAGES ? issued - L::STAGES : 0;
      for (int i = first; i < issued; ++i)
        drain_wait(bar(L::BAR_KV_FULL + (i % L::STAGES)), (i / L::STAGES) & 1);
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    regs_dec<kRegsLow>();
    {
      const uint32_t leader = elect_one();  // the lane that issues async instructions
      constexpr uint32_t idesc_qk = make_idesc(128, 128, true, false, false);
      constexpr uint32_t idesc_pv = make_idesc(128, D, false, false, true);  // fp16 P (TMEM) x fp16 V
      const uint32_t tS[2] = {tmem + L::T_S0, tmem + L::T_S1};
      const uint32_t tO[2] = {tmem + L::T_O0, tmem + L::T_O1};
      const uint32_t sQ[2] = {base + L::OFF_Q0, base + L::OFF_Q1};

      // descriptors are built once; each MMA only adds a constant byte offset
      const uint64_t dQ[2] = {make_sdesc_sw128(sQ[0], 16, 1024), make_sdesc_sw128(sQ[1], 16, 1024)};
      const uint64_t dKV0 = make_sdesc_sw128(base + L::OFF_KV, 16, 1024);       // K-major (K tiles)
      const uint64_t dV0 = make_sdesc_sw128(base + L::OFF_KV, L::BOX, 1024);    // MN-major (V tiles)
      auto issue_qk = [&](uint32_t d_tmem, uint64_t q_desc, int stage) {
        const uint64_t k_desc = sdesc_add(dKV0, stage * L::TILE);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * L::BOX + (k & 3) * 32;
          mma_ss(d_tmem, sdesc_add(q_desc, off), sdesc_add(k_desc, off), idesc_qk, k > 0 ? 1u : 0u, leader);
        }
      };
      // O += P V over keys [64 * part, 64 * part + 64) of the tile
      auto issue_pv_half = [&](uint32_t d_tmem, uint32_t p_tmem, int stage, bool acc, int part) {
        const uint64_t v_desc = sdesc_add(dV0, stage * L::TILE);
#pragma unroll
        for (int kk = 0; kk < L::BN / 32; ++kk) {
          const int k = part * (L::BN / 32) + kk;
          mma_ts(d_tmem, p_tmem + k * 8, sdesc_add(v_desc, k * 2048), idesc_pv, (acc || k > 0) ? 1u : 0u, leader);
        }
      };
      // the first half of the product starts while the softmax still computes the second half of P
      auto issue_pv = [&](int t, uint32_t d_tmem, uint32_t p_tmem, int stage, bool acc, uint32_t parity) -> bool {
        if (!mbar_wait(bar(L::BAR_P_HALF + t), parity, wctx)) return false;
        tc_fence_after();
        issue_pv_half(d_tmem, p_tmem, stage, acc, 0);
        if (!mbar_wait(bar(L::BAR_P_FULL + t), parity, wctx)) return false;
        tc_fence_after();
        issue_pv_half(d_tmem, p_tmem, stage, acc, 1);
        return true;
      };

      bool ok = mbar_wait(bar(L::BAR_Q), 0, wctx);
      tc_fence_after();
      int prev_v_stage = 0;
      for (int j = 0; j < n1 && ok; ++j) {
        const int iK = 2 * j, iV = 2 * j + 1;
        const int stK = iK % L::STAGES, stV = iV % L::STAGES;
        if (!(ok = mbar_wait(bar(L::BAR_KV_FULL + stK), (iK / L::STAGES) & 1, wctx))) break;
        tc_fence_after();
        if (j < n0) {
          issue_qk(tS[0], dQ[0], stK);
          mma_commit(bar(L::BAR_S_FULL + 0), leader);
        }
        if (j > 0) {  // O1 += P1 V_{j-1}
          if (!(ok = issue_pv(1, tO[1], tS[1], prev_v_stage, j - 1 > 0, (j - 1) & 1))) break;
          mma_commit(bar(L::BAR_KV_EMPTY + prev_v_stage), leader);
        }
        issue_qk(tS[1], dQ[1], stK);
        mma_commit(bar(L::BAR_S_FULL + 1), leader);
        mma_commit(bar(L::BAR_KV_EMPTY + stK), leader);
        if (!(ok = mbar_wait(bar(L::BAR_V_CONV + stV), (iV / L::STAGES) & 1, wctx))) break;
        tc_fence_after();
        if (j < n0) {  // O0 += P0 V_j
          if (!(ok = issue_pv(0, tO[0], tS[0], stV, j > 0, j & 1))) break;
          if (j == n0 - 1) mma_commit(bar(L::BAR_O_FULL + 0), leader);
        }
        prev_v_stage = stV;
      }
      if (ok) {  // O1 += P1 V_{n1-1}
        ok = issue_pv(1, tO[1], tS[1], prev_v_stage, n1 - 1 > 0, (n1 - 1) & 1);
        if (ok) {
          mma_commit(bar(L::BAR_KV_EMPTY + prev_v_stage), leader);
          mma_commit(bar(L::BAR_O_FULL + 1), leader);
        }
      }
      // every MMA issued so far has finished before TMEM is released
      mma_commit(bar(L::BAR_MMA_DONE), leader);
      drain_wait(bar(L::BAR_MMA_DONE), 0);
    }
  } else if (warp == 2 || warp == 3) {
    // ===================================================== V tiles: bf16 -> fp16 in place
    // Each tile is converted as V_j 2^v with v = 0 unless its largest |v| exceeds 2^15 (fp16
    // ends at 65504); then v in [-15, -1] brings that maximum into [2^14, 2^15).  The
    // exponent is published (BAR_V_EXP) after a first pass that finds the maximum, and the
    // softmax writes P 2^-v for this tile.  A tile beyond 2^15 even at v = -15 (|v| >= about
    // 2^31), or with a non-finite element, is recorded as kDevRange.
    regs_dec<kRegsLow>();
    const int ct = threadIdx.x - 64;  // 0..63
    volatile uint32_t* vamax = reinterpret_cast<volatile uint32_t*>(gbase + L::OFF_VAMAX);
    volatile int* vexp = reinterpret_cast<volatile int*>(gbase + L::OFF_VEXP);
    bool ok = true;
    for (int j = 0; j < n1 && ok; ++j) {
      const int iV = 2 * j + 1;
      const int st = iV % L::STAGES;
      if (!(ok = mbar_wait(bar(L::BAR_KV_FULL + st), (iV / L::STAGES) & 1, wctx))) break;
      uint4* tile = reinterpret_cast<uint4*>(gbase + L::OFF_KV + st * L::TILE);
      uint32_t am = 0u;  // largest |v| of the tile, as fp32 bits
#pragma unroll 4
      for (int i = ct; i < L::TILE / 16; i += kConvThreads) {
        const uint4 u = tile[i];
        am = abs_bits_max_bf16x2(abs_bits_max_bf16x2(am, u.x), u.y);
        am = abs_bits_max_bf16x2(abs_bits_max_bf16x2(am, u.z), u.w);
      }
      am = __reduce_max_sync(0xffffffffu, am);
      // the two warps' maxima, in a slot pair and barrier that alternate with the tile (a warp
      // writes pair j & 1 again only after the other one arrived for tile j + 1, i.e. after it
      // read pair j & 1); the wait is bounded like every other
      if (lane == 0) vamax[2 * (j & 1) + (warp - 2)] = am;
      mbar_arrive(bar(L::BAR_V_AMAX + (j & 1)));
      if (!(ok = mbar_wait(bar(L::BAR_V_AMAX + (j & 1)), (j >> 1) & 1, wctx))) break;
      am = max(vamax[2 * (j & 1)], vamax[2 * (j & 1) + 1]);
      int v = 0;
      if (am >= kBitsInf) {
        if (ct == 0) atomicExch(p.err, kDevRange);
      } else if (am > 0x47000000u) {  // > 2^15
        v = max(14 - floor_log2_bits(am), -15);
        if (ct == 0 && ldexpf(__uint_as_float(am), v) >= 65520.0f) atomicExch(p.err, kDevRange);
      }
      if (ct == 0) vexp[st] = v;
      mbar_arrive(bar(L::BAR_V_EXP + st));
      const float mult = __int_as_float((127 + v) << 23);  // 2^v
#pragma unroll 4
      for (int i = ct; i < L::TILE / 16; i += kConvThreads) {
        uint4 u = tile[i];
        uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
          w[e] = v == 0 ? pack_f16(f.x, f.y) : pack_f16(f.x * mult, f.y * mult);
        }
        tile[i] = u;
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(L::BAR_V_CONV + st));
    }
  } else if (warp >= 4) {
    // ===================================================== softmax warpgroups
    regs_inc<kRegsHigh>();
    const int t = (warp - 4) >> 2;        // query tile handled by this warpgroup
    const int wq = (warp - 4) & 3;        // TMEM lane quarter
    const int row = wq * 32 + lane;       // row inside the tile
    const int q_base = t ? q_base1 : q_base0;
    const int r = q_base + row;           // query index
    const int n_t = t ? n1 : n0;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + (t ? L::T_S1 : L::T_S0);
    const uint32_t tO = tmem + lane_off + (t ? L::T_O1 : L::T_O0);

    float m = -INFINITY;  // running max of scale*log2(e)*S (possibly stale by < 8)
    float l = 0.f;        // running sum of 2^(scale*log2(e)*S - m)
    bool ok = true;
    const int* vexp = reinterpret_cast<const int*>(gbase + L::OFF_VEXP);
    for (int j = 0; j < n_t; ++j) {
      const int iV = 2 * j + 1, stV = iV % L::STAGES;  // the stage holding V_j
      if (!(ok = fwd_softmax_step<D, false, true>(p, tS, tO, bar(L::BAR_S_FULL + t), j & 1, bar(L::BAR_P_HALF + t),
                                                  bar(L::BAR_P_FULL + t), j, j == 0, q_base, r, m, l, wctx, 0, 0,
                                                  bar(L::BAR_V_EXP + stV), (iV / L::STAGES) & 1, vexp + stV)))
        break;
    }
    // ---- epilogue: O / l -> bf16 -> swizzled staging (the Q tile's buffer) -> TMA store
    if (ok) ok = mbar_wait(bar(L::BAR_O_FULL + t), 0, wctx);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const uint32_t stage = base + (t ? L::OFF_Q1 : L::OFF_Q0);
      // 64-column chunks: O / l rounded to bf16 goes to the swizzled staging tile (one 64-column
      // TMA box); the bf16 residual goes straight to global memory, coalesced across the warp
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t u0[32], u1[32];
        tmem_ld32(tO + 64 * c, u0);
        tmem_ld32(tO + 64 * c + 32, u1);
        tmem_wait_ld();
        uint32_t pk[32], rk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t* uu = i < 16 ? u0 : u1;
          const int k = 2 * (i & 15);
          const float a = __uint_as_float(uu[k]) * inv_l, b = __uint_as_float(uu[k + 1]) * inv_l;
          pk[i] = pack_bf16(a, b);
          const float2 ab = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[i]));
          rk[i] = pack_bf16(a - ab.x, b - ab.y);
        }
        if (p.o_resid != nullptr) {
          uint4 ra[8];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) ra[q4] = make_uint4(rk[4 * q4], rk[4 * q4 + 1], rk[4 * q4 + 2], rk[4 * q4 + 3]);
          warp_store_rows_128b(ra, reinterpret_cast<uint8_t*>(p.o_resid + (size_t)bh * p.N * D + 64 * c), D * 2,
                               q_base + wq * 32, p.N);
        }
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          st_shared_v4(stage + c * L::BOX + sw128_offset(row, q4), pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2],
                       pk[4 * q4 + 3]);
      }
      if (p.lse != nullptr && r < p.N) p.lse[(size_t)bh * p.N + r] = (m + __log2f(l)) * 0.69314718055994531f;
      fence_proxy_async_smem();
    }
    named_bar_sync(1 + t, 128);
    if (ok && row == 0) {
      const uint32_t stage = base + (t ? L::OFF_Q1 : L::OFF_Q0);
      for (int c = 0; c < L::KCH; ++c) tma_store_3d(&tm_o, c * 64, q_base, bh, stage + c * L::BOX);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace

namespace {
// ============================================================================ persistent
// Persistent forward (fa_fwd_ws): one CTA per SM takes work units (pairs of 128-row query
// tiles) one after another from a work counter in the caller's workspace (zeroed by the V
// conversion pass), in the order of unit_order; the producer warp takes each index and
// publishes it to the other roles through a two-slot ring in shared memory (an index >=
// the unit count means "no more work").  The next unit's Q loads and first Q K^T products
// overlap the previous unit's last steps and epilogue.  V is fp16 already.  K/V ring
// positions count loads across units, the per-tile barriers (S_FULL, P_HALF, P_FULL)
// count that tile's steps across units, and the per-unit barriers (Q_FULL, Q_EMPTY,
// O_FULL, O_FREE) count units.  O and the residual leave through a 4 KB staging box per
// softmax warp (its 32 rows x 64 columns, 128-byte swizzle) and one bulk tensor store per box
// (the Q buffers are reloaded for the next unit and cannot serve as staging).
//
// F8 (8-bit inputs, d = 128 or 64): Q, K and V are E4M3, so a row of d elements is one
// 128-byte swizzle row (d = 128; 16 KB tiles) or one 64-byte swizzle row (d = 64; 8 KB tiles);
// S = Q K^T and O += P V run as kind::f8f6f4 products (K = 32 per instruction), V read
// MN-major straight from its (N, d) layout, P written to TMEM as E4M3; the per-tensor
// descales enter through scale_log2 (Q, K) and out_scale (V).
template <int D, bool F8 = false>
struct FwdPLayout {
  static constexpr int ROW_BYTES = F8 ? D : 2 * D;  // bytes of one row of Q, K or V
  static constexpr int SW = ROW_BYTES < 128 ? 64 : 128;  // swizzle span: bytes of one column chunk row
  static_assert(ROW_BYTES % SW == 0, "rows are whole swizzle rows");
  static constexpr int CH_ELEMS = F8 ? SW : SW / 2;  // elements of one column chunk
  static constexpr int KCH = ROW_BYTES / SW;
  static constexpr int BOX = 128 * SW;                // one chunk of 128 rows
  static constexpr int TILE = KCH * BOX;
  static constexpr int STAGES = (TILE == 2 * BOX) ? 4 : 8;
  static constexpr int K_STEP = F8 ? 32 : 16;          // K of one tensor-core instruction
  static constexpr int QK_STEPS = ROW_BYTES / 32;      // instructions per Q K^T (32 bytes of K each)
  static constexpr int QK_STEPS_CH = SW / 32;          // of which inside one column chunk
  static constexpr int ATOM = 8 * SW;                  // bytes of an 8-row swizzle atom
  static constexpr int PARTS = kFwdParts;              // P handed to the tensor core in PARTS parts
  static constexpr int PV_STEPS_PART = 128 / PARTS / K_STEP;  // instructions per part of P V
  static constexpr int PV_B_STEP = K_STEP * SW;        // bytes between the V rows of consecutive steps
  static constexpr int OFF_Q0 = 0;
  static constexpr int OFF_Q1 = TILE;
  static constexpr int OFF_KV = 2 * TILE;
  // epilogue staging: one 32-row x 128-byte swizzled box per softmax warp
  static constexpr int OFF_STG = OFF_KV + STAGES * TILE;
  static constexpr int OFF_BAR = OFF_STG + 8 * 4096;
  static constexpr int BAR_Q_FULL = 0;
  static constexpr int BAR_Q_EMPTY = 1;
  static constexpr int BAR_KV_FULL = 2;
  static constexpr int BAR_KV_EMPTY = 2 + STAGES;
  static constexpr int BAR_S_FULL = 2 + 2 * STAGES;  // [2]
  static constexpr int BAR_P_PART = BAR_S_FULL + 2;  // [PARTS][2]: part h of tile t at BAR_P_PART + t + 2 h
  static constexpr int BAR_O_FULL = BAR_P_PART + 2 * PARTS;  // [2]
  static constexpr int BAR_O_FREE = BAR_O_FULL + 2;  // [2] a tile's epilogue has read O out of TMEM
  static constexpr int BAR_UNIT_FULL = BAR_O_FREE + 2;   // [2]
  static constexpr int BAR_UNIT_EMPTY = BAR_UNIT_FULL + 2;  // [2]
  static constexpr int BAR_MMA_DONE = BAR_UNIT_EMPTY + 2;
  static constexpr int NBAR = BAR_MMA_DONE + 1;
  static constexpr int OFF_UNIT = OFF_BAR + NBAR * 8;  // int[2]
  static constexpr int OFF_TMEM_SLOT = OFF_UNIT + 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM_ALLOC = OFF_ABORT + 8 + 1024;
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O0 = 256, T_O1 = 256 + D;
};

template <int D, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_persist_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o32,
                                const __grid_constant__ CUtensorMap tm_r32, const FwdParams p) {
  using L = FwdPLayout<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_units = p.n_pairs * p.BH;
  // a unit's key tiles: tile t (rows q_base0 + 128 t .. + 127) needs key tiles jlo_t .. jhi_t
  // (causal mask and sliding window); jlo0 <= jlo1 <= jhi0 + 1 and jhi0 <= jhi1, so the
  // unit streams jlo0 .. jhi1 once for both tiles
  struct Unit {
    int bh, bh_kv, q_base0, jlo0, jhi0, jlo1, jhi1;
  };
  auto unit_of = [&](int u) -> Unit {
    Unit x;
    int rank;
    unit_order(u, p.n_pairs, p.BH, p.head_group, x.bh, rank);
    const int pair = p.causal ? (p.n_pairs - 1 - rank) : rank;
    x.bh_kv = kv_head_of(x.bh, p.H, p.H_kv);
    x.q_base0 = pair * 256;
    x.jlo0 = key_lo(x.q_base0, p.N, p.win_left) / 128;
    x.jhi0 = key_hi(x.q_base0 + 127, p.N, p.causal, p.win_right) / 128;
    x.jlo1 = key_lo(x.q_base0 + 128, p.N, p.win_left) / 128;
    x.jhi1 = key_hi(x.q_base0 + 255, p.N, p.causal, p.win_right) / 128;
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
    mbar_init(bar(L::BAR_Q_FULL), 1);
    mbar_init(bar(L::BAR_Q_EMPTY), 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::BAR_KV_FULL + s), 1);
      mbar_init(bar(L::BAR_KV_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::BAR_S_FULL + t), 1);
      for (int h = 0; h < L::PARTS; ++h) mbar_init(bar(L::BAR_P_PART + t + 2 * h), 128);
      mbar_init(bar(L::BAR_O_FULL + t), 1);
      mbar_init(bar(L::BAR_O_FREE + t), 128);
      mbar_init(bar(L::BAR_UNIT_FULL + t), 1);
      mbar_init(bar(L::BAR_UNIT_EMPTY + t), 1 + 256);
    }
    mbar_init(bar(L::BAR_MMA_DONE), 1);
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
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    int issued = 0, q_issued = 0;
    bool ok = true;
    for (int uc = 0;; ++uc) {
      // the ring slot is free once every consumer has read unit uc - 2
      if (uc >= 2 && !(ok = mbar_wait(bar(L::BAR_UNIT_EMPTY + (uc & 1)), ((uc - 2) >> 1) & 1, wctx))) break;
      int u = 0;
      if (lane == 0) u = (int)atomicAdd(p.counter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (lane == 0) {
        unit_ring[uc & 1] = u < n_units ? u : n_units;
        mbar_arrive(bar(L::BAR_UNIT_FULL + (uc & 1)));
      }
      __syncwarp();
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      // this unit's Q tiles replace the previous unit's once its last Q K^T products completed
      if (uc > 0 && !(ok = mbar_wait(bar(L::BAR_Q_EMPTY), (uc - 1) & 1, wctx))) break;
      mbar_arrive_expect_tx(bar(L::BAR_Q_FULL), 2 * L::TILE, leader);
      for (int c = 0; c < L::KCH; ++c) {
        tma_load_3d(base + L::OFF_Q0 + c * L::BOX, &tm_q, c * L::CH_ELEMS, x.q_base0, x.bh, bar(L::BAR_Q_FULL),
                    leader);
        tma_load_3d(base + L::OFF_Q1 + c * L::BOX, &tm_q, c * L::CH_ELEMS, x.q_base0 + 128, x.bh,
                    bar(L::BAR_Q_FULL), leader);
      }
      ++q_issued;
      for (int j = x.jlo0; j <= x.jhi1 && ok; ++j) {
        for (int which = 0; which < 2; ++which) {
          const int st = issued % L::STAGES;
          if (!(ok = mbar_wait(bar(L::BAR_KV_EMPTY + st), ((issued / L::STAGES) & 1) ^ 1u, wctx))) break;
          mbar_arrive_expect_tx(bar(L::BAR_KV_FULL + st), L::TILE, leader);
          const CUtensorMap* m = which ? &tm_v : &tm_k;
          for (int c = 0; c < L::KCH; ++c)
            tma_load_3d(base + L::OFF_KV + st * L::TILE + c * L::BOX, m, c * L::CH_ELEMS, j * 128, x.bh_kv,
                        bar(L::BAR_KV_FULL + st), leader);
          ++issued;
        }
      }
      if (!ok) break;
    }
    // drain: every issued copy has landed before the CTA may exit
    if (q_issued > 0) drain_wait(bar(L::BAR_Q_FULL), (q_issued - 1) & 1);
    for (int i = (issued > L::STAGES ? issued - L::STAGES : 0); i < issued; ++i)
      drain_wait(bar(L::BAR_KV_FULL + (i % L::STAGES)), (i / L::STAGES) & 1);
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    // bf16 Q, K (format 1), or E4M3 (format 0 of kind::f8f6f4; 1 there would mean E5M2)
    constexpr uint32_t idesc_qk = make_idesc(128, 128, !F8, false, false);
    // fp16 P (TMEM) x fp16 V, or E4M3 x E4M3 (format code 0 in both kinds); V MN-major
    constexpr uint32_t idesc_pv = make_idesc(128, D, false, false, true);
    const uint32_t tS[2] = {tmem + L::T_S0, tmem + L::T_S1};
    const uint32_t tO[2] = {tmem + L::T_O0, tmem + L::T_O1};
    auto sdesc = [](uint32_t saddr, uint32_t lbo) -> uint64_t {
      return L::SW == 128 ? make_sdesc_sw128(saddr, lbo, L::ATOM) : make_sdesc_sw64(saddr, lbo, L::ATOM);
    };
    const uint64_t dQ[2] = {sdesc(base + L::OFF_Q0, 16), sdesc(base + L::OFF_Q1, 16)};
    const uint64_t dKV0 = sdesc(base + L::OFF_KV, 16);     // K-major (K tiles)
    const uint64_t dV0 = sdesc(base + L::OFF_KV, L::BOX);  // MN-major (V tiles)
    auto issue_qk = [&](uint32_t d_tmem, uint64_t q_desc, int stage) {
      const uint64_t k_desc = sdesc_add(dKV0, stage * L::TILE);
#pragma unroll
      for (int k = 0; k < L::QK_STEPS; ++k) {
        const uint32_t off = (k / L::QK_STEPS_CH) * L::BOX + (k % L::QK_STEPS_CH) * 32;
        if constexpr (F8)
          mma_ss_f8(d_tmem, sdesc_add(q_desc, off), sdesc_add(k_desc, off), idesc_qk, k > 0 ? 1u : 0u, leader);
        else
          mma_ss(d_tmem, sdesc_add(q_desc, off), sdesc_add(k_desc, off), idesc_qk, k > 0 ? 1u : 0u, leader);
      }
    };
    // P for keys [K_STEP k, K_STEP (k + 1)) sits in TMEM columns [8 k, 8 k + 8) in both forms
    auto issue_pv_part = [&](uint32_t d_tmem, uint32_t p_tmem, int stage, bool acc, int part) {
      const uint64_t v_desc = sdesc_add(dV0, stage * L::TILE);
#pragma unroll
      for (int kk = 0; kk < L::PV_STEPS_PART; ++kk) {
        const int k = part * L::PV_STEPS_PART + kk;
        if constexpr (F8)
          mma_ts_f8(d_tmem, p_tmem + k * 8, sdesc_add(v_desc, k * L::PV_B_STEP), idesc_pv, (acc || k > 0) ? 1u : 0u,
                    leader);
        else
          mma_ts(d_tmem, p_tmem + k * 8, sdesc_add(v_desc, k * L::PV_B_STEP), idesc_pv, (acc || k > 0) ? 1u : 0u,
                 leader);
      }
    };
    int L0 = 0, G0 = 0, G1 = 0;  // K/V loads and tile steps of the previous units
    bool ok = true;
    // O_t += P_t V (tile t's local step jt, K/V stage st); before a unit's first product
    // into O_t the previous unit's epilogue must have read O_t out of TMEM
    auto issue_pv = [&](int t, int jt, int stage, int uc) -> bool {
      if (jt == 0 && uc > 0) {
        if (!mbar_wait(bar(L::BAR_O_FREE + t), (uc - 1) & 1, wctx)) return false;
        tc_fence_after();
      }
      const uint32_t ph = ((t ? G1 : G0) + jt) & 1;
      for (int h = 0; h < L::PARTS; ++h) {
        if (!mbar_wait(bar(L::BAR_P_PART + t + 2 * h), ph, wctx)) return false;
        tc_fence_after();
        issue_pv_part(tO[t], tS[t], stage, jt > 0, h);
      }
      return true;
    };
    for (int uc = 0; ok; ++uc) {
      const int u = next_unit(uc, ok);
      if (lane == 0) mbar_arrive(bar(L::BAR_UNIT_EMPTY + (uc & 1)));
      if (!ok || u >= n_units) break;
      const Unit x = unit_of(u);
      if (!(ok = mbar_wait(bar(L::BAR_Q_FULL), uc & 1, wctx))) break;
      tc_fence_after();
      // per key tile j of the unit's stream: S0_j, O1 += P1 V_(tile 1's previous step), S1_j,
      // O0 += P0 V_j -- each only where tile 0 / tile 1 has j in its range
      int pend1 = -1;        // K/V stage of the V tile of tile 1's pending P V
      int jt0 = 0, jt1 = 0;  // steps of tile 0 / tile 1 so far in this unit
      for (int j = x.jlo0; j <= x.jhi1 && ok; ++j) {
        const int li = j - x.jlo0;
        const int iK = L0 + 2 * li, iV = iK + 1;
        const int stK = iK % L::STAGES, stV = iV % L::STAGES;
        const bool in0 = j <= x.jhi0, in1 = j >= x.jlo1;
        if (!(ok = mbar_wait(bar(L::BAR_KV_FULL + stK), (iK / L::STAGES) & 1, wctx))) break;
        tc_fence_after();
        if (in0) {
          issue_qk(tS[0], dQ[0], stK);
          mma_commit(bar(L::BAR_S_FULL + 0), leader);
        }
        if (in1 && pend1 >= 0) {  // O1 += P1 V of tile 1's previous step
          if (!(ok = issue_pv(1, jt1 - 1, pend1, uc))) break;
          mma_commit(bar(L::BAR_KV_EMPTY + pend1), leader);
        }
        if (in1) {
          issue_qk(tS[1], dQ[1], stK);
          mma_commit(bar(L::BAR_S_FULL + 1), leader);
        }
        mma_commit(bar(L::BAR_KV_EMPTY + stK), leader);
        if (j == x.jhi1) mma_commit(bar(L::BAR_Q_EMPTY), leader);  // the unit's last Q K^T
        if (!(ok = mbar_wait(bar(L::BAR_KV_FULL + stV), (iV / L::STAGES) & 1, wctx))) break;
        tc_fence_after();
        if (in0) {  // O0 += P0 V_j
          if (!(ok = issue_pv(0, jt0, stV, uc))) break;
          if (j == x.jhi0) mma_commit(bar(L::BAR_O_FULL + 0), leader);
          if (!in1) mma_commit(bar(L::BAR_KV_EMPTY + stV), leader);  // tile 1 does not use V_j
          ++jt0;
        }
        if (in1) {
          pend1 = stV;
          ++jt1;
        }
      }
      if (!ok) break;
      if (!(ok = issue_pv(1, jt1 - 1, pend1, uc))) break;  // tile 1's last P V
      mma_commit(bar(L::BAR_KV_EMPTY + pend1), leader);
      mma_commit(bar(L::BAR_O_FULL + 1), leader);
      L0 += 2 * (x.jhi1 - x.jlo0 + 1);
      G0 += jt0;
      G1 += jt1;
    }
    // every MMA issued so far has finished before TMEM is released
    mma_commit(bar(L::BAR_MMA_DONE), leader);
    drain_wait(bar(L::BAR_MMA_DONE), 0);
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle (V is fp16 already)
  } else {
    // ===================================================== softmax warpgroups
    regs_inc<kRegsHigh>();
    const int t = (warp - 4) >> 2;   // query tile handled by this warpgroup
    const int wq = (warp - 4) & 3;   // TMEM lane quarter
    const int row = wq * 32 + lane;  // row inside the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + (t ? L::T_S1 : L::T_S0);
    const uint32_t tO = tmem + lane_off + (t ? L::T_O1 : L::T_O0);
    // the V copy is V 2^e (one exponent for the tensor): O / l is divided by 2^e
    const float out_scale = p.v_exp != nullptr ? ldexpf(p.out_scale, -*p.v_exp) : p.out_scale;
    bool ok = true;
    int G = 0;  // this tile's steps in the previous units
    int u = next_unit(0, ok);
    mbar_arrive(bar(L::BAR_UNIT_EMPTY + 0));
    for (int uc = 0; ok && u < n_units; ++uc) {
      const Unit x = unit_of(u);
      const int q_base = x.q_base0 + 128 * t;
      const int r = q_base + row;  // query index
      const int jlo = t ? x.jlo1 : x.jlo0;
      const int n_t = (t ? x.jhi1 : x.jhi0) - jlo + 1;
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < n_t; ++jj) {
        if (!(ok = fwd_softmax_step<D, F8, false, L::PARTS>(p, tS, tO, bar(L::BAR_S_FULL + t), (G + jj) & 1,
                                                            bar(L::BAR_P_PART + t), bar(L::BAR_P_PART + t + 2),
                                                            jlo + jj, jj == 0, q_base, r, m, l, wctx)))
          break;
      }
      G += n_t;
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 and the bf16 residual
      if (!(ok = mbar_wait(bar(L::BAR_O_FULL + t), uc & 1, wctx))) break;
      tc_fence_after();
      const float inv_l = out_scale / l;
      // this warp's 32 rows through its swizzled staging box, one bulk tensor store per
      // 64-column chunk (and per residual chunk); a box is rewritten only after the
      // previous store has read it
      const uint32_t stg = base + L::OFF_STG + (uint32_t)(warp - 4) * 4096u;
      auto stage_and_store = [&](const uint32_t (&w)[32], const CUtensorMap* m, int col) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          st_shared_v4(stg + sw128_offset(lane, q4), w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(m, col, q_base + wq * 32, x.bh, stg);
          bulk_commit_group();
        }
      };
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t u0[32], u1[32];
        tmem_ld32(tO + 64 * c, u0);
        tmem_ld32(tO + 64 * c + 32, u1);
        tmem_wait_ld();
        if (c == D / 64 - 1) {  // O_t fully read: the next unit may overwrite it
          tc_fence_before();
          mbar_arrive(bar(L::BAR_O_FREE + t));
        }
        uint32_t pk[32], rk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t* uu = i < 16 ? u0 : u1;
          const int k2 = 2 * (i & 15);
          const float a = __uint_as_float(uu[k2]) * inv_l, b = __uint_as_float(uu[k2 + 1]) * inv_l;
          pk[i] = pack_bf16(a, b);
          const float2 ab = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[i]));
          rk[i] = pack_bf16(a - ab.x, b - ab.y);
        }
        stage_and_store(pk, &tm_o32, 64 * c);
        if (p.o_resid != nullptr) stage_and_store(rk, &tm_r32, 64 * c);
      }
      if (p.lse != nullptr && r < p.N) p.lse[(size_t)x.bh * p.N + r] = (m + __log2f(l)) * 0.69314718055994531f;
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

// ============================================================================ head dim 256
// Persistent forward for d = 256 (fa_fwd_ws / fa_attn_fwd with d = 256).  A 128-row tile
// needs S (128 TMEM columns) and O (256), so two tiles do not fit in the 512 columns: a unit
// is ONE 128-row query tile, S is double-buffered (S_A, S_B) and the tensor core runs
// S_{j+1} = Q K_{j+1}^T while the softmax warpgroup turns S_j into P_j; the issue order is
// S_0, S_1, PV_0, S_2, PV_1, ..., so the softmax of step j has the time of S_{j+1} and PV_{j-1}
// (~2100 cycles) to finish.  PV_{j-1} is issued after S_j, so a rescale of O in the softmax
// of step j first waits for PV_{j-1} to complete (BAR_PV_DONE; rescales are rare: the running
// maximum may lag by < 2^8).
// Shared memory: Q (4 boxes of 128 x 64 bf16, 64 KB) and a FIFO of 32 KB slots filled in the
// order the tensor core consumes them -- K_0, K_1, V_0, K_2, V_1, ..., V_{n-1} -- so one running
// index serves producer and issuer.  A K slot holds one d-half of K_j (two 128 x 64 boxes,
// K-major); a V slot holds one key-half of V_j (four 64-key x 64-column fp16 boxes, read
// MN-major by the N = 256 P V products).
struct FwdWLayout {
  static constexpr int D = 256;
  static constexpr int BOX = 128 * 128;  // 128 rows x 64 bf16 columns (Q, K boxes)
  static constexpr int VBOX = 64 * 128;  // 64 rows x 64 fp16 columns (V boxes)
  static constexpr int SLOT = 32768;
  static constexpr int SLOTS = 5;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = 4 * BOX;
  static constexpr int OFF_BAR = OFF_RING + SLOTS * SLOT;
  static constexpr int BAR_Q_FULL = 0;
  static constexpr int BAR_Q_EMPTY = 1;
  static constexpr int BAR_SLOT_FULL = 2;                    // [SLOTS]
  static constexpr int BAR_SLOT_EMPTY = 2 + SLOTS;           // [SLOTS]
  static constexpr int BAR_S_FULL = 2 + 2 * SLOTS;           // [2]
  static constexpr int BAR_P_HALF = BAR_S_FULL + 2;          // [2]
  static constexpr int BAR_P_FULL = BAR_P_HALF + 2;          // [2]
  static constexpr int BAR_PV_DONE = BAR_P_FULL + 2;         // one phase per P V product
  static constexpr int BAR_O_FULL = BAR_PV_DONE + 1;         // a unit's last P V completed
  static constexpr int BAR_O_FREE = BAR_O_FULL + 1;          // the epilogue has read O out of TMEM
  static constexpr int BAR_UNIT_FULL = BAR_O_FREE + 1;       // [2]
  static constexpr int BAR_UNIT_EMPTY = BAR_UNIT_FULL + 2;   // [2]
  static constexpr int BAR_MMA_DONE = BAR_UNIT_EMPTY + 2;
  static constexpr int NBAR = BAR_MMA_DONE + 1;
  static constexpr int OFF_UNIT = OFF_BAR + NBAR * 8;  // int[2]
  static constexpr int OFF_TMEM_SLOT = OFF_UNIT + 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM_ALLOC = OFF_ABORT + 8 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O = 256;
};
static_assert(FwdWLayout::SMEM_ALLOC <= 232448, "d = 256 forward exceeds the shared memory of a CTA");

__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_d256_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdWLayout;
  constexpr int D = L::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_qt = (p.N + 127) / 128;
  const int n_units = n_qt * p.BH;
  struct Unit {
    int bh, bh_kv, q_base, jlo, n;  // key tiles jlo .. jlo + n - 1
  };
  auto unit_of = [&](int u) -> Unit {
    Unit x;
    int rank;
    unit_order(u, n_qt, p.BH, p.head_group, x.bh, rank);
    const int qt = p.causal ? (n_qt - 1 - rank) : rank;
    x.bh_kv = kv_head_of(x.bh, p.H, p.H_kv);
    x.q_base = qt * 128;
    x.jlo = key_lo(x.q_base, p.N, p.win_left) / 128;
    x.n = key_hi(x.q_base + 127, p.N, p.causal, p.win_right) / 128 - x.jlo + 1;  // >= 1
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
    mbar_init(bar(L::BAR_Q_FULL), 1);
    mbar_init(bar(L::BAR_Q_EMPTY), 1);
    for (int s = 0; s < L::SLOTS; ++s) {
      mbar_init(bar(L::BAR_SLOT_FULL + s), 1);
      mbar_init(bar(L::BAR_SLOT_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::BAR_S_FULL + t), 1);
      mbar_init(bar(L::BAR_P_HALF + t), 128);
      mbar_init(bar(L::BAR_P_FULL + t), 128);
      mbar_init(bar(L::BAR_UNIT_FULL + t), 1);
      mbar_init(bar(L::BAR_UNIT_EMPTY + t), 1 + 128);
    }
    mbar_init(bar(L::BAR_PV_DONE), 1);
    mbar_init(bar(L::BAR_O_FULL), 1);
    mbar_init(bar(L::BAR_O_FREE), 128);
    mbar_init(bar(L::BAR_MMA_DONE), 1);
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
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    int issued = 0, q_issued = 0;  // FIFO slot loads and Q loads so far
    bool ok = true;
    // one FIFO entry: the K d-half (kind 0) or V key-half (kind 1) `half` of key tile j
    auto load_slot = [&](int kind, int j, int half, int bh_kv) -> bool {
      const int st = issued % L::SLOTS;
      if (!mbar_wait(bar(L::BAR_SLOT_EMPTY + st), ((issued / L::SLOTS) & 1) ^ 1u, wctx)) return false;
      const uint32_t dst = base + L::OFF_RING + st * L::SLOT;
      mbar_arrive_expect_tx(bar(L::BAR_SLOT_FULL + st), L::SLOT, leader);
      if (kind == 0) {
        for (int c = 0; c < 2; ++c)
          tma_load_3d(dst + c * L::BOX, &tm_k, (2 * half + c) * 64, j * 128, bh_kv, bar(L::BAR_SLOT_FULL + st),
                      leader);
      } else {
        for (int c = 0; c < 4; ++c)
          tma_load_3d(dst + c * L::VBOX, &tm_v, c * 64, j * 128 + 64 * half, bh_kv, bar(L::BAR_SLOT_FULL + st),
                      leader);
      }
      ++issued;
      return true;
    };
    for (int uc = 0;; ++uc) {
      if (uc >= 2 && !(ok = mbar_wait(bar(L::BAR_UNIT_EMPTY + (uc & 1)), ((uc - 2) >> 1) & 1, wctx))) break;
      int u = 0;
      if (lane == 0) u = (int)atomicAdd(p.counter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (lane == 0) {
        unit_ring[uc & 1] = u < n_units ? u : n_units;
        mbar_arrive(bar(L::BAR_UNIT_FULL + (uc & 1)));
      }
      __syncwarp();
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      if (uc > 0 && !(ok = mbar_wait(bar(L::BAR_Q_EMPTY), (uc - 1) & 1, wctx))) break;
      mbar_arrive_expect_tx(bar(L::BAR_Q_FULL), 4 * L::BOX, leader);
      for (int c = 0; c < 4; ++c)
        tma_load_3d(base + L::OFF_Q + c * L::BOX, &tm_q, c * 64, x.q_base, x.bh, bar(L::BAR_Q_FULL), leader);
      ++q_issued;
      // consumption order: K_0, then K_{t+1}, V_t for t = 0 .. n - 2, then V_{n-1}
      for (int h = 0; h < 2 && ok; ++h) ok = load_slot(0, x.jlo, h, x.bh_kv);
      for (int t = 0; t < x.n && ok; ++t) {
        if (t + 1 < x.n)
          for (int h = 0; h < 2 && ok; ++h) ok = load_slot(0, x.jlo + t + 1, h, x.bh_kv);
        for (int h = 0; h < 2 && ok; ++h) ok = load_slot(1, x.jlo + t, h, x.bh_kv);
      }
      if (!ok) break;
    }
    if (q_issued > 0) drain_wait(bar(L::BAR_Q_FULL), (q_issued - 1) & 1);
    for (int i = (issued > L::SLOTS ? issued - L::SLOTS : 0); i < issued; ++i)
      drain_wait(bar(L::BAR_SLOT_FULL + (i % L::SLOTS)), (i / L::SLOTS) & 1);
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    regs_dec<kRegsLow>();
    const uint32_t leader = elect_one();
    constexpr uint32_t idesc_qk = make_idesc(128, 128, true, false, false);  // bf16 Q, K; K-major
    constexpr uint32_t idesc_pv = make_idesc(128, D, false, false, true);    // fp16 P (TMEM) x fp16 V, MN-major
    const uint32_t tS[2] = {tmem + L::T_S0, tmem + L::T_S1};
    const uint32_t tO = tmem + L::T_O;
    const uint64_t dQ = make_sdesc_sw128(base + L::OFF_Q, 16, 1024);
    const uint64_t dRingK = make_sdesc_sw128(base + L::OFF_RING, 16, 1024);       // K slots, K-major
    const uint64_t dRingV = make_sdesc_sw128(base + L::OFF_RING, L::VBOX, 1024);  // V slots, MN-major
    int consumed = 0;  // FIFO entries consumed so far
    int T = 0;         // S / P buffer steps so far (all units)
    bool ok = true;
    auto take = [&]() -> int {  // wait for the next FIFO entry, return its slot
      const int st = consumed % L::SLOTS;
      ok = mbar_wait(bar(L::BAR_SLOT_FULL + st), (consumed / L::SLOTS) & 1, wctx);
      ++consumed;
      return st;
    };
    // S_T = Q K_j^T: 16 products over d, the two d-halves from two FIFO entries
    auto issue_qk = [&](int b) -> bool {
      for (int h = 0; h < 2; ++h) {
        const int st = take();
        if (!ok) return false;
        tc_fence_after();
        const uint64_t k_desc = sdesc_add(dRingK, st * L::SLOT);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t qoff = (2 * h + (k >> 2)) * L::BOX + (k & 3) * 32;
          const uint32_t koff = (k >> 2) * L::BOX + (k & 3) * 32;
          mma_ss(tS[b], sdesc_add(dQ, qoff), sdesc_add(k_desc, koff), idesc_qk, (h | k) > 0 ? 1u : 0u, leader);
        }
        mma_commit(bar(L::BAR_SLOT_EMPTY + st), leader);
      }
      mma_commit(bar(L::BAR_S_FULL + b), leader);
      return true;
    };
    // O += P_t V_t (t: step of this unit, Tt: global step): the two key-halves from two FIFO
    // entries, each after its half of P is in TMEM
    auto issue_pv = [&](int t, int Tt, int uc) -> bool {
      const int b = Tt & 1;
      const uint32_t ph = (Tt >> 1) & 1;
      if (t == 0 && uc > 0) {  // the previous unit's epilogue has read O
        if (!mbar_wait(bar(L::BAR_O_FREE), (uc - 1) & 1, wctx)) return false;
        tc_fence_after();
      }
      for (int h = 0; h < 2; ++h) {
        const int st = take();
        if (!ok) return false;
        if (!mbar_wait(bar(h == 0 ? L::BAR_P_HALF + b : L::BAR_P_FULL + b), ph, wctx)) return false;
        tc_fence_after();
        const uint64_t v_desc = sdesc_add(dRingV, st * L::SLOT);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int k = 4 * h + kk;  // 16-key step
          mma_ts(tO, tS[b] + k * 8, sdesc_add(v_desc, kk * 2048), idesc_pv, (t > 0 || k > 0) ? 1u : 0u, leader);
        }
        mma_commit(bar(L::BAR_SLOT_EMPTY + st), leader);
      }
      mma_commit(bar(L::BAR_PV_DONE), leader);
      return true;
    };
    for (int uc = 0; ok; ++uc) {
      const int u = next_unit(uc, ok);
      if (lane == 0) mbar_arrive(bar(L::BAR_UNIT_EMPTY + (uc & 1)));
      if (!ok || u >= n_units) break;
      const Unit x = unit_of(u);
      if (!(ok = mbar_wait(bar(L::BAR_Q_FULL), uc & 1, wctx))) break;
      tc_fence_after();
      const int T0 = T;
      if (!(ok = issue_qk(T & 1))) break;  // S_0
      ++T;
      for (int t = 1; t < x.n && ok; ++t) {
        ok = issue_qk(T & 1);  // S_t
        if (!ok) break;
        if (t == x.n - 1) mma_commit(bar(L::BAR_Q_EMPTY), leader);  // the unit's last Q K^T
        ++T;
        ok = issue_pv(t - 1, T0 + t - 1, uc);
      }
      if (!ok) break;
      if (x.n == 1) mma_commit(bar(L::BAR_Q_EMPTY), leader);
      if (!(ok = issue_pv(x.n - 1, T0 + x.n - 1, uc))) break;
      mma_commit(bar(L::BAR_O_FULL), leader);
    }
    mma_commit(bar(L::BAR_MMA_DONE), leader);
    drain_wait(bar(L::BAR_MMA_DONE), 0);
  } else if (warp < 4 || warp >= 8) {
    regs_dec<kRegsLow>();  // warps 2-3 and 8-11: idle
  } else {
    // ===================================================== softmax + epilogue warpgroup
    regs_inc<kRegsHigh>();
    const int wq = warp - 4;         // TMEM lane quarter
    const int row = wq * 32 + lane;  // row inside the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + L::T_O;
    const float out_scale = p.v_exp != nullptr ? ldexpf(p.out_scale, -*p.v_exp) : p.out_scale;  // V copy: V 2^e
    bool ok = true;
    int T = 0;
    int u = next_unit(0, ok);
    mbar_arrive(bar(L::BAR_UNIT_EMPTY + 0));
    for (int uc = 0; ok && u < n_units; ++uc) {
      const Unit x = unit_of(u);
      const int r = x.q_base + row;
      float m = -INFINITY, l = 0.f;
      for (int t = 0; t < x.n; ++t, ++T) {
        const int b = T & 1;
        const uint32_t tS = tmem + lane_off + (b ? L::T_S1 : L::T_S0);
        // a rescale of O waits for the previous step's P V (global product T - 1)
        if (!(ok = fwd_softmax_step<D>(p, tS, tO, bar(L::BAR_S_FULL + b), (T >> 1) & 1, bar(L::BAR_P_HALF + b),
                                       bar(L::BAR_P_FULL + b), x.jlo + t, t == 0, x.q_base, r, m, l, wctx,
                                       bar(L::BAR_PV_DONE), (uint32_t)((T - 1) & 1))))
          break;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 and the bf16 residual, stored from registers
      if (!(ok = mbar_wait(bar(L::BAR_O_FULL), uc & 1, wctx))) break;
      tc_fence_after();
      const float inv_l = out_scale / l;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t u0[32], u1[32];
        tmem_ld32(tO + 64 * c, u0);
        tmem_ld32(tO + 64 * c + 32, u1);
        tmem_wait_ld();
        if (c == D / 64 - 1) {  // O fully read: the next unit may accumulate into it
          tc_fence_before();
          mbar_arrive(bar(L::BAR_O_FREE));
        }
        uint4 oa[8], ra[8];
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          uint32_t pk[4], rk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * q4 + e;
            const uint32_t* uu = i < 16 ? u0 : u1;
            const int k = 2 * (i & 15);
            const float a = __uint_as_float(uu[k]) * inv_l, bb = __uint_as_float(uu[k + 1]) * inv_l;
            pk[e] = pack_bf16(a, bb);
            const float2 ab = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[e]));
            rk[e] = pack_bf16(a - ab.x, bb - ab.y);
          }
          oa[q4] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          ra[q4] = make_uint4(rk[0], rk[1], rk[2], rk[3]);
        }
        warp_store_rows_128b(oa, reinterpret_cast<uint8_t*>(p.o + (size_t)x.bh * p.N * D + 64 * c), D * 2,
                             x.q_base + wq * 32, p.N);
        if (p.o_resid != nullptr)
          warp_store_rows_128b(ra, reinterpret_cast<uint8_t*>(p.o_resid + (size_t)x.bh * p.N * D + 64 * c), D * 2,
                               x.q_base + wq * 32, p.N);
      }
      if (p.lse != nullptr && r < p.N) p.lse[(size_t)x.bh * p.N + r] = (m + __log2f(l)) * 0.69314718055994531f;
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
}  // namespace

namespace {
template <int D>
cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                         const FwdParams& p, cudaStream_t s) {
  using L = FwdLayout<D>;
  const dim3 grid((unsigned)(p.n_pairs * p.BH));
  cudaError_t e = cudaFuncSetAttribute(fa_fwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  fa_fwd_sm100_kernel<D><<<grid, kThreads, L::SMEM_ALLOC, s>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

template <int D, bool F8>
cudaError_t launch_persist_t(dim3 grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to32, const CUtensorMap& tr32, const FwdParams& p, cudaStream_t s) {
  using L = FwdPLayout<D, F8>;
  cudaError_t e = cudaFuncSetAttribute(fa_fwd_persist_sm100_kernel<D, F8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  fa_fwd_persist_sm100_kernel<D, F8><<<grid, kThreads, L::SMEM_ALLOC, s>>>(tq, tk, tv, to32, tr32, p);
  return cudaGetLastError();
}

// V (bf16) -> fp16 copy with exponent 0, 8 elements per 16-byte access, on a fixed grid whose
// blocks leave their largest |v| (fp32 bits) in amax_part[block]; the fix-up below picks the
// copy's exponent.  Also zeroes the persistent kernel's work counter.
__global__ void __launch_bounds__(256) fa_fwd_v16_kernel(const uint4* __restrict__ v, uint4* __restrict__ v16,
                                                         long long n8, unsigned* counter, uint32_t* amax_part) {
  if (blockIdx.x == 0 && threadIdx.x == 0 && counter != nullptr) *counter = 0u;  // persistent kernel's work counter
  uint32_t am2 = 0u;  // packed bf16 maxima of |v|
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n8; e += (long long)gridDim.x * blockDim.x) {
    uint4 u = v[e];
    uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      am2 = amax_bf16x2_step(am2, w[i]);
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      w[i] = pack_f16(f.x, f.y);
    }
    v16[e] = u;
  }
  __shared__ uint32_t red[8];
  uint32_t am = __reduce_max_sync(0xffffffffu, amax_bf16x2_bits(am2));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = am;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) am = max(am, red[w]);
    amax_part[blockIdx.x] = am;
  }
}

// Fix-up of the V copy: every block reduces the n_part block maxima to V's largest |v| and
// derives the copy's exponent e (copy_exponent: 0 while it lies in [2^-4, 2^15], else the
// exponent that brings it into [4, 8)); block 0 records e in *v_exp (the attention kernel
// divides O by 2^e) and a non-finite V as kDevRange.  With e != 0 the blocks re-convert V as
// V 2^e.
__global__ void __launch_bounds__(256) fa_fwd_v16_fixup_kernel(const uint4* __restrict__ v, uint4* __restrict__ v16,
                                                               long long n8, const uint32_t* amax_part, int n_part,
                                                               int* v_exp, int* err) {
  __shared__ uint32_t red[8];
  __shared__ int e_s;
  uint32_t am = 0u;
  for (int i = threadIdx.x; i < n_part; i += blockDim.x) am = max(am, amax_part[i]);
  am = __reduce_max_sync(0xffffffffu, am);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = am;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) am = max(am, red[w]);
    e_s = copy_exponent(am, kCopyLoLog2, kCopyHiLog2);
    if (blockIdx.x == 0) {
      *v_exp = e_s;
      if (am >= kBitsInf) atomicExch(err, kDevRange);
    }
  }
  __syncthreads();
  const int e = e_s;
  if (e == 0) return;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    uint4 u = v[i];
    uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
      w[k] = pack_f16(ldexpf(f.x, e), ldexpf(f.y, e));
    }
    v16[i] = u;
  }
}
}  // namespace

cudaError_t launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const FwdParams& p, int d, cudaStream_t s) {
  return d == 128 ? launch_fwd_t<128>(tq, tk, tv, to, p, s) : launch_fwd_t<64>(tq, tk, tv, to, p, s);
}

cudaError_t launch_fwd_persist_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                     const CUtensorMap& to32, const CUtensorMap& tr32, const FwdParams& p, int d,
                                     cudaStream_t s) {
  const long long units = (long long)p.n_pairs * p.BH;
  const dim3 grid((unsigned)(units < p.num_sms ? units : p.num_sms));
  return d == 128 ? launch_persist_t<128, false>(grid, tq, tk, tv, to32, tr32, p, s)
                  : launch_persist_t<64, false>(grid, tq, tk, tv, to32, tr32, p, s);
}

cudaError_t launch_fwd_persist_fp8_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                         const CUtensorMap& to32, const FwdParams& p, int d, cudaStream_t s) {
  const long long units = (long long)p.n_pairs * p.BH;
  const dim3 grid((unsigned)(units < p.num_sms ? units : p.num_sms));
  return d == 128 ? launch_persist_t<128, true>(grid, tq, tk, tv, to32, to32, p, s)
                  : launch_persist_t<64, true>(grid, tq, tk, tv, to32, to32, p, s);
}

cudaError_t launch_fwd_v16(const void* v, void* v16, long long elems, unsigned* counter, uint32_t* amax_part,
                           int* v_exp, int* err, cudaStream_t s) {
  const long long n8 = elems / 8;  // d is a multiple of 8
  long long blocks = (n8 + 255) / 256;
  if (blocks > kVPassBlocks) blocks = kVPassBlocks;
  fa_fwd_v16_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(v), static_cast<uint4*>(v16), n8,
                                                     counter, amax_part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fa_fwd_v16_fixup_kernel<<<kFixupBlocks, 256, 0, s>>>(static_cast<const uint4*>(v), static_cast<uint4*>(v16), n8,
                                                       amax_part, (int)blocks, v_exp, err);
  return cudaGetLastError();
}

cudaError_t launch_fwd_d256_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                  const FwdParams& p, cudaStream_t s) {
  const long long units = (long long)((p.N + 127) / 128) * p.BH;
  const dim3 grid((unsigned)(units < p.num_sms ? units : p.num_sms));
  cudaError_t e = cudaFuncSetAttribute(fa_fwd_d256_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FwdWLayout::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  fa_fwd_d256_sm100_kernel<<<grid, kThreads, FwdWLayout::SMEM_ALLOC, s>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace fa
