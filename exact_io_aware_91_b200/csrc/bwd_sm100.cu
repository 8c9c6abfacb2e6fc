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
// Two kernels, each one CTA per tile, each with
//   warp 0: TMA producer, warp 1: tcgen05.mma issuer, warps 4-7 / 8-11: two
//   compute warpgroups that take alternate tiles of the inner loop (one thread
//   per TMEM lane / tile row), with S and dP double-buffered in tensor memory so
//   the elementwise work on one tile overlaps the MMAs of the next.
//   * dK/dV kernel: 128 keys per CTA, K and V resident; 64-query tiles of Q and
//     dO stream through a ring.  S^T = K Q^T and dP^T = V dO^T land in TMEM;
//     P^T and dS^T are written back to TMEM as fp16 and consumed directly as the
//     A operand of dV += P^T dO and dK += dS^T Q.
//   * dQ kernel: 128 queries per CTA, Q and dO resident; 64-key tiles of K and V
//     stream through a ring.  S = Q K^T, dP = dO V^T, dS to TMEM, dQ += dS K.
// All products run in fp16 (exact copies of the bf16 inputs made by the
// preprocess) with fp32 accumulation; gradients are written in fp32.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kThreads = 384;
// registers per thread: 168 at launch (65536 / 384, rounded down to a multiple of 8);
// warpgroup 0 (TMA, MMA) drops to 64 and the two compute warpgroups rise to 216
constexpr uint32_t kRegsLaunch = 168, kRegsLow = 64, kRegsHigh = 216;
static_assert(kRegsLow + 2 * kRegsHigh <= 3 * kRegsLaunch, "register split exceeds the launch budget");

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
}

// SS product D (+)= A * B^T over K = Dh; A rows in `a_box`-byte boxes, B rows in
// `b_box`-byte boxes; the descriptors are prebuilt, each MMA adds a constant offset.
template <int Dh, uint32_t a_box, uint32_t b_box>
__device__ __forceinline__ void issue_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t issue) {
#pragma unroll
  for (int k = 0; k < Dh / 16; ++k)
    mma_ss(d_tmem, sdesc_add(a_desc, (k >> 2) * a_box + (k & 3) * 32), sdesc_add(b_desc, (k >> 2) * b_box + (k & 3) * 32),
           idesc, k > 0 ? 1u : 0u, issue);
}

// TS product D (+)= A[tmem] * B over K rows of B (MN-major descriptor prebuilt).
template <int K>
__device__ __forceinline__ void issue_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                         bool acc, uint32_t issue) {
#pragma unroll
  for (int k = 0; k < K / 16; ++k)
    mma_ts(d_tmem, a_tmem + k * 8, sdesc_add(b_desc, k * 2048), idesc, (acc || k > 0) ? 1u : 0u, issue);
}

// Write `ncols` fp32 columns of this thread's TMEM lane to global row `dst` (times `mult`).
template <int NC>
__device__ __forceinline__ void store_rows_f32(uint32_t t_row, float* dst, float mult) {
#pragma unroll 1
  for (int c = 0; c < NC / 32; ++c) {
    uint32_t u[32];
    tmem_ld32(t_row + 32 * c, u);
    tmem_wait_ld();
    if (dst != nullptr) {
      float4* out = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        out[i] = make_float4(__uint_as_float(u[4 * i]) * mult, __uint_as_float(u[4 * i + 1]) * mult,
                             __uint_as_float(u[4 * i + 2]) * mult, __uint_as_float(u[4 * i + 3]) * mult);
    }
  }
}

// ============================================================================ dK / dV
template <int D>
struct DkdvLayout {
  static constexpr int KCH = D / 64;
  static constexpr int BOX_KV = 128 * 128;  // 64 cols x 128 rows, fp16
  static constexpr int BOX_Q = 64 * 128;    // 64 cols x 64 rows
  static constexpr int TILE_KV = KCH * BOX_KV;
  static constexpr int TILE_Q = KCH * BOX_Q;
  static constexpr int STAGE = 2 * TILE_Q + 1024;  // Q, dO, lse2[64], delta[64] (padded to 1 KB)
  static constexpr int STAGES = (D == 128) ? 4 : 6;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE_KV;
  static constexpr int OFF_STAGE = 2 * TILE_KV;
  static constexpr int OFF_BAR = OFF_STAGE + STAGES * STAGE;
  static constexpr int BAR_KV = 0;
  static constexpr int BAR_Q_FULL = 1;
  static constexpr int BAR_Q_EMPTY = 1 + STAGES;
  static constexpr int BAR_SDP = 1 + 2 * STAGES;  // [2]
  static constexpr int BAR_DS = BAR_SDP + 2;      // [2]
  static constexpr int BAR_ACC = BAR_DS + 2;
  static constexpr int BAR_DONE = BAR_ACC + 1;
  static constexpr int NBAR = BAR_DONE + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NBAR * 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM_ALLOC = OFF_ABORT + 8 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_DV = 0, T_DK = D, T_BUF = 2 * D;  // buffer b at T_BUF + 128 b: S^T | dP^T
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                             const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             const BwdParams p) {
  using L = DkdvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // head-major order (CTAs running together share Q / dO in L2); within a head the
  // key tiles with the most work under the causal mask (small j) come first
  const int n_kt = (p.N + 127) / 128;
  const int bh = blockIdx.x / n_kt;
  const int j = blockIdx.x % n_kt;
  const int nq = (p.N + 63) / 64;
  const int i_start = p.causal ? 2 * j : 0;
  const int n_it = nq - i_start;  // >= 1

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::BAR_KV), 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::BAR_Q_FULL + s), 1);
      mbar_init(bar(L::BAR_Q_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::BAR_SDP + b), 1);
      mbar_init(bar(L::BAR_DS + b), 128);
    }
    mbar_init(bar(L::BAR_ACC), 1);
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
    regs_dec<kRegsLow>();
    {
      const uint32_t leader = elect_one();  // the lane that issues async instructions
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(bar(L::BAR_KV), 2 * L::TILE_KV, leader);
      for (int c = 0; c < L::KCH; ++c) {
        tma_load_3d(base + L::OFF_K + c * L::BOX_KV, &tm_k, c * 64, j * 128, bh, bar(L::BAR_KV), leader);
        tma_load_3d(base + L::OFF_V + c * L::BOX_KV, &tm_v, c * 64, j * 128, bh, bar(L::BAR_KV), leader);
      }
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int st = it % L::STAGES;
        if (!mbar_wait(bar(L::BAR_Q_EMPTY + st), ((it / L::STAGES) & 1) ^ 1u, wctx)) break;
        const int i = i_start + it;
        const uint32_t sb = base + L::OFF_STAGE + st * L::STAGE;
        const uint32_t fb = bar(L::BAR_Q_FULL + st);
        mbar_arrive_expect_tx(fb, 2 * L::TILE_Q + 512, leader);
        for (int c = 0; c < L::KCH; ++c) {
          tma_load_3d(sb + c * L::BOX_Q, &tm_q, c * 64, i * 64, bh, fb, leader);
          tma_load_3d(sb + L::TILE_Q + c * L::BOX_Q, &tm_do, c * 64, i * 64, bh, fb, leader);
        }
        const size_t roff = (size_t)bh * p.Np + (size_t)i * 64;
        bulk_load(sb + 2 * L::TILE_Q, p.lse2 + roff, 256, fb, leader);
        bulk_load(sb + 2 * L::TILE_Q + 256, p.delta + roff, 256, fb, leader);
        ++issued;
      }
      drain_wait(bar(L::BAR_KV), 0);
      const int first = issued > L::STAGES ? issued - L::STAGES : 0;
      for (int it = first; it < issued; ++it)
        drain_wait(bar(L::BAR_Q_FULL + (it % L::STAGES)), (it / L::STAGES) & 1);
    }
  } else if (warp == 1) {
    regs_dec<kRegsLow>();
    {
      const uint32_t leader = elect_one();  // the lane that issues async instructions
      constexpr uint32_t idesc_s = make_idesc(128, 64, false, false, false);  // M=128 keys, N=64 queries
      constexpr uint32_t idesc_g = make_idesc(128, D, false, false, true);    // N=D, B MN-major
      const uint64_t dK = make_sdesc_sw128(base + L::OFF_K, 16, 1024);
      const uint64_t dV = make_sdesc_sw128(base + L::OFF_V, 16, 1024);
      const uint64_t dStK = make_sdesc_sw128(base + L::OFF_STAGE, 16, 1024);        // Q / dO as K-major B
      const uint64_t dStMN = make_sdesc_sw128(base + L::OFF_STAGE, L::BOX_Q, 1024);  // Q / dO as MN-major B
      auto issue_sdp = [&](int it) {
        const uint32_t so = (it % L::STAGES) * L::STAGE;
        const uint32_t tb = tmem + L::T_BUF + 128 * (it & 1);
        issue_ss<D, L::BOX_KV, L::BOX_Q>(tb, dK, sdesc_add(dStK, so), idesc_s, leader);                     // S^T  = K Q^T
        issue_ss<D, L::BOX_KV, L::BOX_Q>(tb + 64, dV, sdesc_add(dStK, so + L::TILE_Q), idesc_s, leader);    // dP^T = V dO^T
        mma_commit(bar(L::BAR_SDP + (it & 1)), leader);
      };
      bool ok = mbar_wait(bar(L::BAR_KV), 0, wctx);
      if (ok) ok = mbar_wait(bar(L::BAR_Q_FULL + 0), 0, wctx);
      if (ok) {
        tc_fence_after();
        issue_sdp(0);
      }
      for (int it = 0; it < n_it && ok; ++it) {
        if (it + 1 < n_it) {
          const int nx = it + 1;
          if (!(ok = mbar_wait(bar(L::BAR_Q_FULL + (nx % L::STAGES)), (nx / L::STAGES) & 1, wctx))) break;
          tc_fence_after();
          issue_sdp(nx);
        }
        const int b = it & 1;
        if (!(ok = mbar_wait(bar(L::BAR_DS + b), (it >> 1) & 1, wctx))) break;
        tc_fence_after();
        const uint32_t so = (it % L::STAGES) * L::STAGE;
        const uint32_t tb = tmem + L::T_BUF + 128 * b;
        issue_ts<64>(tmem + L::T_DV, tb, sdesc_add(dStMN, so + L::TILE_Q), idesc_g, it > 0, leader);  // dV += P^T dO
        issue_ts<64>(tmem + L::T_DK, tb + 64, sdesc_add(dStMN, so), idesc_g, it > 0, leader);         // dK += dS^T Q
        mma_commit(bar(L::BAR_Q_EMPTY + (it % L::STAGES)), leader);
      }
      if (ok) mma_commit(bar(L::BAR_ACC), leader);
      mma_commit(bar(L::BAR_DONE), leader);
      drain_wait(bar(L::BAR_DONE), 0);
    }
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle
  } else {
    regs_inc<kRegsHigh>();
    const int w = (warp - 4) >> 2;   // warpgroup: takes tiles it = w, w + 2, ...
    const int wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;  // key row inside the tile
    const int key = j * 128 + row;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tb = tmem + lane_off + L::T_BUF + 128 * w;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int it = w; it < n_it; it += 2) {
      if (!(ok = mbar_wait(bar(L::BAR_SDP + w), (it >> 1) & 1, wctx))) break;
      tc_fence_after();
      const int i = i_start + it;
      const uint8_t* sgen = gbase + L::OFF_STAGE + (it % L::STAGES) * L::STAGE;
      const float* lse2 = reinterpret_cast<const float*>(sgen + 2 * L::TILE_Q);
      const float* delta = lse2 + 64;
      float s[64], dp[64];
      {
        uint32_t u[32];
        tmem_ld32(tb, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(u[c]);
        tmem_ld32(tb + 32, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = __uint_as_float(u[c]);
        tmem_ld32(tb + 64, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[c] = __uint_as_float(u[c]);
        tmem_ld32(tb + 96, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[32 + c] = __uint_as_float(u[c]);
        tmem_wait_ld();
      }
      const bool need_mask = p.causal && (i * 64 < j * 128 + 127);
      const uint64_t sl2x2 = f2pack(sl2, sl2);
#pragma unroll
      for (int g = 0; g < 64; g += 16) {  // 16 query columns at a time: 8 packed words of P^T and dS^T
        uint32_t pk_p[8], pk_ds[8];
#pragma unroll
        for (int c = g; c < g + 16; c += 4) {
          // per-query LSE and D are broadcast reads of the stage's vectors (16 bytes at a time)
          const float4 L4 = *reinterpret_cast<const float4*>(lse2 + c);
          const float4 D4 = *reinterpret_cast<const float4*>(delta + c);
          float t0, t1, t2, t3;
          f2unpack(ffma2(f2pack(s[c], s[c + 1]), sl2x2, f2pack(-L4.x, -L4.y)), t0, t1);
          f2unpack(ffma2(f2pack(s[c + 2], s[c + 3]), sl2x2, f2pack(-L4.z, -L4.w)), t2, t3);
          float p0 = ex2_approx(t0), p1 = ex2_approx(t1), p2 = ex2_approx(t2), p3 = ex2_approx(t3);
          if (need_mask) {
            if (i * 64 + c < key) p0 = 0.f;
            if (i * 64 + c + 1 < key) p1 = 0.f;
            if (i * 64 + c + 2 < key) p2 = 0.f;
            if (i * 64 + c + 3 < key) p3 = 0.f;
          }
          float d0, d1, d2, d3;
          f2unpack(fmul2(f2pack(p0, p1), fsub2(f2pack(dp[c], dp[c + 1]), f2pack(D4.x, D4.y))), d0, d1);
          f2unpack(fmul2(f2pack(p2, p3), fsub2(f2pack(dp[c + 2], dp[c + 3]), f2pack(D4.z, D4.w))), d2, d3);
          pk_p[(c - g) / 2] = pack_f16(p0, p1);
          pk_p[(c - g) / 2 + 1] = pack_f16(p2, p3);
          pk_ds[(c - g) / 2] = pack_f16(d0, d1);
          pk_ds[(c - g) / 2 + 1] = pack_f16(d2, d3);
        }
        tmem_st8(tb + g / 2, pk_p);
        tmem_st8(tb + 64 + g / 2, pk_ds);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::BAR_DS + w));
    }
    if (ok) ok = mbar_wait(bar(L::BAR_ACC), 0, wctx);
    if (ok) {
      tc_fence_after();
      // warpgroup 0 writes dV, warpgroup 1 writes scale * dK (rows past N are padding)
      float* dst = (key < p.N) ? ((w == 0 ? p.dv : p.dk) + ((size_t)bh * p.N + key) * D) : nullptr;
      store_rows_f32<D>(tmem + lane_off + (w == 0 ? L::T_DV : L::T_DK), dst, w == 0 ? 1.0f : p.scale);
    }
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
  static constexpr int BOX_Q = 128 * 128;   // 64 cols x 128 rows
  static constexpr int BOX_K = 64 * 128;    // 64 cols x 64 rows
  static constexpr int TILE_Q = KCH * BOX_Q;
  static constexpr int TILE_K = KCH * BOX_K;
  static constexpr int STAGE = 2 * TILE_K;  // K_j, V_j
  static constexpr int STAGES = (D == 128) ? 4 : 6;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE_Q;
  static constexpr int OFF_STAGE = 2 * TILE_Q;
  static constexpr int OFF_BAR = OFF_STAGE + STAGES * STAGE;
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_KV_FULL = 1;
  static constexpr int BAR_KV_EMPTY = 1 + STAGES;
  static constexpr int BAR_SDP = 1 + 2 * STAGES;
  static constexpr int BAR_DS = BAR_SDP + 2;
  static constexpr int BAR_ACC = BAR_DS + 2;
  static constexpr int BAR_DONE = BAR_ACC + 1;
  static constexpr int NBAR = BAR_DONE + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NBAR * 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM_ALLOC = OFF_ABORT + 8 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_DQ = 0, T_BUF = D;  // buffer b at T_BUF + 128 b: S | dP
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const BwdParams p) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_ABORT);
  const WaitCtx wctx{abort_flag, p.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int nq = (p.N + 127) / 128;
  const int nk = (p.N + 63) / 64;
  // head-major order (CTAs running together share K / V in L2); within a head the
  // query tiles with the most work under the causal mask come first
  const int bh = blockIdx.x / nq;
  const int qt = p.causal ? (nq - 1 - (int)(blockIdx.x % nq)) : (int)(blockIdx.x % nq);
  const int n_it = p.causal ? min(nk, (qt * 128 + 127) / 64 + 1) : nk;  // key tiles 0..n_it-1

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::BAR_Q), 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::BAR_KV_FULL + s), 1);
      mbar_init(bar(L::BAR_KV_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::BAR_SDP + b), 1);
      mbar_init(bar(L::BAR_DS + b), 128);
    }
    mbar_init(bar(L::BAR_ACC), 1);
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
    regs_dec<kRegsLow>();
    {
      const uint32_t leader = elect_one();  // the lane that issues async instructions
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(bar(L::BAR_Q), 2 * L::TILE_Q, leader);
      for (int c = 0; c < L::KCH; ++c) {
        tma_load_3d(base + L::OFF_Q + c * L::BOX_Q, &tm_q, c * 64, qt * 128, bh, bar(L::BAR_Q), leader);
        tma_load_3d(base + L::OFF_DO + c * L::BOX_Q, &tm_do, c * 64, qt * 128, bh, bar(L::BAR_Q), leader);
      }
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int st = it % L::STAGES;
        if (!mbar_wait(bar(L::BAR_KV_EMPTY + st), ((it / L::STAGES) & 1) ^ 1u, wctx)) break;
        const uint32_t sb = base + L::OFF_STAGE + st * L::STAGE;
        const uint32_t fb = bar(L::BAR_KV_FULL + st);
        mbar_arrive_expect_tx(fb, 2 * L::TILE_K, leader);
        for (int c = 0; c < L::KCH; ++c) {
          tma_load_3d(sb + c * L::BOX_K, &tm_k, c * 64, it * 64, bh, fb, leader);
          tma_load_3d(sb + L::TILE_K + c * L::BOX_K, &tm_v, c * 64, it * 64, bh, fb, leader);
        }
        ++issued;
      }
      drain_wait(bar(L::BAR_Q), 0);
      const int first = issued > L::STAGES ? issued - L::STAGES : 0;
      for (int it = first; it < issued; ++it)
        drain_wait(bar(L::BAR_KV_FULL + (it % L::STAGES)), (it / L::STAGES) & 1);
    }
  } else if (warp == 1) {
    regs_dec<kRegsLow>();
    {
      const uint32_t leader = elect_one();  // the lane that issues async instructions
      constexpr uint32_t idesc_s = make_idesc(128, 64, false, false, false);  // M=128 queries, N=64 keys
      constexpr uint32_t idesc_g = make_idesc(128, D, false, false, true);
      const uint64_t dQd = make_sdesc_sw128(base + L::OFF_Q, 16, 1024);
      const uint64_t dDO = make_sdesc_sw128(base + L::OFF_DO, 16, 1024);
      const uint64_t dStK = make_sdesc_sw128(base + L::OFF_STAGE, 16, 1024);        // K / V as K-major B
      const uint64_t dStMN = make_sdesc_sw128(base + L::OFF_STAGE, L::BOX_K, 1024);  // K as MN-major B
      auto issue_sdp = [&](int it) {
        const uint32_t so = (it % L::STAGES) * L::STAGE;
        const uint32_t tb = tmem + L::T_BUF + 128 * (it & 1);
        issue_ss<D, L::BOX_Q, L::BOX_K>(tb, dQd, sdesc_add(dStK, so), idesc_s, leader);                    // S  = Q K^T
        issue_ss<D, L::BOX_Q, L::BOX_K>(tb + 64, dDO, sdesc_add(dStK, so + L::TILE_K), idesc_s, leader);   // dP = dO V^T
        mma_commit(bar(L::BAR_SDP + (it & 1)), leader);
      };
      bool ok = mbar_wait(bar(L::BAR_Q), 0, wctx);
      if (ok) ok = mbar_wait(bar(L::BAR_KV_FULL + 0), 0, wctx);
      if (ok) {
        tc_fence_after();
        issue_sdp(0);
      }
      for (int it = 0; it < n_it && ok; ++it) {
        if (it + 1 < n_it) {
          const int nx = it + 1;
          if (!(ok = mbar_wait(bar(L::BAR_KV_FULL + (nx % L::STAGES)), (nx / L::STAGES) & 1, wctx))) break;
          tc_fence_after();
          issue_sdp(nx);
        }
        const int b = it & 1;
        if (!(ok = mbar_wait(bar(L::BAR_DS + b), (it >> 1) & 1, wctx))) break;
        tc_fence_after();
        const uint32_t tb = tmem + L::T_BUF + 128 * b;
        issue_ts<64>(tmem + L::T_DQ, tb, sdesc_add(dStMN, (it % L::STAGES) * L::STAGE), idesc_g, it > 0, leader);  // dQ += dS K
        mma_commit(bar(L::BAR_KV_EMPTY + (it % L::STAGES)), leader);
      }
      if (ok) mma_commit(bar(L::BAR_ACC), leader);
      mma_commit(bar(L::BAR_DONE), leader);
      drain_wait(bar(L::BAR_DONE), 0);
    }
  } else if (warp < 4) {
    regs_dec<kRegsLow>();  // warps 2-3: idle
  } else {
    regs_inc<kRegsHigh>();
    const int w = (warp - 4) >> 2;
    const int wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;
    const int r = qt * 128 + row;  // query index
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tb = tmem + lane_off + L::T_BUF + 128 * w;
    const float sl2 = p.scale_log2;
    const size_t prow = (size_t)bh * p.Np + r;  // r < Np always (Np is a multiple of 128)
    const float lse2 = p.lse2[prow];
    const float delta = p.delta[prow];
    const int lim = p.causal ? min(r, p.N - 1) : (p.N - 1);  // last visible key
    bool ok = true;
    for (int it = w; it < n_it; it += 2) {
      if (!(ok = mbar_wait(bar(L::BAR_SDP + w), (it >> 1) & 1, wctx))) break;
      tc_fence_after();
      float s[64], dp[64];
      {
        uint32_t u[32];
        tmem_ld32(tb, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(u[c]);
        tmem_ld32(tb + 32, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = __uint_as_float(u[c]);
        tmem_ld32(tb + 64, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[c] = __uint_as_float(u[c]);
        tmem_ld32(tb + 96, u);
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[32 + c] = __uint_as_float(u[c]);
        tmem_wait_ld();
      }
      const int kb = it * 64;
      const bool need_mask = (p.causal && kb + 63 > qt * 128) || (kb + 64 > p.N);
      const uint64_t sl2x2 = f2pack(sl2, sl2), nl2 = f2pack(-lse2, -lse2), dd = f2pack(delta, delta);
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float t0, t1;
        f2unpack(ffma2(f2pack(s[2 * c], s[2 * c + 1]), sl2x2, nl2), t0, t1);
        float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
        if (need_mask) {
          if (kb + 2 * c > lim) p0 = 0.f;
          if (kb + 2 * c + 1 > lim) p1 = 0.f;
        }
        float d0, d1;
        f2unpack(fmul2(f2pack(p0, p1), fsub2(f2pack(dp[2 * c], dp[2 * c + 1]), dd)), d0, d1);
        pk[c] = pack_f16(d0, d1);
      }
      tmem_st32(tb, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::BAR_DS + w));
    }
    if (ok) ok = mbar_wait(bar(L::BAR_ACC), 0, wctx);
    if (ok) {
      tc_fence_after();
      // each warpgroup writes half of the columns of scale * dQ
      float* dst = (r < p.N) ? (p.dq + ((size_t)bh * p.N + r) * D + w * (D / 2)) : nullptr;
      store_rows_f32<D / 2>(tmem + lane_off + L::T_DQ + w * (D / 2), dst, p.scale);
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

cudaError_t launch_bwd_dkdv_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const BwdParams& p, int d, cudaStream_t s) {
  const dim3 grid((unsigned)(((p.N + 127) / 128) * p.BH));
  if (d == 128)
    return launch_one<DkdvLayout<128>>(fa_bwd_dkdv_sm100_kernel<128>, grid, tq, tdo, tk, tv, p, s);
  return launch_one<DkdvLayout<64>>(fa_bwd_dkdv_sm100_kernel<64>, grid, tq, tdo, tk, tv, p, s);
}

cudaError_t launch_bwd_dq_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                const CUtensorMap& tv, const BwdParams& p, int d, cudaStream_t s) {
  const dim3 grid((unsigned)(((p.N + 127) / 128) * p.BH));
  if (d == 128) return launch_one<DqLayout<128>>(fa_bwd_dq_sm100_kernel<128>, grid, tq, tdo, tk, tv, p, s);
  return launch_one<DqLayout<64>>(fa_bwd_dq_sm100_kernel<64>, grid, tq, tdo, tk, tv, p, s);
}

}  // namespace fa
