// Backward preprocess, one streaming pass over the rows of O and dO:
//   D_i    = sum_c dO[i,c] * O[i,c]        (equals sum_j P_ij dP_ij; derived)
//            with O = O_bf16 + residual when the forward's residual is given,
//            i.e. the forward's fp32 O, so that D does not carry O's bf16 rounding
//   lse2_i = LSE_i * log2(e)               (so the kernels form P = 2^(s*scale*log2e - lse2))
//   counters         = 0: the work counters of the persistent backward kernels that follow
//   q16, k16, v16, do16 = fp16 copies of the bf16 inputs (k16 / v16 for the first BH_kv
//   heads only: with grouped-query attention K and V have fewer heads than Q)
// Rows N..Np-1 of D / lse2 are padding for the 64/128-row tiles: D = 0 and
// lse2 = +inf, which makes every probability of a padded query exactly 0.
//
// The backward runs its tensor-core products in fp16 so that the probabilities P and the
// score gradients dS, which feed tensor-core products, are rounded to 11 significant bits
// instead of bf16's 8.  fp16 covers |x| < 65504 (and |x| >= 2^-14 at full precision), bf16
// nearly the fp32 range, so each copy is x * 2^e with one exponent e per tensor (see
// copy_exponent): the preprocess converts with e = 0 and leaves per-block maxima of |x|; the
// fix-up kernel reduces them, keeps e = 0 while every tensor's largest magnitude lies in
// [2^-4, 2^15] and 2 d max|dO| max|V| <= 2^15 (the bound on the fp16 dS, below), and
// otherwise re-converts the tensors concerned with the exponent that brings their largest
// magnitude into [4, 8) and scales D into the units of the dO and V copies.  The dK/dV and
// dQ kernels read the exponents and undo them in the softmax scale and their epilogues.
//
// Bound on dS = P (dP - D): 0 <= P <= 1, |dP_ij| <= sum_c |dO_ic| |V_jc| <= d max|dO| max|V|,
// and D_i = sum_j P_ij dP_ij is a convex combination of the same dP, so
// |dS| <= 2 d max|dO| max|V|.
//
// Non-finite inputs (a largest magnitude of inf or NaN) and a non-finite D are reported as
// kDevRange in the device error word.
//
// fa_bwd_ws reuses the fp16 V copy that fa_fwd_ws left in its workspace (the same V, the
// same exponent rule for V on its own): the preprocess then reads no V, the fix-up takes
// max |V| from the forward's V-pass maxima, and V is converted again (into the forward's
// copy) only when the dS bound asks for another exponent than the copy holds.
//
// Each row is read with 16-byte loads by d/8 consecutive lanes; the grid is fixed
// (kPreBlocks blocks or fewer) and its warps stride over the rows.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace fa {
namespace {

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 in, float (&f)[8]) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&in);
  uint4 out;
  __half2* h = reinterpret_cast<__half2*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(b[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
    h[i] = __floats2half2_rn(x.x, x.y);
  }
  return out;
}

// The same conversion of x * 2^e (exact power-of-two scaling before the rounding to fp16).
__device__ __forceinline__ uint4 bf16x8_to_f16x8_scaled(uint4 in, int e) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&in);
  uint4 out;
  __half2* h = reinterpret_cast<__half2*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(b[i]);
    h[i] = __floats2half2_rn(ldexpf(x.x, e), ldexpf(x.y, e));
  }
  return out;
}

// running packed maxima of |x| (see amax_bf16x2_step)
__device__ __forceinline__ uint32_t amax_bf16x8(uint32_t acc2, uint4 u) {
  acc2 = amax_bf16x2_step(acc2, u.x);
  acc2 = amax_bf16x2_step(acc2, u.y);
  acc2 = amax_bf16x2_step(acc2, u.z);
  return amax_bf16x2_step(acc2, u.w);
}

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdPreParams p) {
  constexpr int LPR = D / 8;          // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp and iteration
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int sub = lane % LPR;
  // 64-bit: B * H * Np rows reach 2^31 at the largest problems (2^24 heads)
  const long long total = (long long)p.BH * p.Np;
  const long long warp_global = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);

  if (blockIdx.x == 0 && threadIdx.x < kNumCounters) p.counters[threadIdx.x] = 0u;

  uint32_t am_q = 0u, am_k = 0u, am_v = 0u, am_do = 0u;  // max |x| seen, as packed bf16 pairs
  bool bad_d = false;
  for (long long base = warp_global * RPW; base < total; base += warps * RPW) {  // warp-uniform
    const long long row_global = base + lane / LPR;  // over BH * Np
    const bool valid_slot = row_global < total;
    const int bh = valid_slot ? (int)(row_global / p.Np) : 0;
    const int i = valid_slot ? (int)(row_global % p.Np) : 0;
    const bool real = valid_slot && i < p.N;
    float dsum = 0.f;
    if (real) {
      const size_t off = ((size_t)bh * p.N + i) * D + (size_t)sub * 8;  // element offset
      const uint4 vq = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + off);
      const uint4 vo = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o) + off);
      const uint4 vd = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dout) + off);
      float fq[8], fk[8], fv[8], fo[8], fd[8];
      *reinterpret_cast<uint4*>(static_cast<__half*>(p.q16) + off) = bf16x8_to_f16x8(vq, fq);
      *reinterpret_cast<uint4*>(static_cast<__half*>(p.do16) + off) = bf16x8_to_f16x8(vd, fd);
      am_q = amax_bf16x8(am_q, vq);
      am_do = amax_bf16x8(am_do, vd);
      if (bh < p.BH_kv) {  // key/value rows share the (head, row) index space of the first BH_kv heads
        const uint4 vk = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.k) + off);
        *reinterpret_cast<uint4*>(static_cast<__half*>(p.k16) + off) = bf16x8_to_f16x8(vk, fk);
        am_k = amax_bf16x8(am_k, vk);
        if (p.v_amax_fwd == nullptr) {  // else the forward's V copy is reused
          const uint4 vv = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.v) + off);
          *reinterpret_cast<uint4*>(static_cast<__half*>(p.v16) + off) = bf16x8_to_f16x8(vv, fv);
          am_v = amax_bf16x8(am_v, vv);
        }
      }
      bf16x8_to_f16x8(vo, fo);
      if (p.o_resid != nullptr) {
        float fr[8];
        const uint4 vr = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o_resid) + off);
        bf16x8_to_f16x8(vr, fr);
#pragma unroll
        for (int c = 0; c < 8; ++c) fo[c] += fr[c];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) dsum = fmaf(fd[c], fo[c], dsum);
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    if (valid_slot && sub == 0) {
      const size_t r = (size_t)bh * p.Np + i;
      if (real) {
        p.delta[r] = dsum;
        p.lse2[r] = p.lse[(size_t)bh * p.N + i] * 1.4426950408889634f;
        bad_d |= !(fabsf(dsum) < INFINITY);
      } else {
        p.delta[r] = 0.f;
        p.lse2[r] = INFINITY;
      }
    }
  }
  if (bad_d) atomicExch(p.err, kDevRange);
  // per-block maxima of the four tensors, as fp32 bits
  __shared__ uint32_t red[8][4];
  am_q = __reduce_max_sync(0xffffffffu, amax_bf16x2_bits(am_q));
  am_k = __reduce_max_sync(0xffffffffu, amax_bf16x2_bits(am_k));
  am_v = __reduce_max_sync(0xffffffffu, amax_bf16x2_bits(am_v));
  am_do = __reduce_max_sync(0xffffffffu, amax_bf16x2_bits(am_do));
  if (lane == 0) {
    red[warp][0] = am_q;
    red[warp][1] = am_k;
    red[warp][2] = am_v;
    red[warp][3] = am_do;
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    uint32_t m = 0u;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = max(m, red[w][threadIdx.x]);
    p.amax_part[threadIdx.x * kPreBlocks + blockIdx.x] = m;
  }
}

// Fix-up: every block reduces the per-block maxima (n_part of them per tensor) and derives
// the same exponents; block 0 records them.  When one is not 0 the blocks re-convert that
// tensor from its bf16 original, and D is scaled by 2^(e_V + e_dO).
__global__ void __launch_bounds__(256) fa_bwd_fixup_kernel(const BwdPreParams p, int n_part) {
  __shared__ uint32_t red[8][4];
  __shared__ int ex[4];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ int ev_copy;  // exponent the V copy holds now (0, or the forward's when it is reused)
  const bool reuse_v = p.v_amax_fwd != nullptr;
  uint32_t m[4] = {0u, 0u, 0u, 0u};
  for (int i = threadIdx.x; i < n_part; i += blockDim.x)
#pragma unroll
    for (int t = 0; t < 4; ++t) m[t] = max(m[t], p.amax_part[t * kPreBlocks + i]);
  if (reuse_v)  // max |V| from the forward's V pass (the preprocess did not read V)
    for (int i = threadIdx.x; i < p.v_n_part_fwd; i += blockDim.x) m[kExpV] = max(m[kExpV], p.v_amax_fwd[i]);
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    m[t] = __reduce_max_sync(0xffffffffu, m[t]);
    if (lane == 0) red[warp][t] = m[t];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a[4] = {0u, 0u, 0u, 0u};
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w)
      for (int t = 0; t < 4; ++t) a[t] = max(a[t], red[w][t]);
    int e[4];
    for (int t = 0; t < 4; ++t) e[t] = copy_exponent(a[t], kCopyLoLog2, kCopyHiLog2);
    // the fp16 dS is in the units of the dO and V copies: keep its bound within 2^15
    const float bound = 2.0f * (float)p.d * ldexpf(__uint_as_float(a[kExpV]), e[kExpV]) *
                        ldexpf(__uint_as_float(a[kExpDO]), e[kExpDO]);
    if (!(bound <= kDsBound) && a[kExpV] < kBitsInf && a[kExpDO] < kBitsInf) {
      e[kExpV] = target_exponent(a[kExpV]);
      e[kExpDO] = target_exponent(a[kExpDO]);
    }
    for (int t = 0; t < 4; ++t) ex[t] = e[t];
    ev_copy = reuse_v ? *p.v_exp_fwd : 0;
    if (blockIdx.x == 0) {
      for (int t = 0; t < 4; ++t) p.exps[t] = e[t];
      if (a[0] >= kBitsInf || a[1] >= kBitsInf || a[2] >= kBitsInf || a[3] >= kBitsInf) atomicExch(p.err, kDevRange);
    }
  }
  __syncthreads();
  const int eq = ex[kExpQ], ek = ex[kExpK], ev = ex[kExpV], edo = ex[kExpDO];
  const bool redo_v = ev != ev_copy;  // the V copy holds 2^ev_copy V: convert again with 2^ev
  if ((eq | ek | edo) == 0 && !redo_v && ev == 0) return;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long first = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long n8 = (long long)p.BH * p.N * p.d / 8, n8kv = (long long)p.BH_kv * p.N * p.d / 8;
  auto reconvert = [&](const void* src, void* dst, long long n, int e) {
    const uint4* s = static_cast<const uint4*>(src);
    uint4* t = static_cast<uint4*>(dst);
    for (long long i = first; i < n; i += stride) t[i] = bf16x8_to_f16x8_scaled(s[i], e);
  };
  if (eq != 0) reconvert(p.q, p.q16, n8, eq);
  if (ek != 0) reconvert(p.k, p.k16, n8kv, ek);
  if (redo_v) reconvert(p.v, p.v16, n8kv, ev);
  if (edo != 0) reconvert(p.dout, p.do16, n8, edo);
  if (ev + edo != 0) {
    const long long rows = (long long)p.BH * p.Np;
    for (long long i = first; i < rows; i += stride) p.delta[i] = ldexpf(p.delta[i], ev + edo);
  }
}

// dK, dV of grouped-query attention when one key/value head's query heads were split
// over several CTAs: out[e] = sum over splits of part[split][e], in a fixed order.
__global__ void __launch_bounds__(256) fa_bwd_kv_reduce_kernel(const float4* __restrict__ dk_part,
                                                              const float4* __restrict__ dv_part,
                                                              float4* __restrict__ dk, float4* __restrict__ dv,
                                                              long long n4, int splits) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (long long)gridDim.x * blockDim.x) {
    float4 a = dk_part[e], b = dv_part[e];
    for (int s = 1; s < splits; ++s) {
      const float4 x = dk_part[(long long)s * n4 + e], y = dv_part[(long long)s * n4 + e];
      a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
      b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
    }
    dk[e] = a;
    dv[e] = b;
  }
}

}  // namespace

cudaError_t launch_bwd_kv_reduce(const float* dk_part, const float* dv_part, float* dk, float* dv, long long elems,
                                 int splits, cudaStream_t s) {
  const long long n4 = elems / 4;  // d is a multiple of 4
  long long blocks = (n4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  fa_bwd_kv_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(dk_part),
                                                           reinterpret_cast<const float4*>(dv_part),
                                                           reinterpret_cast<float4*>(dk),
                                                           reinterpret_cast<float4*>(dv), n4, splits);
  return cudaGetLastError();
}

cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t s) {
  const long long rows = (long long)p.BH * p.Np;
  const int rpw = 32 / (p.d / 8);
  const long long warps = (rows + rpw - 1) / rpw;
  long long blocks = (warps + 7) / 8;
  if (blocks > kPreBlocks) blocks = kPreBlocks;
  if (p.d == 256)
    fa_bwd_pre_kernel<256><<<(unsigned)blocks, 256, 0, s>>>(p);
  else if (p.d == 128)
    fa_bwd_pre_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(p);
  else
    fa_bwd_pre_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fa_bwd_fixup_kernel<<<kFixupBlocks, 256, 0, s>>>(p, (int)blocks);
  return cudaGetLastError();
}

}  // namespace fa
