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
// The fp16 copies are exact for |x| in [2^-14, 65504] (bf16 has 8 significant
// bits, fp16 11); the backward runs its tensor-core products in fp16 so that the
// probabilities P and the score gradients dS, which feed tensor-core products,
// are rounded to 11 significant bits instead of bf16's 8.
//
// Each row is read with 16-byte loads by d/8 consecutive lanes.
#include "fa_internal.h"

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

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdPreParams p) {
  constexpr int LPR = D / 8;          // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp
  const int lane = threadIdx.x & 31;
  // 64-bit: B * H * Np rows reach 2^31 at the largest problems (2^24 heads)
  const long long warp_global = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long row_global = warp_global * RPW + lane / LPR;  // over BH * Np
  const int sub = lane % LPR;
  const long long total = (long long)p.BH * p.Np;
  const bool valid_slot = row_global < total;
  const int bh = valid_slot ? (int)(row_global / p.Np) : 0;
  const int i = valid_slot ? (int)(row_global % p.Np) : 0;
  const bool real = valid_slot && i < p.N;

  if (blockIdx.x == 0 && threadIdx.x < kNumCounters) p.counters[threadIdx.x] = 0u;

  float dsum = 0.f;
  if (real) {
    const size_t off = ((size_t)bh * p.N + i) * D + (size_t)sub * 8;  // element offset
    const uint4 vq = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + off);
    const uint4 vo = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o) + off);
    const uint4 vd = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dout) + off);
    float fq[8], fk[8], fv[8], fo[8], fd[8];
    *reinterpret_cast<uint4*>(static_cast<__half*>(p.q16) + off) = bf16x8_to_f16x8(vq, fq);
    *reinterpret_cast<uint4*>(static_cast<__half*>(p.do16) + off) = bf16x8_to_f16x8(vd, fd);
    if (bh < p.BH_kv) {  // key/value rows share the (head, row) index space of the first BH_kv heads
      const uint4 vk = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.k) + off);
      const uint4 vv = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.v) + off);
      *reinterpret_cast<uint4*>(static_cast<__half*>(p.k16) + off) = bf16x8_to_f16x8(vk, fk);
      *reinterpret_cast<uint4*>(static_cast<__half*>(p.v16) + off) = bf16x8_to_f16x8(vv, fv);
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
    } else {
      p.delta[r] = 0.f;
      p.lse2[r] = INFINITY;
    }
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
  const long long blocks = (warps + 7) / 8;
  if (p.d == 128)
    fa_bwd_pre_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(p);
  else
    fa_bwd_pre_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace fa
