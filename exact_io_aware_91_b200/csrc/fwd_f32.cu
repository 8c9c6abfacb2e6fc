// fp32 forward (CUDA cores, no tensor cores) for fp32 inputs, so that a small
// fp32 problem is checked without rounding its inputs to bf16.  Same method as
// the sm_100a kernel -- key blocks streamed through shared memory with an online
// softmax (running max and exp-sum, rescaled partial output; "FlashAttention
// (EL)", section "Online computation of Softmax") -- at a scale where speed does
// not matter.
//
// One CTA = 16 query rows of one (b, h), two rows per warp; a key block of 32
// keys is staged in shared memory; lane c of the warp scores key c of the block.
#include <cmath>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kRows = 16;      // query rows per CTA
constexpr int kKeys = 32;      // keys per block
constexpr int kWarps = 8;
constexpr int kRowsPerWarp = kRows / kWarps;
constexpr int kMaxD = 128;

__global__ void __launch_bounds__(kWarps * 32)
    fa_fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                      float* __restrict__ o, float* __restrict__ lse, int N, int d, float scale, int causal) {
  __shared__ float sk[kKeys][kMaxD + 1];
  __shared__ float sv[kKeys][kMaxD];
  __shared__ float sq[kRows][kMaxD];
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * kRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t head = (size_t)bh * N * d;

  for (int i = threadIdx.x; i < kRows * d; i += blockDim.x) {
    const int rr = i / d, cc = i % d;
    sq[rr][cc] = (q0 + rr < N) ? q[head + (size_t)(q0 + rr) * d + cc] : 0.f;
  }
  // per row state: output columns c = lane + 32*u
  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][kMaxD / 32];
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
    for (int u = 0; u < kMaxD / 32; ++u) acc[r][u] = 0.f;
  }
  const int last_row = min(q0 + kRows, N) - 1;
  const int key_end = causal ? last_row + 1 : N;
  for (int kb = 0; kb < key_end; kb += kKeys) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKeys * d; i += blockDim.x) {
      const int rr = i / d, cc = i % d;
      const bool in = kb + rr < N;
      sk[rr][cc] = in ? k[head + (size_t)(kb + rr) * d + cc] : 0.f;
      sv[rr][cc] = in ? v[head + (size_t)(kb + rr) * d + cc] : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int row = warp * kRowsPerWarp + r;
      const int qi = q0 + row;
      const int key = kb + lane;
      float s = 0.f;
      for (int c = 0; c < d; ++c) s = fmaf(sq[row][c], sk[lane][c], s);
      s *= scale;
      const bool visible = key < N && (!causal || key <= qi);
      if (!visible) s = -INFINITY;
      float mx = s;
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[r], mx);
      if (m_new == -INFINITY) continue;  // nothing visible yet for this row
      const float corr = expf(m[r] - m_new);
      const float pj = visible ? expf(s - m_new) : 0.f;
      float ps = pj;
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[r] = l[r] * corr + ps;
      for (int u = 0; u < d / 32; ++u) acc[r][u] *= corr;
      for (int jj = 0; jj < kKeys; ++jj) {
        const float pjj = __shfl_sync(0xffffffffu, pj, jj);
        for (int u = 0; u < d / 32; ++u) acc[r][u] = fmaf(pjj, sv[jj][lane + 32 * u], acc[r][u]);
      }
      m[r] = m_new;
    }
  }
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int qi = q0 + warp * kRowsPerWarp + r;
    if (qi >= N) continue;
    const float inv = 1.f / l[r];
    for (int u = 0; u < d / 32; ++u) o[head + (size_t)qi * d + lane + 32 * u] = acc[r][u] * inv;
    if (lse != nullptr && lane == 0) lse[(size_t)bh * N + qi] = m[r] + logf(l[r]);
  }
}

}  // namespace

cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int BH, int N,
                           int d, float scale, int causal, cudaStream_t s) {
  const dim3 grid((unsigned)((N + kRows - 1) / kRows), (unsigned)BH);
  fa_fwd_f32_kernel<<<grid, kWarps * 32, 0, s>>>(q, k, v, o, lse, N, d, scale, causal);
  return cudaGetLastError();
}

}  // namespace fa
