// Internal launch interface shared by the C-ABI host code and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace fa {

struct FwdParams {
  float* lse;        // (B*H, N) fp32, natural-log LSE of the scaled scores; may be null
  __nv_bfloat16* o;  // (B*H, N, d) bf16 output (the persistent kernel stores it directly)
  unsigned* counter; // persistent kernel: work units handed out so far (zeroed by the V conversion)
  int num_sms;       // persistent kernel: grid size
  __nv_bfloat16* o_resid;  // (B*H, N, d) bf16 residual O_fp32 - O_bf16; may be null
  int N;             // sequence length (queries = keys)
  int BH;            // B * H (query heads)
  int H, H_kv;       // query heads and key/value heads per batch entry (H a multiple of H_kv)
  int n_pairs;       // ceil(N / 256): work units per head (two 128-row query tiles each)
  int head_group;    // heads per group in the CTA order (unit_order)
  float scale_log2;  // softmax scale * log2(e) (times the Q and K descales for 8-bit inputs)
  float out_scale;   // factor on O / l: 1, or the V descale for 8-bit inputs
  const int* v_exp;  // persistent kernels: exponent e of the fp16 V copy (V16 = V * 2^e), or null (0)
  int causal;
  int win_left, win_right;  // sliding window: query i sees keys i - left .. i + right (-1 unbounded)
  int* err;          // device error word
};

// Visible keys of query row i under the causal mask and the sliding window (inclusive
// bounds; rows past N behave like row N - 1, so every row keeps at least one key).
__host__ __device__ __forceinline__ int key_lo(int i, int N, int wl) {
  const int r = i < N ? i : N - 1;
  return (wl >= 0 && r - wl > 0) ? r - wl : 0;
}
__host__ __device__ __forceinline__ int key_hi(int i, int N, int causal, int wr) {
  const int r = i < N ? i : N - 1;
  if (causal) return r;
  return (wr >= 0 && r + wr < N - 1) ? r + wr : N - 1;
}
// Queries that see key k (the inverse of the row ranges above; N = query count).
__host__ __device__ __forceinline__ int query_lo(int k, int causal, int wr) {
  if (causal) return k;
  return (wr >= 0 && k - wr > 0) ? k - wr : 0;
}
__host__ __device__ __forceinline__ int query_hi(int k, int N, int wl) {
  return (wl >= 0 && k + wl < N - 1) ? k + wl : N - 1;
}

constexpr int kNumCounters = 3;  // work counters: [0] dQ kernel, [1] dK/dV (d = 256: dV) kernel, [2] d = 256 dK kernel

// Streaming passes that make fp16 copies (the forward's V pass, the backward preprocess)
// run on a fixed grid and leave one partial maximum |x| per block and tensor (float bits);
// the fix-up kernel that follows reduces them and picks each copy's exponent.
constexpr int kVPassBlocks = 148 * 16;  // forward V pass
constexpr int kPreBlocks = 148 * 8;     // backward preprocess
constexpr int kFixupBlocks = 148 * 4;   // fix-up kernels (re-conversion only when a copy needs 2^e != 1)
// Copy exponents (see copy_exponent): a copy keeps e = 0 while its tensor's largest
// magnitude lies in [2^kCopyLoLog2, 2^kCopyHiLog2].
constexpr int kCopyLoLog2 = -4;
constexpr int kCopyHiLog2 = 15;
// The backward's dS = P * (dP - D) is packed to fp16 unscaled in the units of the dO and V
// copies: |dS| <= 2 d max|dO| max|V| must stay <= 2^15 there.
constexpr float kDsBound = 32768.0f;
enum { kExpQ = 0, kExpK = 1, kExpV = 2, kExpDO = 3 };  // slots of the backward's exponent table

struct BwdPreParams {
  const void* q;     // bf16 (BH, N, d)
  const void* k;
  const void* v;
  const void* o;
  const void* o_resid;  // may be null: D then uses the bf16 O alone
  const void* dout;
  const float* lse;  // (BH, N)
  void* q16;         // fp16 copies (BH, N, d)
  void* k16;
  void* v16;
  void* do16;
  float* delta;      // (BH, Np): rowsum(dO * O) (times 2^(e_V + e_dO) after the fix-up); 0 on padded rows
  float* lse2;       // (BH, Np): LSE * log2(e); +inf on padded rows
  int N, Np, BH, d;
  int BH_kv;         // B * H_kv: rows of k / v / k16 / v16 (<= BH)
  unsigned* counters;  // work counters of the persistent kernels, zeroed here (kNumCounters)
  uint32_t* amax_part; // [4][kPreBlocks] partial max |x| (float bits) of Q, K, V, dO per block
  int* exps;         // [4] exponents of the Q, K, V, dO copies (written by the fix-up)
  int* err;          // device error word
  // Reuse of the forward's V copy (fa_bwd_ws), else null / 0: v16 then points into the
  // forward's workspace, the preprocess leaves V alone, the fix-up takes max |V| from the V
  // pass's per-block maxima and re-converts the copy only when the backward's exponent for V
  // differs from the copy's (*v_exp_fwd; the dK/dV kernel then records the new one).
  const uint32_t* v_amax_fwd;  // [v_n_part_fwd] the V pass's per-block max |V| (float bits)
  int v_n_part_fwd;
  const int* v_exp_fwd;        // exponent of the forward's V copy
};

struct BwdParams {
  int* v_exp_fwd;      // fa_bwd_ws: the forward workspace's V exponent, set to exps[kExpV] (else null)
  const float* delta;  // (BH, Np), in the units of the dO and V copies
  const float* lse2;   // (BH, Np)
  const int* exps;     // [4] exponents of the Q, K, V, dO copies (kExpQ ...)
  float* dq;           // fp32 (BH, N, d)
  float* dk;
  float* dv;
  int N, Np, BH;
  int H, H_kv;         // query heads and key/value heads per batch entry (H a multiple of H_kv)
  int head_group;      // query heads per group in the dQ kernel's CTA order (unit_order)
  int head_group_kv;   // key/value heads per group in the dK/dV kernel's CTA order
  int kv_split;        // CTAs sharing one (key/value head, key tile): each takes H/H_kv/kv_split query heads
  float* dk_part;      // with kv_split > 1: fp32 (kv_split, B*H_kv, N, d) partial dK (scaled) and dV,
  float* dv_part;      //   summed into dk / dv by launch_bwd_kv_reduce; unused when kv_split == 1
  int num_sms;         // multiprocessors of the device (grid of the persistent kernels)
  unsigned* dq_counter;  // work units handed out so far by the persistent dQ kernel (zeroed by the preprocess)
  unsigned* dkdv_counter;  // the same for the persistent dK/dV kernel (d = 256: the dV kernel)
  unsigned* dk_counter;    // the same for the d = 256 dK kernel
  float scale;         // softmax scale (applied to dQ and dK)
  float scale_log2;    // scale * log2(e)
  int causal;
  int win_left, win_right;  // sliding window (see FwdParams)
  int* err;
};

// Tensor maps are 3-D views (d, N, B*H) of a (B, H, N, d) tensor with the
// 128-byte swizzle and a box of 64 columns x `box_rows` rows.
// Heads per group in the CTA order: as many heads as keep the streamed operand pair
// (K and V in the forward and dQ kernels, Q and dO in the dK/dV kernel; `per_head`
// bytes per head of the CTA order) within `budget` bytes of L2.  Measured on B200 (N = 2048 and 8192, d = 128):
// the forward runs best with 16 MB groups, the backward with 8 MB.
constexpr unsigned long long kFwdGroupBytes = 16ull << 20;
constexpr unsigned long long kBwdGroupBytes = 8ull << 20;
inline int head_group_size(int BH, unsigned long long per_head, unsigned long long budget) {
  unsigned long long g = budget / (per_head ? per_head : 1ull);
  if (g < 1ull) g = 1ull;
  return g > (unsigned long long)BH ? BH : (int)g;
}

// (d, N, BH) tensor, boxes of box_cols x box_rows, with the 128- or 64-byte swizzle (a box row
// of box_cols elements must be exactly that many bytes)
bool make_tmap_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int N, int BH,
                  int box_cols, int box_rows, int swizzle_bytes);

cudaError_t launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const FwdParams& p, int d, cudaStream_t s);
// V pass of the workspace forward: V -> fp16 copy (exponent 0) with per-block maxima, then the
// fix-up that picks the copy's exponent (v_exp) and re-converts V if it is not 0.
cudaError_t launch_fwd_v16(const void* v, void* v16, long long elems, unsigned* counter, uint32_t* amax_part,
                           int* v_exp, int* err, cudaStream_t s);
// to32, tr32: O and the residual in 64-column x 32-row boxes (the epilogue's bulk stores)
cudaError_t launch_fwd_persist_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                     const CUtensorMap& to32, const CUtensorMap& tr32, const FwdParams& p, int d,
                                     cudaStream_t s);
cudaError_t launch_fwd_d256_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                  const FwdParams& p, cudaStream_t s);  // d = 256, fp16 V in 64 x 64 boxes
cudaError_t launch_fwd_persist_fp8_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                         const CUtensorMap& to32, const FwdParams& p, int d,
                                         cudaStream_t s);  // d = 128 or 64, E4M3
cudaError_t launch_selftest_wait(int* err, cudaStream_t s);
cudaError_t launch_selftest_exp2(const float* x, float* y, int n, cudaStream_t s);
cudaError_t launch_bwd_kv_reduce(const float* dk_part, const float* dv_part, float* dk, float* dv,
                                 long long elems, int splits, cudaStream_t s);
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int BH, int N,
                           int d, float scale, int causal, cudaStream_t s);
// Backward preprocess (D, LSE * log2(e), fp16 copies with exponent 0, per-block maxima), then
// the fix-up that picks the copies' exponents, re-converts where they are not 0 and scales D.
cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t s);
// tdv, tdk: fp32 dV and dK (or, with kv_split > 1, the partial buffers: kv_split * B * H_kv
// heads) in 32-column x 32-row boxes, for the epilogue's bulk stores (d = 64, 128)
cudaError_t launch_bwd_dkdv_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const CUtensorMap& tdv, const CUtensorMap& tdk,
                                  const BwdParams& p, int d, cudaStream_t s);
cudaError_t launch_bwd_dq_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                const CUtensorMap& tv, const BwdParams& p, int d, cudaStream_t s);

int* device_error_word();  // address of the library's device error word on the current device

}  // namespace fa
