// Host side of the C ABI declared in include/fa.h: argument checks, tensor-map
// encoding, workspace carving and kernel launches.  No allocation happens here.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"

namespace fa {

// The library's one piece of device state: an error word per device, written by
// kernels that give up a bounded wait.
__device__ int g_fa_err_word;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices];
int g_cc_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 unsupported
std::mutex g_mu;
int g_num_sms[kMaxDevices] = {};  // multiprocessor count per device (persistent grids)
thread_local void* const* t_phase_events = nullptr;  // see fa_bwd_set_phase_events

// Checks the current device (compute capability 10.0) and resolves its error word.
fa_status device_setup(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_cc_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    g_cc_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (g_cc_ok[dev] < 0) return FA_ERR_UNSUPPORTED;
  if (g_num_sms[dev] == 0 &&
      cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (g_err_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_fa_err_word) != cudaSuccess) return FA_ERR_CUDA;
    g_err_ptr[dev] = static_cast<int*>(ptr);
  }
  *dev_out = dev;
  return FA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Shared validation of sizes/scalars.  Returns FA_OK and sets *empty when there is nothing to do.
// H_kv: key/value heads (H for plain multi-head attention); H must be a multiple of it.
// allow_d256: the forward with a workspace and the backward also take d = 256 (kernels of their own)
fa_status check_problem(int B, int H, int H_kv, int N, int d, float scale, int causal, bool* empty,
                        bool allow_d256 = false) {
  if (B < 0 || H < 0 || N < 0 || H_kv < 0) return FA_ERR_INVALID_ARG;
  if (H > 0 && (H_kv < 1 || H % H_kv != 0)) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && !(allow_d256 && d == 256)) return FA_ERR_UNSUPPORTED;
  *empty = (B == 0 || H == 0 || N == 0);
  if (*empty) return FA_OK;
  const long long BH = (long long)B * H;
  // grid.x = work units <= 2^31-1; every TMA coordinate fits in int32; N padded to 128 fits in int
  if (BH > (1LL << 24) || N > (1 << 30)) return FA_ERR_UNSUPPORTED;
  const long long units = BH * ((N + 127) / 128);
  if (units > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

bool window_ok(int wl, int wr) { return wl >= -1 && wr >= -1; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Forward workspace: the fp16 copy of V, then a 256-byte control block (the persistent
// kernel's work counter at 0, the copy's exponent at 4), then the V pass's per-block maxima.
struct FwdLayout {
  size_t off_ctrl, off_amax, total;
};
FwdLayout fwd_layout(int B, int H_kv, int N, int d) {
  FwdLayout w{};
  w.off_ctrl = align256((size_t)B * H_kv * N * d * 2);
  w.off_amax = w.off_ctrl + 256;
  w.total = w.off_amax + align256(sizeof(uint32_t) * kVPassBlocks);
  return w;
}

struct BwdLayout {
  size_t off_q16, off_k16, off_v16, off_do16, off_delta, off_lse2, off_dk_part, off_dv_part, off_ctrl, off_amax,
      total;
  int Np;
  int kv_split;
};
// The 256-byte control block of the backward workspace: the persistent kernels' work
// counters, then the exponents of the Q, K, V, dO copies.
constexpr size_t kCtrlCounters = 0, kCtrlExps = 16;

// Grouped-query attention with few key/value heads leaves the dK/dV kernel (one CTA per
// key/value head and key tile) with too few, very unequal CTAs: then each group's query
// heads are split over kv_split CTAs -- the smallest divisor of the group size that gives at
// least four CTAs per SM -- whose partial sums a reduction kernel adds up.
constexpr long long kDkdvMinUnits = 4 * 148;
int kv_split_for(int B, int H, int H_kv, int N, int d) {
  const int group = H / H_kv;
  (void)d;  // one unit per key tile (at d = 256 in each of the two dK/dV kernels)
  const long long units = (long long)B * H_kv * ((N + 127) / 128);
  for (int s = 1; s < group; ++s)
    if (group % s == 0 && units * s >= kDkdvMinUnits) return s;
  return group;
}

// Workspace: fp16 copies of Q and dO (B*H heads) and of K and V (B*H_kv heads), then
// D and LSE*log2(e) per query row padded to a multiple of 128 rows, then (only when the
// group is split, see kv_split_for) fp32 partial dK and dV per split, then a 256-byte control
// block (work counters of the persistent kernels, exponents of the copies), then the
// preprocess's per-block maxima of |Q|, |K|, |V|, |dO|.
// Without own_v16 (fa_bwd_ws: the forward's V copy is used) the V copy's space is left out.
BwdLayout bwd_layout(int B, int H, int H_kv, int N, int d, bool own_v16 = true) {
  BwdLayout w{};
  w.kv_split = kv_split_for(B, H, H_kv, N, d);
  const size_t t16 = align256((size_t)B * H * N * d * 2);
  const size_t t16kv = align256((size_t)B * H_kv * N * d * 2);
  w.Np = ((N + 127) / 128) * 128;
  const size_t rows = align256((size_t)B * H * w.Np * 4);
  w.off_q16 = 0;
  w.off_do16 = t16;
  w.off_k16 = 2 * t16;
  w.off_v16 = 2 * t16 + t16kv;
  w.off_delta = 2 * t16 + (own_v16 ? 2 : 1) * t16kv;
  w.off_lse2 = w.off_delta + rows;
  w.off_dk_part = w.off_lse2 + rows;
  const size_t part = w.kv_split > 1 ? align256((size_t)w.kv_split * B * H_kv * N * d * 4) : 0;
  w.off_dv_part = w.off_dk_part + part;
  w.off_ctrl = w.off_dv_part + part;
  w.off_amax = w.off_ctrl + 256;
  w.total = w.off_amax + align256(4 * sizeof(uint32_t) * kPreBlocks);
  return w;
}

}  // namespace

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  return g_err_ptr[dev];
}

bool make_tmap_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int N, int BH,
                  int box_cols, int box_rows, int swizzle_bytes) {
  if ((swizzle_bytes != 128 && swizzle_bytes != 64) || box_cols * elem_bytes != swizzle_bytes) return false;
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * elem_bytes, (cuuint64_t)N * d * elem_bytes};
  const cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_str(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_RANGE: return "FA_ERR_RANGE";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, fa_stream_t stream) {
  return fa_fwd_gqa(q, k, v, o, lse, nullptr, B, H, H, N, d, scale, causal, stream);
}

namespace {
// Shared body of fa_fwd_gqa (V converted on chip) and fa_fwd_ws (V converted to fp16 into
// the workspace by a streaming pass first).
fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, void* o_resid, int B, int H,
                   int H_kv, int N, int d, float scale, int causal, int wl, int wr, void* workspace,
                   size_t workspace_bytes, fa_stream_t stream) {
  bool empty = false;
  if (!window_ok(wl, wr)) return FA_ERR_INVALID_ARG;
  fa_status st = check_problem(B, H, H_kv, N, d, scale, causal, &empty, workspace != nullptr);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(o_resid, 16) || !aligned(workspace, 256))
    return FA_ERR_MISALIGNED;
  const FwdLayout fl = fwd_layout(B, H_kv, N, d);
  if (workspace != nullptr && workspace_bytes < fl.total) return FA_ERR_INVALID_ARG;
  int dev = 0;
  if ((st = device_setup(&dev)) != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H, BH_kv = B * H_kv;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  unsigned* counter = workspace != nullptr ? reinterpret_cast<unsigned*>(wsb + fl.off_ctrl) : nullptr;
  int* v_exp = workspace != nullptr ? reinterpret_cast<int*>(wsb + fl.off_ctrl + 4) : nullptr;
  if (workspace != nullptr &&
      launch_fwd_v16(v, workspace, (long long)BH_kv * N * d, counter, reinterpret_cast<uint32_t*>(wsb + fl.off_amax),
                     v_exp, g_err_ptr[dev], s) != cudaSuccess)
    return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv, to;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool v16 = workspace != nullptr;
  if (d == 256) {  // V (fp16, in the workspace) in 64-key x 64-column boxes for the d = 256 kernel
    if (!make_tmap_3d(&tv, workspace, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, N, BH_kv, 64, 64, 128))
      return FA_ERR_CUDA;
  } else if (!make_tmap_3d(&tv, v16 ? workspace : v, v16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : bf, 2, d, N, BH_kv,
                           64, 128, 128)) {
    return FA_ERR_CUDA;
  }
  if (!make_tmap_3d(&tq, q, bf, 2, d, N, BH, 64, 128, 128) ||
      !make_tmap_3d(&tk, k, bf, 2, d, N, BH_kv, 64, 128, 128) ||
      !make_tmap_3d(&to, o, bf, 2, d, N, BH, 64, 128, 128))
    return FA_ERR_CUDA;
  FwdParams p{};
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_resid = static_cast<__nv_bfloat16*>(o_resid);
  p.counter = counter;
  p.num_sms = g_num_sms[dev];
  p.N = N;
  p.BH = BH;
  p.H = H;
  p.H_kv = H_kv;
  p.n_pairs = (N + 255) / 256;
  // K and V bytes per query head: a group of H / H_kv query heads shares them
  p.head_group = head_group_size(BH, 4ull * N * d / (H / H_kv), kFwdGroupBytes);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out_scale = 1.0f;
  p.v_exp = v_exp;  // the V copy's exponent (persistent kernels); the on-chip kernel scales per tile
  p.causal = causal;
  p.win_left = wl;
  p.win_right = wr;
  p.err = g_err_ptr[dev];
  // with a workspace: the persistent kernel (work counter in the workspace); without: one CTA
  // per unit, V converted on chip
  cudaError_t e;
  if (d == 256) {
    e = launch_fwd_d256_sm100(tq, tk, tv, p, s);
  } else if (v16) {
    // O and the residual in 32-row boxes for the persistent kernel's per-warp bulk stores
    CUtensorMap to32, tr32;
    if (!make_tmap_3d(&to32, o, bf, 2, d, N, BH, 64, 32, 128) ||
        !make_tmap_3d(&tr32, o_resid != nullptr ? o_resid : o, bf, 2, d, N, BH, 64, 32, 128))
      return FA_ERR_CUDA;
    e = launch_fwd_persist_sm100(tq, tk, tv, to32, tr32, p, d, s);
  } else {
    e = launch_fwd_sm100(tq, tk, tv, to, p, d, s);
  }
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
}  // namespace

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, void* o_resid, int B, int H,
                     int H_kv, int N, int d, float scale, int causal, fa_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, o_resid, B, H, H_kv, N, d, scale, causal, -1, -1, nullptr, 0, stream);
}

size_t fa_fwd_workspace_size(int B, int H_kv, int N, int d) {
  bool empty = false;
  if (check_problem(B, H_kv, H_kv, N, d, 1.0f, 0, &empty, true) != FA_OK || empty) return 0;
  return fwd_layout(B, H_kv, N, d).total;  // fp16 V, control block, per-block maxima
}

fa_status fa_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, void* o_resid, int B, int H,
                    int H_kv, int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                    fa_stream_t stream) {
  if (workspace == nullptr) {
    bool empty = false;
    const fa_status st = check_problem(B, H, H_kv, N, d, scale, causal, &empty, true);
    return (st != FA_OK || empty) ? st : FA_ERR_INVALID_ARG;
  }
  return fwd_impl(q, k, v, o, lse, o_resid, B, H, H_kv, N, d, scale, causal, -1, -1, workspace, workspace_bytes,
                  stream);
}

fa_status fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N,
                     int d, float scale, int causal, fa_stream_t stream) {
  bool empty = false;
  fa_status st = check_problem(B, H, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(o, 4) || !aligned(lse, 4))
    return FA_ERR_MISALIGNED;
  int dev = 0;
  if ((st = device_setup(&dev)) != FA_OK) return st;
  return launch_fwd_f32(q, k, v, o, lse, B * H, N, d, scale, causal, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) { return fa_bwd_gqa_workspace_size(B, H, H, N, d); }

size_t fa_bwd_gqa_workspace_size(int B, int H, int H_kv, int N, int d) {
  bool empty = false;
  if (check_problem(B, H, H_kv, N, d, 1.0f, 0, &empty, true) != FA_OK || empty) return 0;
  return bwd_layout(B, H, H_kv, N, d).total;
}

size_t fa_bwd_ws_workspace_size(int B, int H, int H_kv, int N, int d) {
  bool empty = false;
  if (check_problem(B, H, H_kv, N, d, 1.0f, 0, &empty, true) != FA_OK || empty) return 0;
  return bwd_layout(B, H, H_kv, N, d, false).total;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 float* dq, float* dk, float* dv, int B, int H, int N, int d, float scale, int causal,
                 void* workspace, fa_stream_t stream) {
  // the caller provides at least fa_bwd_workspace_size(B, H, N, d) bytes (the signature carries no size)
  return fa_bwd_gqa(q, k, v, o, nullptr, dout, lse, dq, dk, dv, B, H, H, N, d, scale, causal, workspace,
                    fa_bwd_workspace_size(B, H, N, d), stream);
}

namespace {
fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                   const void* dout, const float* lse, float* dq, float* dk, float* dv, int B, int H, int H_kv, int N,
                   int d, float scale, int causal, int wl, int wr, void* workspace, size_t workspace_bytes,
                   fa_stream_t stream, void* fwd_workspace = nullptr);
}  // namespace

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                     const void* dout, const float* lse, float* dq, float* dk, float* dv, int B, int H, int H_kv,
                     int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                     fa_stream_t stream) {
  return bwd_impl(q, k, v, o, o_resid, dout, lse, dq, dk, dv, B, H, H_kv, N, d, scale, causal, -1, -1, workspace,
                  workspace_bytes, stream);
}

fa_status fa_bwd_ws(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                    const void* dout, const float* lse, float* dq, float* dk, float* dv, int B, int H, int H_kv, int N,
                    int d, float scale, int causal, void* fwd_workspace, size_t fwd_workspace_bytes, void* workspace,
                    size_t workspace_bytes, fa_stream_t stream) {
  bool empty = false;
  const fa_status st = check_problem(B, H, H_kv, N, d, scale, causal, &empty, true);
  if (st != FA_OK || empty) return st;
  if (fwd_workspace == nullptr || fwd_workspace_bytes < fwd_layout(B, H_kv, N, d).total) return FA_ERR_INVALID_ARG;
  if (!aligned(fwd_workspace, 256)) return FA_ERR_MISALIGNED;
  return bwd_impl(q, k, v, o, o_resid, dout, lse, dq, dk, dv, B, H, H_kv, N, d, scale, causal, -1, -1, workspace,
                  workspace_bytes, stream, fwd_workspace);
}

namespace {
fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                   const void* dout, const float* lse, float* dq, float* dk, float* dv, int B, int H, int H_kv, int N,
                   int d, float scale, int causal, int wl, int wr, void* workspace, size_t workspace_bytes,
                   fa_stream_t stream, void* fwd_workspace) {
  bool empty = false;
  if (!window_ok(wl, wr)) return FA_ERR_INVALID_ARG;
  fa_status st = check_problem(B, H, H_kv, N, d, scale, causal, &empty, true);  // d in {64, 128, 256}
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  const bool reuse_v = fwd_workspace != nullptr;  // the V copy of fa_fwd_ws's workspace (fa_bwd_ws)
  const BwdLayout w = bwd_layout(B, H, H_kv, N, d, !reuse_v);
  if (workspace_bytes < w.total) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(o_resid, 16) || !aligned(lse, 4) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(workspace, 256))
    return FA_ERR_MISALIGNED;
  int dev = 0;
  if ((st = device_setup(&dev)) != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H, BH_kv = B * H_kv, group = H / H_kv;
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  BwdPreParams pp{};
  pp.q = q;
  pp.k = k;
  pp.v = v;
  pp.o = o;
  pp.o_resid = o_resid;
  pp.dout = dout;
  pp.lse = lse;
  pp.q16 = ws + w.off_q16;
  pp.k16 = ws + w.off_k16;
  pp.do16 = ws + w.off_do16;
  int* v_exp_fwd = nullptr;
  if (reuse_v) {  // the forward workspace: V copy at 0, its exponent in the control block, V-pass maxima
    const FwdLayout fl = fwd_layout(B, H_kv, N, d);
    uint8_t* fws = static_cast<uint8_t*>(fwd_workspace);
    const long long n8 = (long long)B * H_kv * N * d / 8;
    pp.v16 = fws;
    v_exp_fwd = reinterpret_cast<int*>(fws + fl.off_ctrl + 4);
    pp.v_exp_fwd = v_exp_fwd;
    pp.v_amax_fwd = reinterpret_cast<const uint32_t*>(fws + fl.off_amax);
    pp.v_n_part_fwd = (int)std::min<long long>((n8 + 255) / 256, kVPassBlocks);  // the V pass's grid
  } else {
    pp.v16 = ws + w.off_v16;
  }
  pp.delta = reinterpret_cast<float*>(ws + w.off_delta);
  pp.lse2 = reinterpret_cast<float*>(ws + w.off_lse2);
  pp.N = N;
  pp.Np = w.Np;
  pp.BH = BH;
  pp.BH_kv = BH_kv;
  pp.counters = reinterpret_cast<unsigned*>(ws + w.off_ctrl + kCtrlCounters);
  pp.amax_part = reinterpret_cast<uint32_t*>(ws + w.off_amax);
  pp.exps = reinterpret_cast<int*>(ws + w.off_ctrl + kCtrlExps);
  pp.err = g_err_ptr[dev];
  pp.d = d;
  if (launch_bwd_pre(pp, s) != cudaSuccess) return FA_ERR_CUDA;
  if (t_phase_events != nullptr && t_phase_events[0] != nullptr &&
      cudaEventRecord(static_cast<cudaEvent_t>(t_phase_events[0]), s) != cudaSuccess)
    return FA_ERR_CUDA;

  const CUtensorMapDataType h = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap t_q, t_do, t_k, t_v;  // 128-row boxes, shared by the dK/dV and dQ kernels
  if (!make_tmap_3d(&t_q, pp.q16, h, 2, d, N, BH, 64, 128, 128) ||
      !make_tmap_3d(&t_do, pp.do16, h, 2, d, N, BH, 64, 128, 128) ||
      !make_tmap_3d(&t_k, pp.k16, h, 2, d, N, BH_kv, 64, 128, 128) ||
      !make_tmap_3d(&t_v, pp.v16, h, 2, d, N, BH_kv, 64, 128, 128))
    return FA_ERR_CUDA;
  BwdParams bp{};
  bp.v_exp_fwd = v_exp_fwd;
  bp.delta = pp.delta;
  bp.lse2 = pp.lse2;
  bp.exps = pp.exps;
  bp.dq = dq;
  bp.dk = dk;
  bp.dv = dv;
  bp.N = N;
  bp.Np = w.Np;
  bp.BH = BH;
  bp.H = H;
  bp.H_kv = H_kv;
  // dQ orders query heads (K and V bytes per query head shared by the group); dK/dV orders
  // key/value heads (Q and dO of the whole group per key/value head)
  bp.head_group = head_group_size(BH, 4ull * N * d / group, kBwdGroupBytes);
  bp.head_group_kv = head_group_size(BH_kv, 4ull * N * d * (group / w.kv_split), kBwdGroupBytes);
  bp.kv_split = w.kv_split;
  bp.num_sms = g_num_sms[dev];
  bp.dq_counter = pp.counters;
  bp.dkdv_counter = pp.counters + 1;
  bp.dk_counter = pp.counters + 2;
  bp.dk_part = w.kv_split > 1 ? reinterpret_cast<float*>(ws + w.off_dk_part) : nullptr;
  bp.dv_part = w.kv_split > 1 ? reinterpret_cast<float*>(ws + w.off_dv_part) : nullptr;
  bp.scale = scale;
  bp.scale_log2 = scale * 1.4426950408889634f;
  bp.causal = causal;
  bp.win_left = wl;
  bp.win_right = wr;
  bp.err = g_err_ptr[dev];
  // dV, dK (or their partial sums per group split) in 32 x 32 fp32 boxes for the dK/dV epilogue
  CUtensorMap t_dv, t_dk;
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const int out_heads = w.kv_split > 1 ? w.kv_split * BH_kv : BH_kv;
  if (!make_tmap_3d(&t_dv, w.kv_split > 1 ? static_cast<void*>(bp.dv_part) : dv, f32, 4, d, N, out_heads, 32, 32, 128) ||
      !make_tmap_3d(&t_dk, w.kv_split > 1 ? static_cast<void*>(bp.dk_part) : dk, f32, 4, d, N, out_heads, 32, 32, 128))
    return FA_ERR_CUDA;
  if (launch_bwd_dkdv_sm100(t_q, t_do, t_k, t_v, t_dv, t_dk, bp, d, s) != cudaSuccess) return FA_ERR_CUDA;
  if (w.kv_split > 1 &&
      launch_bwd_kv_reduce(bp.dk_part, bp.dv_part, dk, dv, (long long)BH_kv * N * d, w.kv_split, s) != cudaSuccess)
    return FA_ERR_CUDA;
  if (t_phase_events != nullptr && t_phase_events[1] != nullptr &&
      cudaEventRecord(static_cast<cudaEvent_t>(t_phase_events[1]), s) != cudaSuccess)
    return FA_ERR_CUDA;
  if (launch_bwd_dq_sm100(t_q, t_do, t_k, t_v, bp, d, s) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

}  // namespace

// ---- descriptor-based entry points (every option: grouped heads, sliding window)
size_t fa_attn_fwd_workspace_size(const fa_attn_problem* pr) {
  if (pr == nullptr || !window_ok(pr->window_left, pr->window_right)) return 0;
  return fa_fwd_workspace_size(pr->B, pr->H_kv, pr->N, pr->d);
}

fa_status fa_attn_fwd(const fa_attn_problem* pr, const void* q, const void* k, const void* v, void* o, float* lse,
                      void* o_resid, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (pr == nullptr) return FA_ERR_INVALID_ARG;
  if (workspace == nullptr) {
    bool empty = false;
    const fa_status st = check_problem(pr->B, pr->H, pr->H_kv, pr->N, pr->d, pr->scale, pr->causal, &empty, true);
    return (st != FA_OK || empty) ? st : FA_ERR_INVALID_ARG;
  }
  return fwd_impl(q, k, v, o, lse, o_resid, pr->B, pr->H, pr->H_kv, pr->N, pr->d, pr->scale, pr->causal,
                  pr->window_left, pr->window_right, workspace, workspace_bytes, stream);
}

size_t fa_attn_bwd_workspace_size(const fa_attn_problem* pr) {
  if (pr == nullptr || !window_ok(pr->window_left, pr->window_right)) return 0;
  return fa_bwd_gqa_workspace_size(pr->B, pr->H, pr->H_kv, pr->N, pr->d);
}

fa_status fa_attn_bwd(const fa_attn_problem* pr, const void* q, const void* k, const void* v, const void* o,
                      const void* o_resid, const void* dout, const float* lse, float* dq, float* dk, float* dv,
                      void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (pr == nullptr) return FA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, o_resid, dout, lse, dq, dk, dv, pr->B, pr->H, pr->H_kv, pr->N, pr->d, pr->scale,
                  pr->causal, pr->window_left, pr->window_right, workspace, workspace_bytes, stream);
}

// ---- 8-bit forward: E4M3 inputs with per-tensor descales (d = 128 or 64)
size_t fa_attn_fwd_fp8_workspace_size(const fa_attn_problem* pr) {
  if (pr == nullptr || !window_ok(pr->window_left, pr->window_right)) return 0;
  return 256;  // the persistent kernel's work counter
}

fa_status fa_attn_fwd_fp8(const fa_attn_problem* pr, const void* q, const void* k, const void* v, float q_descale,
                          float k_descale, float v_descale, void* o, float* lse, void* workspace,
                          size_t workspace_bytes, fa_stream_t stream) {
  if (pr == nullptr || !window_ok(pr->window_left, pr->window_right)) return FA_ERR_INVALID_ARG;
  const int B = pr->B, H = pr->H, H_kv = pr->H_kv, N = pr->N, d = pr->d;
  bool empty = false;
  fa_status st = check_problem(B, H, H_kv, N, d, pr->scale, pr->causal, &empty);
  if (st != FA_OK) return st;
  for (const float ds : {q_descale, k_descale, v_descale})
    if (!(std::isfinite(ds) && ds > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 128 && d != 64) return FA_ERR_UNSUPPORTED;  // one 128- or 64-byte swizzle row per Q / K / V row
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !workspace || workspace_bytes < 256) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(workspace, 256))
    return FA_ERR_MISALIGNED;
  int dev = 0;
  if ((st = device_setup(&dev)) != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H, BH_kv = B * H_kv;
  unsigned* counter = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(counter, 0, sizeof(unsigned), s) != cudaSuccess) return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMap to32;  // bf16 O in 32-row boxes (the epilogue's bulk stores)
  if (!make_tmap_3d(&tq, q, u8, 1, d, N, BH, d, 128, d) || !make_tmap_3d(&tk, k, u8, 1, d, N, BH_kv, d, 128, d) ||
      !make_tmap_3d(&tv, v, u8, 1, d, N, BH_kv, d, 128, d) ||
      !make_tmap_3d(&to32, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, BH, 64, 32, 128))
    return FA_ERR_CUDA;
  FwdParams p{};
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_resid = nullptr;
  p.counter = counter;
  p.num_sms = g_num_sms[dev];
  p.N = N;
  p.BH = BH;
  p.H = H;
  p.H_kv = H_kv;
  p.n_pairs = (N + 255) / 256;
  p.head_group = head_group_size(BH, 2ull * N * d / (H / H_kv), kFwdGroupBytes);  // 8-bit K and V
  // S = q_descale * k_descale * (Q8 K8^T): both descales fold into the exponent's scale
  p.scale_log2 = (float)((double)pr->scale * q_descale * k_descale * 1.4426950408889634);
  p.out_scale = v_descale;
  p.causal = pr->causal;
  p.win_left = pr->window_left;
  p.win_right = pr->window_right;
  p.err = g_err_ptr[dev];
  return launch_fwd_persist_fp8_sm100(tq, tk, tv, to32, p, d, s) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

void fa_bwd_set_phase_events(void* const* events) { t_phase_events = events; }

fa_status fa_selftest_wait_timeout(fa_stream_t stream) {
  int dev = 0;
  const fa_status st = device_setup(&dev);
  if (st != FA_OK) return st;
  return launch_selftest_wait(g_err_ptr[dev], reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK
                                                                                                      : FA_ERR_CUDA;
}

fa_status fa_selftest_exp2(const float* x, float* y, int n, fa_stream_t stream) {
  if (n < 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (x == nullptr || y == nullptr) return FA_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(y, 4)) return FA_ERR_MISALIGNED;
  int dev = 0;
  const fa_status st = device_setup(&dev);
  if (st != FA_OK) return st;
  return launch_selftest_exp2(x, y, n, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_last_device_status(fa_stream_t stream) {
  int dev = 0;
  fa_status st = device_setup(&dev);
  if (st != FA_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fa_err_word, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fa_err_word, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return v == FA_ERR_RANGE ? FA_ERR_RANGE : FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

fa_status fa_device_status(fa_stream_t stream) { return fa_last_device_status(stream); }

}  // extern "C"
