// Thin inline-PTX wrappers for the Blackwell (sm_100a) features the attention
// kernels use: mbarriers, TMA tensor copies, tensor memory (TMEM) and the
// tcgen05 tensor-core MMA.  Encodings follow the public PTX ISA (tcgen05 shared
// memory descriptor and instruction descriptor tables).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace fa {

// ----------------------------------------------------------------- error word
// Device-side failures are recorded here (the host reads and clears it with
// fa_last_device_status()): a bounded wait that ran out (kDevTimeout), or a value outside
// what the arithmetic can represent -- a non-finite input, a score Q K^T beyond the fp32
// range, a V element too large for the scaled fp16 copy (kDevRange).
enum : int { kDevOk = 0, kDevTimeout = 5, kDevRange = 6 };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Warp-convergent issue: the producer and MMA roles run their loops on all 32
// lanes (so addresses and descriptors stay warp-uniform) and predicate each async
// instruction on `issue`, which is true in exactly one elected lane.
__device__ __forceinline__ uint32_t elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes, uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %2, 0;\n\t"
      "@q mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes), "r"(issue)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared abort flag + bounded wait.  Every wait gives up after `kWaitLimitNs`
// of wall time (or as soon as another role has given up), records kDevTimeout
// in the device error word and returns false; callers then skip the remaining
// work and fall through to the common exit, so no wait can hang the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

struct WaitCtx {
  volatile int* abort_flag;  // in shared memory
  int* err_word;             // in global memory
};

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (((++spins) & 63u) == 0u) {
      if (*w.abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *w.abort_flag = 1;
        atomicExch(w.err_word, kDevTimeout);
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------- register split
// Warp-specialised kernels move registers from the producer / MMA warpgroup to the
// compute warpgroups.  The shares must add up to at most the launch's registers per
// thread-slot, or the increase would wait forever: every kernel that calls these
// static_asserts its split against its launch bound.
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ----------------------------------------------------------------- coalesced row stores
// Lane l of a warp holds 128 bytes (a[0..7], 16 bytes each) of row `row0 + l`, to be written
// at dst + (row0 + l) * ld_bytes.  One lane per row would make every store instruction touch
// 32 rows (32 cache lines); instead each 8-lane group transposes its 8 x 8 block of 16-byte
// units with three xor-shuffle butterfly stages (after the stage with distance s, position m
// of lane l holds what position m ^ s of lane l ^ s held, wherever bit s of m differs from
// bit s of l), after which store instruction i writes row 8g + i of every group g with 8
// consecutive lanes: four full 128-byte lines per instruction.  Rows >= n_rows are skipped.
__device__ __forceinline__ void warp_store_rows_128b(uint4 (&a)[8], uint8_t* dst, size_t ld_bytes, int row0,
                                                     int n_rows) {
  const int lane = threadIdx.x & 31;
  const int gl = lane & 7;      // lane inside its group of 8
  const int gbase = lane & ~7;  // first row (relative to row0) of this group
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
    const bool hi = (gl & s) != 0;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      if (m & s) continue;
      const uint4 send = hi ? a[m] : a[m | s];
      uint4 recv;
      recv.x = __shfl_xor_sync(0xffffffffu, send.x, s);
      recv.y = __shfl_xor_sync(0xffffffffu, send.y, s);
      recv.z = __shfl_xor_sync(0xffffffffu, send.z, s);
      recv.w = __shfl_xor_sync(0xffffffffu, send.w, s);
      if (hi)
        a[m] = recv;
      else
        a[m | s] = recv;
    }
  }
  // lane gl now holds bytes [16 gl, 16 gl + 16) of rows gbase + i in a[i]
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = row0 + gbase + i;
    if (r < n_rows) *reinterpret_cast<uint4*>(dst + (size_t)r * ld_bytes + 16 * gl) = a[i];
  }
}

// ----------------------------------------------------------------- work order
// CTA index -> (head, rank) where rank 0 is the unit with the most work.  Heads are taken
// in groups of `group`; inside a group the units go heaviest first, interleaved over the
// group's heads.  The hardware hands out CTAs roughly in index order, so the lightest units
// of each group come last (short tail), while the CTAs resident at any time read the K/V
// (or Q/dO) of one group of heads, sized by the host to stay in L2.  group = 1 is plain
// head-major order.
__device__ __forceinline__ void unit_order(int cta, int per_head, int n_heads, int group, int& head, int& rank) {
  const int per_group = group * per_head;
  const int g = cta / per_group;
  const int g0 = g * group;
  const int gs = min(group, n_heads - g0);  // heads in this group (the last may be smaller)
  const int r = cta - g * per_group;        // every earlier group is full
  rank = r / gs;
  head = g0 + r % gs;
}

// Grouped-query attention: consecutive groups of H / H_kv query heads share one
// key/value head.  Head indices here run over batch x heads.
__device__ __forceinline__ int kv_head_of(int bh, int H, int H_kv) {
  const int b = bh / H;
  return b * H_kv + (bh - b * H) / (H / H_kv);
}
__device__ __forceinline__ int q_head_of(int bh_kv, int g, int H, int H_kv) {
  const int b = bh_kv / H_kv;
  return b * H + (bh_kv - b * H_kv) * (H / H_kv) + g;
}

// ----------------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ----------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled load global -> shared, completion counted on `bar` (transaction bytes).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, int c0, int c1, int c2,
                                            uint32_t bar, uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %6, 0;\n\t"
      "@q cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "r"(issue)
      : "memory");
}

// 3-D tiled store shared -> global (rows outside the tensor are clipped by the unit).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, int c0, int c1, int c2, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(c0), "r"(c1), "r"(c2), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                          uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %4, 0;\n\t"
      "@q cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "r"(issue)
      : "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (TMA store, MMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------- TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bit, 32 consecutive columns: thread t of the warp gets lane (base lane + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// ----------------------------------------------------------------- tcgen05.mma
// Instruction descriptor for kind::f16 (fp32 accumulate).  Bit layout (PTX ISA,
// "Instruction descriptor" for .kind::f16): [4,6) D format (1 = f32), [7,10) A
// format, [10,13) B format (0 = f16, 1 = bf16), bit 15 / 16 A / B major
// (0 = K-major, 1 = MN-major), [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool bf16, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle.  Bit layout (PTX ISA,
// "Shared memory descriptor"): [0,14) start address >> 4, [16,30) leading
// dimension byte offset >> 4, [32,46) stride dimension byte offset >> 4,
// [46,48) fixed 0b01, [49,52) base offset (0: atoms are 1024-byte aligned),
// [61,64) swizzle mode (2 = 128-byte swizzle).
//   K-major operand : rows of 128 bytes, 8-row atoms `sbo` = 1024 bytes apart;
//                     `lbo` unused.  Advance the start by 32 bytes per K=16 step.
//   MN-major operand: 64-element (128-byte) MN blocks `lbo` bytes apart, 8-row
//                     K groups `sbo` = 1024 bytes apart.  Advance by 2048 bytes
//                     per K=16 step.
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// The same descriptor with the 64-byte swizzle (mode 4): rows of 64 bytes, 8-row atoms of
// 512 bytes.  K-major: `sbo` = 512, start advanced by 32 bytes per instruction step inside
// a row.  MN-major: 64-byte MN blocks `lbo` apart, 8-row K groups `sbo` = 512 apart.  The
// 64-byte swizzle of the tensor-memory-access unit writes exactly this layout into a
// 512-byte-aligned buffer.
__device__ __forceinline__ uint64_t make_sdesc_sw64(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (4ull << 61);
}

// Advance a descriptor's start address by `bytes` (a multiple of 16; the 14-bit
// field holds addresses < 256 KB, so the add never carries out of it).
__device__ __forceinline__ uint64_t sdesc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// D[tmem] (+)= A[smem] * B[smem]^T  (both operands described by descriptors)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate, uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(issue)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]   (A: M lanes x K, two 16-bit elements per 32-bit column)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate, uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(issue)
      : "memory");
}
// The same two products for 8-bit operands (kind::f8f6f4, K = 32 per instruction; the
// instruction descriptor's A / B format 0 is E4M3).  For the TMEM operand each 32-bit column
// holds four consecutive K elements, lowest K in the lowest byte.
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate, uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(issue)
      : "memory");
}
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate, uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(issue)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar, uint32_t issue = 1) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %1, 0;\n\t"
      "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar),
      "r"(issue)
      : "memory");
}

// ----------------------------------------------------------------- math helpers
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// max(a, b) that is NaN if either operand is NaN (fmaxf returns the other operand).
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// ----------------------------------------------------------------- power-of-two range scaling
// The tensor-core products of the kernels take fp16 copies of bf16 tensors (fp16 keeps 11
// significant bits where bf16 keeps 8, but covers only |x| < 65504 and rounds |x| < 2^-14
// to its subnormal grid).  A copy is therefore made as x * 2^e with one exponent e per
// tensor, and every product that reads it undoes 2^e exactly (a power of two) in a scalar
// that it applies anyway: the softmax's scale, the output's 1/l, a gradient's scale.
// amax (the tensor's largest |x|) is handled as its float bits, which order like the values
// for non-negative floats (and put NaN above +inf).
constexpr uint32_t kBitsInf = 0x7F800000u;
__device__ __forceinline__ uint32_t abs_bits(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }
__device__ __forceinline__ uint32_t abs_bits_max_bf16x2(uint32_t acc, uint32_t two_bf16) {
  // |x| of both bf16 halves widened exactly to fp32 bit patterns
  const uint32_t lo = (two_bf16 << 16) & 0x7FFF0000u, hi = two_bf16 & 0x7FFF0000u;
  return max(acc, max(lo, hi));
}
// Streaming form for the passes that read whole tensors: a running pair of bf16 maxima of |x|
// (one packed NaN-propagating max per 32-bit word), folded to fp32 bits once at the end.
__device__ __forceinline__ uint32_t amax_bf16x2_step(uint32_t acc2, uint32_t two_bf16) {
  __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&acc2);
  const uint32_t m = two_bf16 & 0x7FFF7FFFu;
  a = __hmax2_nan(a, *reinterpret_cast<const __nv_bfloat162*>(&m));
  return *reinterpret_cast<const uint32_t*>(&a);
}
__device__ __forceinline__ uint32_t amax_bf16x2_bits(uint32_t acc2) {  // fp32 bits of max(|lo|, |hi|)
  return max(acc2 << 16, acc2 & 0xFFFF0000u);
}
// floor(log2(x)) of a positive finite float given as its bits (subnormals included).
__host__ __device__ __forceinline__ int floor_log2_bits(uint32_t bits) {
  if (bits >= 0x00800000u) return (int)(bits >> 23) - 127;
  int E = -150;  // subnormal: the position of the leading mantissa bit
  for (uint32_t m = bits; m != 0u; m >>= 1) ++E;
  return E;
}
// Exponent that brings a largest magnitude (bits) into [4, 8): e = 2 - floor(log2(amax)),
// capped at 64 (magnitudes below 2^-62 gain nothing further); 0 for zero and non-finite.
__host__ __device__ __forceinline__ int target_exponent(uint32_t amax_bits) {
  if (amax_bits == 0u || amax_bits >= kBitsInf) return 0;
  const int e = 2 - floor_log2_bits(amax_bits);
  return e > 64 ? 64 : e;
}
// Exponent of the copy of a tensor whose largest magnitude has bits `amax_bits`: 0 while
// amax lies in [2^lo_log2, 2^hi_log2] (the common case: the copy is the plain conversion),
// else target_exponent.
__host__ __device__ __forceinline__ int copy_exponent(uint32_t amax_bits, int lo_log2, int hi_log2) {
  if (amax_bits == 0u || amax_bits >= kBitsInf) return 0;
  const int E = floor_log2_bits(amax_bits);
  if (E >= lo_log2 && (E < hi_log2 || (E == hi_log2 && (amax_bits & 0x007FFFFFu) == 0u))) return 0;
  return target_exponent(amax_bits);
}
// (x0, x1) * (s, s) + (t, t) with one packed instruction.
__device__ __forceinline__ void fma2(float& x0, float& x1, float s, float t) {
  uint64_t a, b, c;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(s), "f"(s));
  asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(t), "f"(t));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(a) : "l"(a), "l"(b), "l"(c));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(a));
}
// Packed pair helpers: (x0, x1) op (y0, y1) with one f32x2 instruction.
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
// (a0, a1) * (b0, b1) + (c0, c1)
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fsub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// s0 += low fp16 half of h, s1 += high fp16 half of h (exact widening, fp32 add).
__device__ __forceinline__ void add_f16x2_to_f32(float& s0, float& s1, uint32_t h) {
  asm("{\n\t.reg .f16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.f16 %0, lo, %0;\n\t"
      "add.rn.f32.f16 %1, hi, %1;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "r"(h));
}
// 2^x for a pair of values on the FMA pipe instead of the MUFU unit (16 exponentials
// per clock per SM, the softmax's throughput limit on sm_100a).  Method: round-to-
// nearest range reduction x = j + f, j integer, f in [-1/2, 1/2] (adding 1.5 * 2^23
// leaves round(x) in the low mantissa bits), 2^f by a degree-3 polynomial fitted for
// minimum relative error on [-1/2, 1/2] (max relative error 7.5e-5 in fp32 Horner form on
// [-125.99, 8], below the 2^-11 rounding that P gets next when it is packed to fp16; within
// 1e-4 of -126 the result is an fp32 denormal, relative error up to 1.5e-4), and 2^j
// applied by adding j to the exponent field.  Inputs are clamped to >= -126 so the
// scaled result stays a normal float (2^-126 becomes 0 once rounded to fp16); the
// largest input the softmax produces is 8 (a stale running maximum).  A NaN argument passes
// the clamp and comes out as a huge value (about 3.4e38) rather than NaN: NaN scores come only
// from non-finite inputs or fp32 overflow, which the kernels report as a range error (input
// maxima, the forward's tile sums of P).
constexpr float kExp2Shifter = 12582912.0f;  // 1.5 * 2^23
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111400127411f;
constexpr float kExp2C3 = 0.0551716685295105f;
__device__ __forceinline__ void exp2_fma_pipe(float& a, float& b) {
  a = max_nan(a, -126.0f);
  b = max_nan(b, -126.0f);
  uint64_t x, t, f, p;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a), "f"(b));
  const uint64_t shifter = ((uint64_t)__float_as_uint(kExp2Shifter) << 32) | __float_as_uint(kExp2Shifter);
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(x), "l"(shifter));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f) : "l"(t), "l"(shifter));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f) : "l"(x), "l"(f));
  auto splat = [](float c) { return ((uint64_t)__float_as_uint(c) << 32) | __float_as_uint(c); };
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(splat(kExp2C3)), "l"(f), "l"(splat(kExp2C2)));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(splat(kExp2C1)));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(splat(kExp2C0)));
  float p0, p1, t0, t1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(p0), "=f"(p1) : "l"(p));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(t0), "=f"(t1) : "l"(t));
  a = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  b = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Four floats -> four E4M3 bytes (round to nearest even, saturating to +-448), a in the
// lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xFFFFu) | (hi << 16);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a tile stored
// with the 128-byte swizzle (rows of 128 bytes, 8-row / 1024-byte atoms).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace fa
