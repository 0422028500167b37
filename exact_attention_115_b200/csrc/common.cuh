// Shared device helpers for the sm_100a attention kernels: shared-memory
// barriers with bounded waits, TMA tensor loads, and the tcgen05 (5th
// generation tensor core) instructions with their operand descriptors.
//
// Every wait on an mbarrier is bounded: after kWaitLimitNs of wall time the
// waiting thread records FA_ERR_TIMEOUT in the device error word, raises the
// CTA's abort flag and returns false.  Every later wait in the CTA sees the
// flag and returns at once, so all roles run to the final barrier and the
// TMEM allocation is always freed.  Nothing here traps.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa.h"

namespace fa {

// Device error word, one per translation unit (so no relocatable device
// code is needed); each kernel file exports a host accessor made with
// FA_ERROR_ACCESSOR that reads and clears it for fa_status.
static __device__ int g_fa_error = 0;
// Code of the first wait that timed out (file base + source line), 0 if none.
static __device__ int g_fa_site = 0;

#define FA_ERROR_ACCESSOR(name)                                                 \
  cudaError_t name(int* word, int* site) {                                      \
    int w = 0, st = 0;                                                          \
    cudaError_t e = cudaMemcpyFromSymbol(&w, g_fa_error, sizeof(int));          \
    if (e != cudaSuccess) return e;                                             \
    e = cudaMemcpyFromSymbol(&st, g_fa_site, sizeof(int));                      \
    if (e != cudaSuccess) return e;                                             \
    *word |= w;                                                                 \
    if (st != 0 && *site == 0) *site = st;                                      \
    if (w != 0 || st != 0) {                                                    \
      const int z = 0;                                                          \
      e = cudaMemcpyToSymbol(g_fa_error, &z, sizeof(int));                      \
      if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_fa_site, &z, sizeof(int)); \
    }                                                                           \
    return e;                                                                   \
  }

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Bits OR-ed into the error word by kernels.
enum : int {
  kErrTimeout = 1,  // a bounded wait expired
  kErrLayout = 2,   // a kernel found its dynamic shared memory misaligned and did nothing
  kErrBounds = 4,   // debug builds: an index check failed (the access was skipped)
};

// Index checks of the debug build (FA_DEBUG): FA_INBOUNDS(cond) is true when
// cond holds; otherwise it records kErrBounds and the check's site (file
// base + line) in the device error word and is false, and the caller skips
// the access.  Release builds compile it to `true`.
__device__ __forceinline__ bool fa_inbounds(bool ok, int site) {
  if (!ok) {
    atomicOr(&g_fa_error, kErrBounds);
    atomicCAS(&g_fa_site, 0, site);
  }
  return ok;
}
#ifdef FA_DEBUG
#define FA_INBOUNDS(cond) fa_inbounds(bool(cond), FA_SITE_BASE + __LINE__)
#else
#define FA_INBOUNDS(cond) true
#endif

constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Launch order of a 1-D grid over (head, block) pairs.  Heads (b·H + h) go in
// groups of `group`; inside a group the CTAs run block index by block index,
// every head of the group at each index.  The caller numbers its blocks so
// that index 0 is the most work (the longest causal row or column range):
// the hardware then starts the heavy CTAs first and the short ones fill the
// end of the launch, while the CTAs alive at one time touch the inputs of
// only one or two groups of heads, sized on the host to stay in L2.
__device__ __forceinline__ void grouped_order(int lin, int BH, int nblk, int group, int& bh,
                                              int& blk) {
  const int per_group = group * nblk;
  const int g = lin / per_group;
  const int rem = lin - g * per_group;
  const int gh = min(group, BH - g * group);  // heads in this group (the last one may be short)
  blk = rem / gh;
  bh = g * group + (rem - blk * gh);
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: if the phase is not complete the thread
// is parked (it issues nothing) until the phase completes or `hint_ns`
// passes.  A waiting warp therefore does not take issue slots from the warps
// of its SM sub-partition that have work, the MMA-issuing thread included.
constexpr uint32_t kSuspendHintNs = 1000000;  // 1 ms; the thread wakes at completion
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Wait until the phase of `bar` with the given parity has completed.
// Returns false (and leaves the CTA aborted) on timeout or if the CTA was
// already aborted by another thread.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int site = 0,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait_sleep(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(&g_fa_error, kErrTimeout);
      atomicCAS(&g_fa_site, 0, site);
      return false;
    }
  }
}
// mbar_wait tagged with the call's source line (plus a per-file base set by
// FA_SITE_BASE) so a timeout can be traced to its wait.
#define MBAR_WAIT(bar, parity, abort_flag) mbar_wait(bar, parity, abort_flag, FA_SITE_BASE + __LINE__)
// The same, by every lane of a converged warp, with a warp-uniform result.
#define MBAR_WAIT_WARP(bar, parity, abort_flag) \
  __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, FA_SITE_BASE + __LINE__))

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled tensor load into this CTA's shared memory, completing on `bar`.
// x is the innermost coordinate (elements); it is always a multiple of the
// 128-byte swizzle width here, so x * element size is 16-byte aligned.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ------------------------------------------------------------------ bulk groups, fences, named barriers
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier that also ANDs a predicate over the participating threads,
// so a go/no-go decision is uniform across them.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// 4-D tiled load of one box (x = element in the row, y = row, z = head,
// w = batch): attention tensors with arbitrary batch / head / row strides.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}


// Tiled store of one box from shared memory (bulk-group completion: the
// caller commits and waits on the group before reusing `src` or exiting).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 2-D tiled store / reduce-add of one box from shared memory (bulk-group
// completion, as tma_store_3d).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x,
                                                  int y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y)
      : "memory");
}

// A [B, H, N, d] tensor's box at (x, row, head-and-batch index bh): through a
// 3-D map (d, N, B·H) when the layout lets heads and batches merge into one
// index, else a 4-D map (d, N, H, B).
__device__ __forceinline__ void tma_load_bh(void* dst, const CUtensorMap* map, bool map4d,
                                            uint64_t* bar, int x, int y, int bh, int H) {
  if (map4d)
    tma_load_4d(dst, map, bar, x, y, bh % H, bh / H);
  else
    tma_load_3d(dst, map, bar, x, y, bh);
}
__device__ __forceinline__ void tma_store_bh(const CUtensorMap* map, bool map4d, const void* src,
                                             int x, int y, int bh, int H) {
  if (map4d)
    tma_store_4d(map, src, x, y, bh % H, bh / H);
  else
    tma_store_3d(map, src, x, y, bh);
}

// Keys visible to head index bh = b·H + h: all Nk, or the key-padding length
// kv_len[b] clamped to [0, Nk].
__device__ __forceinline__ int keys_of(const int* kv_len, int bh, int H, int Nk) {
  return kv_len ? min(max(__ldg(kv_len + bh / H), 0), Nk) : Nk;
}

// ------------------------------------------------------------------ tcgen05
// True in exactly one lane of the calling warp (elect.sync over all 32 lanes,
// which must all execute it).  The MMA-issuing warps run their loops with the
// whole warp, so descriptor arithmetic stays warp-uniform, and only the
// elected lane issues each tcgen05.mma / tcgen05.commit.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive (once) on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]
template <bool TF32>
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  if constexpr (TF32) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// D[tmem] (+)= A[tmem] * B[smem]
template <bool TF32>
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  if constexpr (TF32) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// Load 32 consecutive 32-bit TMEM columns of this warp's 32 lanes (one lane
// per thread).  The values are valid only after tmem_ld_wait().
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 16-column variants (one lane per thread, 16 consecutive 32-bit columns).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a tile stored in the 128-byte swizzled
// canonical layout (rows of 128 bytes, 8-row groups of 1024 bytes).
//   K-major operand: lbo unused (16), sbo = 1024 (next 8-row group).
//   MN-major operand: lbo = bytes between 128-byte-wide column blocks,
//                     sbo = 1024 (next group of 8 K rows).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;  // descriptor version for sm_100
  d |= uint64_t(2) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor for kind::f16 / kind::tf32 with fp32 accumulation.
// fmt: 0 = f16, 1 = bf16, 2 = tf32 (same for A and B).
__host__ __device__ constexpr uint32_t make_idesc(uint32_t fmt, int M, int N, int a_mn_major,
                                                  int b_mn_major) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (uint32_t(a_mn_major) << 15) |
         (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Per-warpgroup register budget (all 4 warps of an aligned warpgroup must
// execute it).  The sum over the CTA must not exceed the registers the CTA
// was launched with; the host checks that before launching.
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
// N registers per thread for the warpgroup, from the launch count L.
template <int N, int L>
__device__ __forceinline__ void regs_set() {
  if constexpr (N > L) regs_inc<N>();
  else if constexpr (N < L) regs_dec<N>();
}

// ------------------------------------------------------------------ math
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100 f32x2 instructions): one instruction for two
// lanes of work in the softmax inner loops.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 upk2(uint64_t r) {
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(r));
  return d;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a pair of floats on the FMA/ALU pipes: x = n + f with n = round(x)
// (via the 1.5·2^23 rounding constant), f in [-1/2, 1/2]; 2^f from a degree-3
// polynomial with minimal maximum relative error (1.0e-4; coefficients from
// gen_exp2_poly.py); 2^n added to the exponent field.  x is clamped at -125
// so that masked (-inf) arguments cannot wrap the exponent: they give
// ~2^-125, or exactly 0 with ZERO_BELOW.
template <bool ZERO_BELOW>
__device__ __forceinline__ float2 exp2_pair_fma(float2 x) {
  const bool z0 = x.x < -125.f, z1 = x.y < -125.f;
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const uint64_t magic = pk2(12582912.f, 12582912.f);
  const uint64_t t = fadd2(pk2(x.x, x.y), magic);
  const uint64_t n = fadd2(t, pk2(-12582912.f, -12582912.f));
  const uint64_t f = ffma2(n, pk2(-1.f, -1.f), pk2(x.x, x.y));
  uint64_t pp = ffma2(pk2(0.05500893f, 0.05500893f), f, pk2(0.24221095f, 0.24221095f));
  pp = ffma2(pp, f, pk2(0.6932829f, 0.6932829f));
  pp = ffma2(pp, f, pk2(1.f, 1.f));
  const float2 pv = upk2(pp), tv = upk2(t);
  float2 r = make_float2(__int_as_float(__float_as_int(pv.x) + (__float_as_int(tv.x) << 23)),
                         __int_as_float(__float_as_int(pv.y) + (__float_as_int(tv.y) << 23)));
  if constexpr (ZERO_BELOW) {
    if (z0) r.x = 0.f;
    if (z1) r.y = 0.f;
  }
  return r;
}

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <typename T>
struct ElemTraits;
template <>
struct ElemTraits<__nv_bfloat16> {
  static constexpr uint32_t fmt = 1;
  static constexpr bool tf32 = false;
  __device__ static uint32_t pack2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ static float2 unpack2(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
  }
  __device__ static __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
};
template <>
struct ElemTraits<__half> {
  static constexpr uint32_t fmt = 0;
  static constexpr bool tf32 = false;
  __device__ static uint32_t pack2(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ static float2 unpack2(uint32_t u) {
    __half2 v = *reinterpret_cast<__half2*>(&u);
    return __half22float2(v);
  }
  __device__ static __half from_float(float x) { return __float2half_rn(x); }
};
template <>
struct ElemTraits<float> {
  static constexpr uint32_t fmt = 2;
  static constexpr bool tf32 = true;
  __device__ static float from_float(float x) { return x; }
};

}  // namespace fa
