// qg_device.cuh -- sm_100a device helpers shared by the library's kernels:
// bounded mbarrier waits that report through a status word instead of
// trapping, TMA tile loads, and the tcgen05 (5th-generation tensor core)
// instructions: TMEM allocation, MMA issue/commit, TMEM loads/stores.
//
// Inline PTX only; no CUTLASS/CuTe types.  Descriptor bit layouts follow the
// PTX ISA for tcgen05 (shared-memory matrix descriptor and instruction
// descriptor of kind::i8 / kind::f16).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <type_traits>

#include "../../include/qg.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libqg kernels are written for sm_100a only"
#endif

namespace qg {

// ---------------------------------------------------------------------------
// Device status word.  Each translation unit owns one (a file-scope
// __device__ word); the first failing site records
// (code | site << 8 | block << 24).
// ---------------------------------------------------------------------------
enum DevErr : uint32_t { kDevOk = 0, kDevTimeout = 1, kDevBadArg = 2, kDevDebugCheck = 3 };

// Device-side checks of the debug library (built with QG_DEBUG): dcheck(ok,
// status, site) records kDevDebugCheck with the site in the kernel's status
// word when `ok` is false and returns false, so the caller skips the access;
// without QG_DEBUG it is the constant true and the check compiles away.
#ifdef QG_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool dcheck(bool ok, unsigned long long* status, uint32_t site) {
  if (!kDebugChecks) return true;
  if (!ok)
    atomicCAS(status, 0ull,
              (unsigned long long)kDevDebugCheck | ((unsigned long long)site << 8) |
                  ((unsigned long long)(blockIdx.x + gridDim.x * blockIdx.y) << 24));
  return ok;
}
// The TMA rule for a tiled copy: the innermost coordinate times the element
// size is a multiple of 16 bytes (nothing else checks it before the copy runs).
__device__ __forceinline__ bool tma_x_ok(int32_t x, int esize) { return ((int64_t)x * esize) % 16 == 0; }
// dcheck for a condition a whole warp must agree on (it guards .aligned
// tensor-memory loads): false on every lane if it fails on one.  Compiled away
// without QG_DEBUG.
__device__ __forceinline__ bool dcheck_warp(bool ok, unsigned long long* status, uint32_t site) {
  if constexpr (!kDebugChecks) return true;
  return __all_sync(0xffffffffu, dcheck(ok, status, site));
}
// A TMA copy's coordinates and shared-memory address under the debug checks:
// the innermost coordinate x (elements of esize bytes) on a 16-byte boundary,
// and the shared-memory end of the copy 16-byte aligned (smem 0: none).
__device__ __forceinline__ bool tma_ok(uint32_t smem, int32_t x, int esize, unsigned long long* status,
                                       uint32_t site) {
  return dcheck(tma_x_ok(x, esize) && (smem & 15u) == 0, status, site);
}
// [off, off + bytes) inside an area of `size` bytes
__device__ __forceinline__ bool in_area(int64_t off, int64_t bytes, int64_t size) {
  return off >= 0 && bytes >= 0 && off + bytes <= size;
}

// A wait gives up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

// One poll.  A thread whose phase is not complete is suspended until the
// phase completes or the suspend-time hint (ns) expires, instead of spinning
// and taking issue slots from the warps doing the work.
constexpr uint32_t kSuspendHintNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// One poll with acquire at cluster scope: for barriers that other CTAs of the
// cluster arrive on (mbar_arrive_remote), so their prior writes are visible.
// No suspend-time hint: the implementation's own (short) limit applies.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false
// (and records a timeout in *status) if that takes longer than limit_ns
// (kWaitLimitNs unless a test shortens it).  The timer is read only once per
// 64 unsuccessful polls, so a wait that completes promptly never touches it.
template <bool kCluster>
__device__ __forceinline__ bool mbar_wait_scoped(uint32_t bar, uint32_t parity, unsigned long long* status,
                                                 uint32_t site, uint64_t limit_ns = kWaitLimitNs) {
  auto poll = [&]() { return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
#pragma unroll 1
  for (int i = 0; i < 64; ++i)
    if (poll()) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (poll()) return true;
    if (globaltimer() - t0 > limit_ns) {
      unsigned long long code =
          (unsigned long long)kDevTimeout | ((unsigned long long)site << 8) |
          ((unsigned long long)(blockIdx.x + gridDim.x * blockIdx.y) << 24);
      atomicCAS(status, 0ull, code);
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned long long* status,
                                          uint32_t site, uint64_t limit_ns = kWaitLimitNs) {
  return mbar_wait_scoped<false>(bar, parity, status, site, limit_ns);
}

// mbar_wait for a barrier that other CTAs of the cluster arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, unsigned long long* status,
                                                  uint32_t site) {
  return mbar_wait_scoped<true>(bar, parity, status, site);
}

// ---------------------------------------------------------------------------
// TMA (tiled, 2-D, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Load the box at coordinates (c0 = innermost, c1) into shared memory; the
// transfer completes on mbarrier `bar` (complete_tx of the box's bytes).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Same, with an L2 eviction-priority policy (createpolicy) for streamed data.
// TMA load into this CTA's shared memory for a cta_group::2 pair: the copy's
// completion (complete_tx of its bytes) is signalled on `bar`, which may be an
// mbarrier of the peer CTA (its address from mapa_shared).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                      int32_t c0, int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int32_t c0, int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
      : "memory");
}

// Fetch the box at (c0, c1) from global memory into L2 only (no shared-memory
// destination, nothing to wait for).  A prefetch never makes a later load
// return stale data -- L2 is the point of coherence for every writer -- so it
// may be issued before griddepcontrol.wait.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}

// Store the box at (c0 = innermost, c1) from shared memory to global memory
// (bulk-group completion; rows/columns outside the tensor are not written).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}

// Copy `bytes` (a multiple of 16) from this CTA's shared memory to the shared
// memory of a CTA of the cluster (dst and bar from mapa_shared); the copy
// completes on that CTA's mbarrier `bar` (complete_tx of the bytes).
__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "r"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until every committed bulk store of this thread has completed (its
// global writes done, its shared-memory source free).
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Make generic-proxy shared-memory writes visible to the async proxy
// (tensor core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory
// ---------------------------------------------------------------------------
// Whole warp: allocate `ncols` TMEM columns (power of two >= 32); the base
// address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
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

// CTA-pair forms (cta_group::2): the same warp (same warp index) of both CTAs
// of a two-CTA cluster issues them with the same shared-memory slot; the
// allocation covers the same columns in both CTAs' tensor memory.  A kernel
// uses either these or the single-CTA forms above, never both.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor for a K-major operand tile stored in the
// 128-byte swizzle layout that TMA writes with CU_TENSOR_MAP_SWIZZLE_128B:
// rows of 128 bytes, 8-row atoms of 1024 bytes (stride byte offset), 16-byte
// chunks XOR-ed with (row % 8).  The tile base must be 1024-byte aligned.
//   bits  0-13 start address >> 4     bits 16-29 leading byte offset >> 4 (unused: 1)
//   bits 32-45 stride byte offset >> 4  bits 46-47 version (1 on sm_100)
//   bits 49-51 base offset (0)        bits 61-63 layout (2 = SWIZZLE_128B)
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor (32 bits), dense, K-major A and B:
//   bits 4-5 D format (0 f16, 1 f32, 2 s32); bits 7-9 A format; bits 10-12 B
//   format (kind::i8: 0 unsigned, 1 signed; kind::f16: 0 f16, 1 bf16);
//   bit 15/16 A/B major (0 = K); bits 17-22 N >> 3; bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_i8_s32(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// tcgen05: MMA issue (one thread) and commit
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// A operand from tensor memory (lane m = row m of A, K packed two fp16 per
// 32-bit column, even k in the low half), B from a shared-memory descriptor.
// kind::i8 with the A operand in tensor memory (lane m = row m of A, four int8
// of consecutive k per 32-bit column, lowest k in the lowest byte)
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// CTA-pair MMA, issued by one thread of the even CTA of the pair: D (M = 256
// rows, half in each CTA's tensor memory at the same address) += A (128 rows
// from each CTA's shared memory) x B (N/2 rows from each CTA's shared memory);
// the descriptors name the same shared-memory offsets in both CTAs.
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Pair form of mma_commit: when every pair MMA issued by this thread has
// completed, arrive once on the barrier at shared-memory offset `bar` of each
// CTA in `cta_mask` (bit r = cluster rank r).
__device__ __forceinline__ void mma_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}

// Arrive on an mbarrier of another CTA of the cluster (`remote` from
// mapa_shared) without release semantics.  For signals whose payload is
// already complete when the arrive is issued: a tensor-memory load finished
// with tcgen05.wait::ld, or a TMA copy whose completion this thread has
// observed on its own barrier.  (A release at cluster scope measured ~0.6 us
// per arrive on B200 while this CTA's TMA copies were in flight.)
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

// Arrive once on `bar` when every MMA previously issued by this thread has
// completed (and its shared-memory operands may be overwritten).
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM -> registers.  32x32b shape: thread t of the warp reads lane
// (lane_base + t), consecutive 32-bit columns starting at the address column.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// 32 consecutive columns in one instruction (32 registers).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
}

// Registers -> TMEM, same 32x32b shape: thread t writes lane (lane_base + t),
// 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library is launched with
// programmatic stream serialization allowed; it calls pdl_wait() before its
// first global-memory access (which waits for the preceding grid to complete
// and its writes to become visible) and pdl_trigger() once its setup is done,
// so the next kernel's launch and setup overlap this one.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// CTA barriers for warp-specialized kernels.  __syncthreads() is the .aligned
// barrier, which requires every thread of the CTA to reach the same barrier
// instruction convergently; in warp-specialized code (one lane of a warp in a
// role loop while its other lanes wait) that does not hold, and the aligned
// barrier was observed on B200 to release warps before all threads arrived.
// The non-aligned form counts individual threads, so it waits for all of them.
__device__ __forceinline__ void cta_barrier_all() { asm volatile("barrier.sync 0;" ::: "memory"); }

// Named (non-aligned) barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Activation applied to an fp32 epilogue value before the output rounding
// (page "INT4/FP16混合精度GEMM" §8, fused linear_gelu).  GELU is taken from its
// definition, v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)).
__device__ __forceinline__ float gelu_f32(float v) { return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f)); }

__device__ __forceinline__ float apply_act(float v, int act) { return act == QG_ACT_GELU ? gelu_f32(v) : v; }

// The activation as a compile-time choice: f(std::true_type) for GELU, else
// f(std::false_type), so that a loop written inside f carries no GELU code in
// its plain variant (a runtime test inside a loop may be compiled as
// predicated-off instructions that still issue for every element).
template <class F>
__device__ __forceinline__ void dispatch_act(int act, F&& f) {
  if (act == QG_ACT_GELU) f(std::true_type{});
  else f(std::false_type{});
}

template <bool kGelu, int NV>
__device__ __forceinline__ void apply_act_c(float (&v)[NV]) {
  if constexpr (kGelu) {
#pragma unroll
    for (int j = 0; j < NV; ++j) v[j] = gelu_f32(v[j]);
  }
}

// Arrive on a named barrier without waiting (the waiting side uses
// named_barrier with the same id and count).
__device__ __forceinline__ void named_barrier_arrive(uint32_t id, uint32_t count) {
  asm volatile("barrier.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------
// GPU-scope release/acquire (cross-CTA hand-off through global memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---------------------------------------------------------------------------
// Thread-block cluster (distributed shared memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Split cluster barrier: arrive early (relaxed), wait later.  A CTA may touch
// another CTA's shared memory only after every CTA of the cluster has
// started, which the first arrive/wait pair guarantees.
// (Not .aligned: threads of a warp may reach them at different points.)
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}

// Split cluster barrier arrive that also publishes this thread's prior
// writes (to be read by other CTAs after their matching wait).
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void st_dsmem_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                            uint32_t d) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Asynchronous store of 16 bytes into the shared memory of a CTA of the
// cluster (addr from mapa_shared); it completes on that CTA's mbarrier `bar`
// (also from mapa_shared) as complete_tx of 16 bytes, so the receiver waits on
// its own barrier instead of a cluster-wide barrier.
__device__ __forceinline__ void st_async_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                            uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1,%2,%3,%4}, [%5];" ::"r"(addr),
               "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar)
               : "memory");
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ int4 ld_dsmem_v4(uint32_t addr) {
  int4 v;
  asm volatile("ld.shared::cluster.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

}  // namespace qg
