// Shared device helpers for the sm_100a indexer kernels: mbarriers with bounded
// waits, TMA (tiled and 1-D bulk) copies, tcgen05 / TMEM wrappers, the UMMA
// shared-memory and instruction descriptors, and the library's fault word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace lsi {

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per device (the attribute is a per-device setting).  `done`
// holds one bit per device ordinal below 64, set after a successful call;
// threads that race on a device's first launch at worst set it twice.
inline cudaError_t smem_limit_once(std::atomic<uint64_t>& done, const void* fn, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// --------------------------------------------------------------------------
// fault word: set by a kernel whose bounded wait ran out; read by the host
// --------------------------------------------------------------------------
enum : int {
  FAULT_NONE = 0,
  FAULT_WAIT_TIMEOUT = 1,   // an mbarrier wait exceeded its time limit
  FAULT_BAD_INDEX = 2,      // a gathered row index was outside [0, N)
};

// The library is one translation unit (api.cu includes every kernel header),
// so this definition is unique.
__device__ int g_fault = 0;

// Wait limit for every mbarrier spin (nanoseconds of %globaltimer).  A normal
// launch finishes in milliseconds; the limit only ends a wait that cannot end.
#ifndef LSI_WAIT_LIMIT_NS
#define LSI_WAIT_LIMIT_NS 2000000000ull
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// --------------------------------------------------------------------------
// mbarrier
// --------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// The dynamic shared block rounded up to a 1024-byte boundary by pointer
// arithmetic on the shared array itself, so accesses through the result (and
// pointers derived from it) stay shared loads, stores and atomics rather than
// generic ones.
__device__ __forceinline__ uint8_t* smem_align1024(uint8_t* raw) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(raw));
  return raw + ((1024u - (a & 1023u)) & 1023u);
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

// The same test, letting the thread sleep up to suspend_ns while the phase is
// incomplete (it wakes as soon as the phase completes): a waiting warp then
// takes no issue slots from the warps that do the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}
constexpr uint32_t kWaitSuspendNs = 20000;

// Bounded wait for the phase with the given parity.  Returns false (and sets
// the CTA abort flag and the global fault word) when the limit runs out or
// another role of the CTA has already aborted.
// kSleep = false keeps the plain test (the indexer scorer, whose short
// units measured a little faster with it).
template <bool kSleep = true>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (kSleep ? mbar_try_wait_sleep(bar, parity, kWaitSuspendNs) : mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > LSI_WAIT_LIMIT_NS) {
      *abort_flag = 1;
      atomicOr(&g_fault, FAULT_WAIT_TIMEOUT);
      return false;
    }
  }
}

// Drain wait: bounded by time only (used after an abort).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, kWaitSuspendNs)) {
    if (globaltimer_ns() - t0 > LSI_WAIT_LIMIT_NS) {
      atomicOr(&g_fault, FAULT_WAIT_TIMEOUT);
      return;
    }
  }
}

// Warp-uniform bounded wait: lane 0 waits, every lane gets its verdict, so
// warp-collective instructions after the wait never see a partial warp.
template <bool kSleep = true>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait<kSleep>(bar, parity, abort_flag);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// --------------------------------------------------------------------------
// TMA
// --------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load; x is the innermost coordinate (elements), y the row.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 1-D bulk load of `bytes` (multiple of 16, both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (tcgen05).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------------------------
// tcgen05 / TMEM
// --------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
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

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with e4m3 A and B, fp32 D (kind::f8f6f4,
// K = 32 per instruction).
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same MMA issued by a converged warp: every lane executes the call (so
// the descriptors stay warp-uniform) and one elected lane performs it.  A lone
// lane issuing under divergent control flow takes several times longer per MMA.
__device__ __forceinline__ void umma_f16_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Commit from a converged warp: the elected lane (the one that issued the
// MMAs through umma_f16_warp) arrives on `bar` when they are done.
__device__ __forceinline__ void umma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, f16 inputs: A is read from tensor memory
// (row i in lane i, two 16-bit elements per 32-bit column).  Issued by a
// converged warp through one elected lane, like umma_f16_warp.
__device__ __forceinline__ void umma_f16_tmem_a_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                     uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit words from registers into TMEM: thread i of
// the warp writes lane (base+i), columns col..col+31.
__device__ __forceinline__ void tmem_st_32x32(uint32_t taddr, const uint32_t (&r)[32]) {
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

// Wait until this thread's tcgen05.st writes are done.
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 4-byte asynchronous global -> shared copy (no register round trip).
__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// 16-byte asynchronous global -> shared copy, bypassing L1 (both addresses
// 16-byte aligned).
__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Close the group of cp.async copies this thread issued since the last one.
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's committed cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The mbarrier gets one more pending arrival now, and receives it once every
// cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive on `bar` once every tcgen05 op issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 columns of fp32: thread i of the warp receives lane (base+i),
// columns col..col+31.
__device__ __forceinline__ void tmem_ld_32x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  // The wait is in the same asm statement as the load so that no consumer of
  // the registers can be scheduled between them.
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// The same load without the wait; tmem_wait_ld() must follow before any use of
// r.  The wait names the registers as read-write operands, so the compiler
// cannot move a consumer of r above it.
__device__ __forceinline__ void tmem_ld_32x32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
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

__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                 "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                 "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored with the
// 128-byte swizzle: rows of 128 B (64 bf16), 8-row groups 1024 B apart.
// Bits: start>>4 [0,14), LBO>>4 [16,30) (unused for this layout, 1),
// SBO>>4 [32,46), descriptor version 1 [46,48), layout 2 = SWIZZLE_128B [61,64).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  desc |= static_cast<uint64_t>(1) << 16;
  desc |= static_cast<uint64_t>(1024 >> 4) << 32;
  desc |= static_cast<uint64_t>(1) << 46;
  desc |= static_cast<uint64_t>(2) << 61;
  return desc;
}

// Shared-memory matrix descriptor for an MN-major operand under the 128-byte
// swizzle: atoms of 64 MN-elements (128 B, 16-bit types) x 8 K-rows, rows
// 128 B apart inside an atom (the same bytes as a K-major SW128 staging of
// the K-rows); `lbo` = bytes between atoms along MN, 1024 between atoms
// along K.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  desc |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  desc |= static_cast<uint64_t>(1024 >> 4) << 32;
  desc |= static_cast<uint64_t>(1) << 46;
  desc |= static_cast<uint64_t>(2) << 61;
  return desc;
}

// Instruction descriptor, kind::f16: A = B = bf16, D = f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                  // D format f32
         | (1u << 7)                                // A format bf16
         | (1u << 10)                               // B format bf16
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// Instruction descriptor, kind::f16: A = B = f16, D = f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                                  // D format f32 (A, B format 0 = f16)
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4: A = B = e4m3 (format 0), D = f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                                  // D format f32 (A, B format 0 = e4m3)
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// 2^e as a float, exactly, for -126 <= e <= 127 (clamped).
__device__ __forceinline__ float exp2i(int e) {
  e = e < -126 ? -126 : (e > 127 ? 127 : e);
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// Shift that brings a head's largest |q| into [2^14, 2^15): q * 2^s is then
// an fp16 value without overflow, and keeps full fp16 precision for every
// element within 2^28 of that largest one.  0 for an all-zero or non-finite head.
__device__ __forceinline__ int f16_head_shift(float maxabs) {
  const uint32_t bits = __float_as_uint(maxabs);
  const int e = static_cast<int>((bits >> 23) & 0xffu);
  if (maxabs == 0.f || e == 0xff) return 0;
  const int sh = 14 - (e - 127);
  return sh > 126 ? 126 : sh;  // keeps 2^s and 2^-s both normal floats
}

// --------------------------------------------------------------------------
// 8-bit keys and the query tile in fp16
// --------------------------------------------------------------------------
// 4 signed bytes -> 4 fp16, exactly: the half pattern 0x6400 | (v + 128) is
// 1024 + v + 128, and subtracting 1152 leaves v.
__device__ __forceinline__ void i8x4_to_f16x4(uint32_t x, uint32_t& lo, uint32_t& hi) {
  const uint32_t y = x ^ 0x80808080u;
  const uint32_t t0 = __byte_perm(y, 0x64646464u, 0x4140);
  const uint32_t t1 = __byte_perm(y, 0x64646464u, 0x4342);
  const uint32_t m = 0x64806480u;  // 1152.0 in each half
  __half2 r0 = __hsub2(*reinterpret_cast<const __half2*>(&t0), *reinterpret_cast<const __half2*>(&m));
  __half2 r1 = __hsub2(*reinterpret_cast<const __half2*>(&t1), *reinterpret_cast<const __half2*>(&m));
  lo = *reinterpret_cast<uint32_t*>(&r0);
  hi = *reinterpret_cast<uint32_t*>(&r1);
}

// 4 e4m3 codes -> 4 fp16, exactly (one conversion per pair).
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

// The query tile of one problem (32 heads x 128, K-major, 128-byte swizzle) in
// shared memory: lane h rescales head h by 2^s_h and rounds it to fp16 in
// place (the swizzle only permutes 16-byte chunks inside a head's row).
__device__ __forceinline__ void q_tile_to_f16(uint8_t* tile, int half_bytes, int lane) {
  float mx = 0.f;
#pragma unroll
  for (int pnl = 0; pnl < 2; ++pnl) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(tile + pnl * half_bytes + lane * 128 + c * 16);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mx = fmaxf(mx, fabsf(__uint_as_float(w4[i] << 16)));
        mx = fmaxf(mx, fabsf(__uint_as_float(w4[i] & 0xffff0000u)));
      }
    }
  }
  const float sc = exp2i(f16_head_shift(mx));
#pragma unroll
  for (int pnl = 0; pnl < 2; ++pnl) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4* pp = reinterpret_cast<uint4*>(tile + pnl * half_bytes + lane * 128 + c * 16);
      uint4 v = *pp;
      uint32_t* w4 = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 h = __floats2half2_rn(__uint_as_float(w4[i] << 16) * sc,
                                            __uint_as_float(w4[i] & 0xffff0000u) * sc);
        w4[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *pp = v;
    }
  }
}

// The same head shift, derived from the bf16 query rows in global memory.
__device__ __forceinline__ int q_head_shift_global(const uint16_t* row) {
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  float mx = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint4 v = __ldg(r4 + c);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx = fmaxf(mx, fabsf(__uint_as_float(w4[i] << 16)));
      mx = fmaxf(mx, fabsf(__uint_as_float(w4[i] & 0xffff0000u)));
    }
  }
  return f16_head_shift(mx);
}

// --------------------------------------------------------------------------
// small helpers
// --------------------------------------------------------------------------

// Position of a persistent CTA in its contiguous run of work units, ordered
// problem (b), then query group (g), then key tile; advanced without division.
struct UnitPos {
  int tile, g, b;
  __device__ __forceinline__ void init(long long u0, int NT, int G) {
    tile = static_cast<int>(u0 % NT);
    const long long bg = u0 / NT;
    g = static_cast<int>(bg % G);
    b = static_cast<int>(bg / G);
  }
  __device__ __forceinline__ void next(int NT, int G) {
    if (++tile == NT) {
      tile = 0;
      if (++g == G) {
        g = 0;
        ++b;
      }
    }
  }
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// Two fp32 lanes packed in one 64-bit register pair (the operand form of the
// packed fp32x2 arithmetic of sm_100a).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// acc += (x + |x|) * w on a pair of lanes.  x + |x| is 2 * max(x, 0) exactly
// (one FADD with an absolute-value operand, on the FMA pipe); the factor 2 is
// taken out once per key at the end (a power of two, so nothing is lost).
// The two ReLU results are produced straight into the register pair the
// packed FMA reads, and the accumulator and weights stay packed throughout,
// so no register moves are needed between the steps.
__device__ __forceinline__ void relu2_fma2(uint64_t& acc, uint32_t x0, uint32_t x1, uint64_t w) {
  asm("{\n\t.reg .f32 a0, a1, t0, t1;\n\t.reg .b64 ra;\n\t"
      "mov.b32 t0, %1;\n\t"
      "mov.b32 t1, %2;\n\t"
      "abs.f32 a0, t0;\n\t"
      "abs.f32 a1, t1;\n\t"
      "add.f32 a0, t0, a0;\n\t"
      "add.f32 a1, t1, a1;\n\t"
      "mov.b64 ra, {a0, a1};\n\t"
      "fma.rn.f32x2 %0, ra, %3, %0;\n\t}"
      : "+l"(acc)
      : "r"(x0), "r"(x1), "l"(w));
}

// Sum of four packed partial sums, halved (see relu2_fma2).
__device__ __forceinline__ float finish_pairs(const uint64_t (&acc)[4]) {
  uint64_t s01, s23, s;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(s01) : "l"(acc[0]), "l"(acc[1]));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(s23) : "l"(acc[2]), "l"(acc[3]));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(s) : "l"(s01), "l"(s23));
  float lo, hi;
  unpack_f32x2(s, lo, hi);
  return 0.5f * (lo + hi);
}

// The 32 head weights of one query as 16 packed pairs.
struct HeadWeights {
  uint64_t v[16];
  __device__ __forceinline__ void load(const float* __restrict__ w) {  // 16-byte aligned
    const ulonglong2* w2 = reinterpret_cast<const ulonglong2*>(w);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const ulonglong2 t = __ldg(w2 + i);
      v[2 * i] = t.x;
      v[2 * i + 1] = t.y;
    }
  }
};

// Weighted-ReLU head reduction of one key's 32 head dot products r (fp32 bit
// patterns, one TMEM row):  sum_h w[h] * max(0, r[h]),  with four independent
// packed partial sums (a single running sum would serialise 16 dependent FMAs).
__device__ __forceinline__ float head_reduce_w(const uint32_t (&r)[32], const HeadWeights& w) {
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int h = 0; h < 32; h += 2) relu2_fma2(acc[(h >> 1) & 3], r[h], r[h + 1], w.v[h >> 1]);
  return finish_pairs(acc);
}

// The same with the weights read from global memory (16-byte aligned).
__device__ __forceinline__ float head_reduce(const uint32_t (&r)[32], const float* __restrict__ w) {
  HeadWeights hw;
  hw.load(w);
  return head_reduce_w(r, hw);
}

// sum_h w[h] * max(0, sc * v[h]) for a per-key scale sc of either sign:
// = |sc| * sum_h w[h] * max(0, sign(sc) * v[h]).  The sign is uniform across a
// warp in practice (scales are magnitudes), so the branch does not diverge.
__device__ __forceinline__ float head_reduce_scaled(const uint32_t (&r)[32], const HeadWeights& w, float sc) {
  float base;
  if (sc >= 0.f) {
    base = head_reduce_w(r, w);
  } else {
    uint32_t neg[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) neg[i] = r[i] ^ 0x80000000u;
    base = head_reduce_w(neg, w);
  }
  return fabsf(sc) * base;
}

// Order-preserving 32-bit code of a score: larger score -> larger code;
// -0.0 and +0.0 share a code; every NaN maps to 0, below -inf.
__device__ __forceinline__ uint32_t order_code(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Selection histograms count the top 11 bits of the order code (2048 bins).
constexpr int kHistBits = 11;
constexpr int kHistBins = 1 << kHistBits;
__device__ __forceinline__ uint32_t hist_bin(uint32_t code) { return code >> (32 - kHistBits); }

// Named barrier over the `count` threads of a role (id 0 is __syncthreads).
__device__ __forceinline__ void role_barrier(int id, int count) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Shared-memory histogram of one row's scores, flushed into the row's global
// histogram by the threads of a role when the row changes or the CTA ends.
__device__ __forceinline__ void flush_hist(uint32_t* shist, uint32_t* ghist_row, int tid_in_role, int role_threads) {
  for (int i = tid_in_role; i < kHistBins; i += role_threads) {
    const uint32_t v = shist[i];
    if (v) {
      atomicAdd(ghist_row + i, v);
      shist[i] = 0;
    }
  }
}

}  // namespace lsi
