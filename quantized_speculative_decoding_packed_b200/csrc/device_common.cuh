// Device-side building blocks for sm_100a: shared-memory barriers with
// bounded waits, TMA tile loads, and the tcgen05 tensor-core / tensor-memory
// instructions.  Written from the public PTX ISA description of these
// instructions; every wait in this file gives up after a wall-clock limit
// instead of spinning forever.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

// Debug builds (-DQSPEC_TRACE) record, per warp, the last checkpoint reached
// into a host-mapped buffer that stays readable after a device fault, and
// check operand alignment in software (record and skip instead of faulting).
#ifdef QSPEC_TRACE
static __device__ unsigned int* g_qspec_trace = nullptr;
#define QSPEC_TRACE_AT(info)                                                            \
  do {                                                                                  \
    if (g_qspec_trace && (threadIdx.x & 31) == 0) {                                     \
      volatile unsigned int* t_ = g_qspec_trace + (blockIdx.x * 64u + (threadIdx.x >> 5)); \
      *t_ = (static_cast<unsigned>(__LINE__) << 16) | (static_cast<unsigned>(info) & 0xFFFFu); \
      __threadfence_system();                                                           \
    }                                                                                   \
  } while (0)
// Coarse phase events (global timer, ns, comparable across SMs and launches),
// appended to a log: {time, kind << 56 | launch << 32 | cta << 16 | event}.
// `kTraceKind` names the kernel and `trace_launch` (24 bits) the launch; each
// kernel defines both.
static __device__ unsigned long long* g_qspec_events = nullptr;
static __device__ unsigned int g_qspec_event_count = 0;
constexpr unsigned kQspecEventCap = 1u << 20;
#define QSPEC_PHASE(ev)                                                                 \
  do {                                                                                  \
    if (g_qspec_events) {                                                               \
      const unsigned i_ = atomicAdd(&g_qspec_event_count, 1u);                          \
      if (i_ < kQspecEventCap) {                                                        \
        g_qspec_events[2u * i_] = global_timer_ns();                                    \
        g_qspec_events[2u * i_ + 1u] = (static_cast<unsigned long long>(kTraceKind) << 56) | \
                                       (static_cast<unsigned long long>(trace_launch & 0xFFFFFFu) << 32) | \
                                       (static_cast<unsigned long long>(blockIdx.x) << 16) | (ev); \
      }                                                                                 \
    }                                                                                   \
  } while (0)
#define QSPEC_ALIGN_OK(addr, a)                                                          \
  ((static_cast<unsigned long long>(addr) % (a)) == 0 ||                                 \
   (g_qspec_trace && (g_qspec_trace[8191] = (0xA0000000u | __LINE__), __threadfence_system(), false)))
#else
#define QSPEC_TRACE_AT(info) \
  do {                       \
  } while (0)
#define QSPEC_ALIGN_OK(addr, a) true
#define QSPEC_PHASE(ev) \
  do {                  \
  } while (0)
#endif

namespace qspec {

// Device status bits written to the first word of a workspace.
constexpr uint32_t kDevTimeout = 1u;
constexpr uint32_t kDevBadInput = 2u;

// A wait that has not completed after this long is treated as a fault.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;   // 1 s

// Row stride (in fp16 scales) of the group-scale matrix ws: k/group rounded
// up to a multiple of 8, so that each row starts on a 16-byte boundary and
// the GEMM can fetch 8 groups x 128 rows of scales with one TMA copy.  The
// padding entries hold zeros.
__host__ __device__ constexpr int64_t scale_row_stride(int64_t groups_per_row) {
  return (groups_per_row + 7) / 8 * 8;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- cp.async
// 4-byte global -> shared copy that needs no register; bytes past `src_bytes`
// (0..4) are zero-filled and not read.  Both addresses 4-byte aligned.
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
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

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of a phase (try_wait may suspend the thread for a while).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or the hint (ns) expires, instead of spinning on shared
// memory and stealing issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Returns false (and
// raises the CTA-wide abort flag and the device status word) if the wait
// runs past kWaitLimitNs or another thread of the CTA has already aborted.
// The slow path lives out of line: the hot loops keep one try_wait and a
// branch, and their code stays compact in the instruction caches.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            uint32_t* status, uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t start = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;   // sleeps <= 0.2 ms
    if (*abort_flag) return false;
    if (global_timer_ns() - start > limit_ns) {
      *abort_flag = 1;
      if (status) atomicOr(status, kDevTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  if (__builtin_expect(mbar_try_wait(bar, parity), 1)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, status);
}

// Warp-level wait: every lane polls (one warp-wide instruction per poll, no
// divergent region -- a lane-0-only branch costs far more than the poll) and
// the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status));
}

// True in exactly one lane of a converged warp.
__device__ __forceinline__ bool elect_one_lane() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Short bounded wait used while draining copies on the abort path.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t start = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - start > kWaitLimitNs / 10) return;
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (tensor core / TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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

// Shared-memory matrix descriptor for a K-major operand stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);         // start address
  d |= static_cast<uint64_t>(1u) << 16;                       // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;               // stride byte offset: 8 rows
  d |= static_cast<uint64_t>(1u) << 46;                       // descriptor version
  d |= static_cast<uint64_t>(2u) << 61;                       // 128-byte swizzle
  return d;
}

// Instruction descriptors (dense, K-major A and B, M = 128).
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4)                  // D: s32
         | (1u << 7) | (1u << 10)   // A, B: signed 8-bit
         | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4)                  // D: f32
         | (1u << 7) | (1u << 10)   // A, B: bf16
         | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// Arrives on `bar` once all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns; thread i of the warp gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 16 consecutive 32-bit columns from registers: thread i of the warp
// writes lane (base lane + i).  Complete (for this thread) after tmem_st_wait.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D (tensor memory) (+)= A (tensor memory: lane = row, 32-bit columns along K,
// lowest K in the low bits) x B (shared-memory descriptor).
template <bool kInt8>
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  if constexpr (kInt8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
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

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

}  // namespace qspec
