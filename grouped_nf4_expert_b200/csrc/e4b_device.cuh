// Device-side building blocks for sm_100a: mbarriers with bounded waits,
// TMA tile loads, tcgen05 (TMEM allocation, UMMA, commit, TMEM loads),
// shared-memory matrix descriptors, and the NF4 block decoder.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/e4b.h"

namespace e4b {

// ----------------------------------------------------------------------------
// Device error word (first bytes of the caller's workspace).
// ----------------------------------------------------------------------------
struct DeviceError {
  int code;       // 0 or an e4b_status
  int site;       // which wait gave up (kernel-specific id)
  int block;      // blockIdx.x of the first CTA that gave up
  int pad[61];    // keeps the rest of the workspace 256-byte aligned
};
static_assert(sizeof(DeviceError) == 256, "error word block must be 256 bytes");

// Waits give up after this many nanoseconds by default (about a second).
constexpr long long kDefaultTimeoutNs = 2000000000LL;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded waits measure elapsed time with the SM cycle counter, which is
// cheap to read (the global timer is not).  A limit of T ns is taken as 2T
// cycles: at least T ns at any SM clock up to 2 GHz.
__device__ __forceinline__ long long wait_limit_cycles(long long timeout_ns) { return 2 * timeout_ns; }

__device__ __forceinline__ void record_error(DeviceError* err, int code, int site) {
  if (err != nullptr) {
    if (atomicCAS(&err->code, 0, code) == 0) {
      err->site = site;
      err->block = blockIdx.x;
    }
  }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but a thread whose phase has not completed may be
// suspended for up to `hint_ns` (it resumes as soon as the phase completes),
// so that waiting warps leave the issue slots to the working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Shared control block of a CTA: an abort flag that every bounded wait
// watches, so that when one role gives up the others stop too.
struct CtaControl {
  volatile int abort;
  int pad;
};

// Waits for the phase with `parity` of `bar` to complete.  Gives up (returns
// false) when `timeout_ns` elapses or another thread of the CTA has given up;
// a thread that gives up records E4B_ERR_DEVICE_TIMEOUT with `site`.
// Upper bound of one suspended wait; the abort flag and the timeout are
// checked between them.
constexpr uint32_t kWaitSleepNs = 20000;

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, CtaControl* ctl,
                                          DeviceError* err, long long timeout_ns, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long c0 = clock64(), limit = wait_limit_cycles(timeout_ns);
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if (ctl->abort) return false;
    if (clock64() - c0 > limit) {
      ctl->abort = 1;
      record_error(err, E4B_ERR_DEVICE_TIMEOUT, site);
      return false;
    }
  }
}

// Bounded wait for roles off the critical path (producers far ahead of their
// consumers, epilogues waiting for a whole tile): sleeps `sleep_ns` between
// polls so that the decoding warps get the issue slots.
__device__ __forceinline__ bool mbar_wait_lazy(uint64_t* bar, uint32_t parity, CtaControl* ctl, DeviceError* err,
                                               long long timeout_ns, int site, uint32_t sleep_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long c0 = clock64(), limit = wait_limit_cycles(timeout_ns);
  while (true) {
    __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (ctl->abort) return false;
    if (clock64() - c0 > limit) {
      ctl->abort = 1;
      record_error(err, E4B_ERR_DEVICE_TIMEOUT, site);
      return false;
    }
  }
}

// ----------------------------------------------------------------------------
// Thread-block clusters (pairs of CTAs sharing one 2-SM UMMA)
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of every CTA of the cluster: release this CTA's prior writes,
// acquire the peers'.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}


// Non-blocking signal to another CTA of the cluster: stores `v` to the word at
// `remote_word` and performs complete_tx(4 bytes) on the mbarrier at
// `remote_bar` (both cluster addresses from mapa_shared).  The complete_tx has
// release semantics at cluster scope, so this thread's prior writes (and those
// it has synchronised with) are visible to whoever observes the barrier phase,
// without the thread stalling as a release-arrive would.
__device__ __forceinline__ void st_async_signal(uint32_t remote_word, uint32_t remote_bar, uint32_t v) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(remote_word),
               "r"(v), "r"(remote_bar)
               : "memory");
}

// Arrival without release semantics: it orders none of this thread's earlier
// memory writes (use it when the receiver needs only the arrival, e.g. that
// this thread's TMEM reads have completed, and not this thread's global stores).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking phase tests (the thread is never suspended): issued ahead of
// time, their latency overlaps whatever the thread issues next.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_test_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on a barrier that receives arrivals from other CTAs of the
// cluster (cluster-scope acquire); otherwise as mbar_wait.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, CtaControl* ctl,
                                                  DeviceError* err, long long timeout_ns, int site) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long c0 = clock64(), limit = wait_limit_cycles(timeout_ns);
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (ctl->abort) return false;
    if (clock64() - c0 > limit) {
      ctl->abort = 1;
      record_error(err, E4B_ERR_DEVICE_TIMEOUT, site);
      return false;
    }
  }
}

// ----------------------------------------------------------------------------
// Proxy fences
// ----------------------------------------------------------------------------
// Makes this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core reads through UMMA descriptors).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), tile mode, no multicast.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// TMA bulk store of a shared-memory tile to global memory (bulk-group
// completion), its group commit, and the waits: `.read` returns once the
// source shared memory of all but the newest N groups has been read (the
// buffer may be rewritten); the plain form once their writes are performed.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 4-byte asynchronous global -> shared copy (cp.async), and an mbarrier
// arrival that fires once every cp.async this thread issued has landed.  The
// arrival is pre-counted in the barrier's expected count (.noinc).
__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// 16-byte variant: both addresses 16-byte aligned.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// 16-byte copy that writes zeros past the first `src_bytes` (0 or 16) bytes:
// with src_bytes == 0 nothing is read and the 16 destination bytes become 0.
__device__ __forceinline__ void cp_async_16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
// Groups of cp.async: commit this thread's copies issued so far as one
// group; wait until at most N of its groups are pending (the others' data is
// then visible to this thread).
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: TMEM allocation, UMMA, commit, TMEM -> registers
// ----------------------------------------------------------------------------
// Whole warp: allocates `ncols` TMEM columns (power of two >= 32) and writes
// the base address to `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
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

// True in exactly one active lane of the (converged) warp.  Issuing roles
// run their loops and waits with the whole warp, so that loop state stays
// warp-uniform, and put only the tcgen05 issue under this predicate.
__device__ __forceinline__ bool elect_one_sync() {
  uint32_t pred;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "elect.sync _|p, 0xffffffff;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(pred));
  return pred != 0;
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every UMMA this thread issued so far completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 2-SM variants: one warp in EACH CTA of the pair executes the allocation
// (same columns in both CTAs); the UMMA is issued by one thread of the even
// CTA and spans both CTAs' shared memory and TMEM; the commit arrives on the
// barrier at the same offset in every CTA of `cta_mask`.
__device__ __forceinline__ void tmem_alloc_2sm(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_2sm() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_2sm(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16_2sm(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit_2sm(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// Each thread of a warp reads 16 consecutive fp32 columns of its TMEM lane.
// The warp may only address lanes 32*(warp%4) .. +31.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Whole warp: 32 consecutive 32-bit columns of this thread's TMEM lane, the
// load and its wait in one statement (the registers are defined only after
// the wait, so no use can be scheduled between the two).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}


// Whole warp: each thread writes 32 consecutive 32-bit columns of its own
// TMEM lane (the warp's 32-lane quadrant), then waits for the writes.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulation.  A is
// M lanes x K/2 columns, two consecutive K elements per 32-bit column (the
// lower-index element in the low half).
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ----------------------------------------------------------------------------
// UMMA descriptors
// ----------------------------------------------------------------------------
// Swizzle modes of the shared-memory matrix descriptor (bits 61-63).
enum : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };

// Shared-memory matrix descriptor.  `lbo` and `sbo` are byte offsets:
//  K-major, swizzled: sbo = stride between 8-row groups; lbo unused.
//  MN-major, swizzled: lbo = stride between MN atoms (atom = swizzle width),
//                      sbo = stride between 8-row K groups.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t swz) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)(swz & 7u) << 61;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15)            // A major-ness
         | ((b_mn_major ? 1u : 0u) << 16)            // B major-ness
         | ((uint32_t)(N >> 3) << 17)                // N / 8
         | ((uint32_t)(M >> 4) << 24);               // M / 16
}

// Swizzle mode for a row of `row_bytes` (32, 64 or 128).
__host__ __device__ constexpr uint32_t swz_for_row_bytes(int row_bytes) {
  return row_bytes == 128 ? kSw128 : (row_bytes == 64 ? kSw64 : kSw32);
}

// ----------------------------------------------------------------------------
// bf16 helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (bits 0-15), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// ----------------------------------------------------------------------------
// NF4 decode.
// A weight is bf16_rn(float32(level[code]) * float32(absmax)).  For one block
// of 64 codes the 16 possible products are formed once (16 float32 multiplies,
// rounded to bf16), split into a low-byte plane and a high-byte plane, and
// every code then becomes a byte-permute lookup: exact by construction.
// ----------------------------------------------------------------------------
// The NF4 levels (QLoRA's NormalFloat-4 code book, as printed in its appendix).
__host__ __device__ __forceinline__ float nf4_level(int c) {
  constexpr float kLevels[16] = {-1.0f,
                                 -0.6961928009986877f,
                                 -0.5250730514526367f,
                                 -0.39491748809814453f,
                                 -0.28444138169288635f,
                                 -0.18477343022823334f,
                                 -0.09105003625154495f,
                                 0.0f,
                                 0.07958029955625534f,
                                 0.16093020141124725f,
                                 0.24611230194568634f,
                                 0.33791524171829224f,
                                 0.44070982933044434f,
                                 0.5626170039176941f,
                                 0.7229568362236023f,
                                 1.0f};
  return kLevels[c];
}

struct Nf4Planes {
  uint32_t lo[4];  // lo[g] = low bytes of the bf16 products of levels 4g..4g+3
  uint32_t hi[4];  // hi[g] = high bytes of the same
};

__device__ __forceinline__ Nf4Planes nf4_block_planes(float absmax) {
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = __fmul_rn(nf4_level(2 * i), absmax);
    const float b = __fmul_rn(nf4_level(2 * i + 1), absmax);
    pk[i] = pack_bf16x2(a, b);
  }
  Nf4Planes p;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    p.lo[g] = prmt(pk[2 * g], pk[2 * g + 1], 0x6420u);
    p.hi[g] = prmt(pk[2 * g], pk[2 * g + 1], 0x7531u);
  }
  return p;
}

// Powers of two the decoder multiplies by to move bits right.  They are read
// at run time so that the compiler keeps the multiplications, which run on
// the FMA pipe, instead of turning them into shifts on the integer ALU pipe
// that the table lookups below already fill.
struct Nf4Shift {
  uint32_t k16;  // 2^16: hi(x * k16) = x >> 16
  uint32_t k31;  // 2^31: hi(x * k31) = x >> 1
};
__device__ __forceinline__ Nf4Shift nf4_shift_consts() {
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  const uint32_t z = dyn >> 31;  // 0: no launch has 2 GiB of shared memory
  return {65536u >> z, 0x80000000u >> z};
}
__device__ __forceinline__ uint32_t mul_hi_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t mul_lo_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t mad_lo_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t mad_hi_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Decodes the 8 codes of one little-endian 32-bit word (bytes b0..b3,
// element 2m = high nibble of byte m) into 4 bf16x2 words holding elements
// (0,1), (2,3), (4,5), (6,7) -- lower element in the low half.
//
// Each byte plane is a 16-entry table split in two 8-byte halves: one byte
// permute looks up codes 0..7 (selector = the code), one looks up 8..15
// (selector = code ^ 8), a third picks per byte by bit 3 of the code, and two
// more interleave the low and high bytes into bf16 pairs.
__device__ __forceinline__ void nf4_decode_word(uint32_t w, const Nf4Planes& p, Nf4Shift k, uint32_t* out) {
  const uint32_t wx = w ^ 0x88888888u;                               // codes 8..15 -> 0..7
  const uint32_t wp = mad_hi_u32(w & 0x88888888u, k.k31, 0x32103210u);  // byte i from lookup 0..7 or 8..15
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    // Selector nibbles i = 0..3 hold the codes of elements 1, 0, 3, 2 of this half.
    const uint32_t s = (h == 0) ? w : mul_hi_u32(w, k.k16);
    const uint32_t s_hi = (h == 0) ? wx : mul_hi_u32(wx, k.k16);
    const uint32_t pick = (h == 0) ? wp : mul_hi_u32(wp, k.k16);
    const uint32_t xl = prmt(p.lo[0], p.lo[1], s);
    const uint32_t yl = prmt(p.lo[2], p.lo[3], s_hi);
    const uint32_t xh = prmt(p.hi[0], p.hi[1], s);
    const uint32_t yh = prmt(p.hi[2], p.hi[3], s_hi);
    const uint32_t fl = prmt(xl, yl, pick);
    const uint32_t fh = prmt(xh, yh, pick);
    out[2 * h] = prmt(fl, fh, 0x4051u);
    out[2 * h + 1] = prmt(fl, fh, 0x6273u);
  }
}

// Decodes one block: 32 bytes of codes (as 8 words) -> 64 bf16 (32 words).
__device__ __forceinline__ void nf4_decode_block(const uint32_t (&codes)[8], float absmax, uint32_t (&out)[32]) {
  const Nf4Planes p = nf4_block_planes(absmax);
  const Nf4Shift k = nf4_shift_consts();
#pragma unroll
  for (int i = 0; i < 8; ++i) nf4_decode_word(codes[i], p, k, &out[4 * i]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}


// silu and the logistic sigmoid with the fast exponential and the fast
// (reciprocal-based) division: a few ulp, far below bf16 output rounding.  For
// very negative g the denominator overflows to inf and both give 0.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }
__device__ __forceinline__ float sigmoid_f(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }

// Rounds a pointer into the dynamic shared-memory window up to a 1024-byte
// boundary (swizzle atoms).  The offset is added to the original pointer, so
// the compiler still knows the result addresses shared memory and emits
// shared (not generic) loads and stores through it.
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}

}  // namespace e4b
