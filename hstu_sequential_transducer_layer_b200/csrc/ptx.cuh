// ptx.cuh — thin inline-PTX wrappers for sm_100a: mbarriers with bounded
// waits, TMA tile loads, tcgen05 (TMEM alloc, MMA, commit, loads) and the
// shared-memory matrix descriptors the MMAs read.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"

#define DEVI __device__ __forceinline__

namespace hstu {

// A wait that has not completed after this many microseconds (by default;
// a kernel may set a shorter limit in its AbortState) gives up, sets the
// device status to HSTU_ERR_TIMEOUT and lets the kernel wind down.
constexpr uint32_t kWaitLimitUs = kDefaultWaitLimitUs;

DEVI uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-space loads and stores by 32-bit shared-window address: no generic
// address resolution, and loads are tracked with the short (shared-memory)
// latency.  The "memory" clobber keeps them ordered with the surrounding
// memory operations and barriers.
DEVI float lds_f32(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
DEVI uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "r"(addr)
      : "memory");
  return v;
}
DEVI void sts_u128(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

DEVI uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
DEVI void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
DEVI void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
DEVI void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
DEVI void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// A thread whose phase has not completed sleeps in the hardware until it
// does, for at most the suspend-time hint (20 us), instead of spinning: a
// waiting warp takes no issue slots from the working ones.
DEVI bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}

// Per-CTA failure state shared by all roles of a kernel.
struct AbortState {
  int flag;           // set once any wait of this CTA gave up
  uint32_t limit_us;  // how long one wait may take before it gives up
};

DEVI void raise_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Single-thread bounded wait.  Returns false if it gave up (or another role
// of this CTA already did).
DEVI bool mbar_wait(uint64_t* bar, uint32_t parity, AbortState* ab, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*((volatile int*)&ab->flag)) return false;
      if (global_timer_ns() - t0 > 1000ull * ab->limit_us) {
        *((volatile int*)&ab->flag) = 1;
        raise_status(status, HSTU_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: every lane polls; the outcome is the same for
// all 32 lanes (the caller's warp must be converged).
DEVI bool mbar_wait_warp(uint64_t* bar, uint32_t parity, AbortState* ab, int* status) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if ((it & 31u) == 0) {
      int give_up = 0;
      if (threadIdx.x % 32 == 0) {
        if (*((volatile int*)&ab->flag)) give_up = 1;
        else if (global_timer_ns() - t0 > 1000ull * ab->limit_us) {
          *((volatile int*)&ab->flag) = 1;
          raise_status(status, HSTU_ERR_TIMEOUT);
          give_up = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
    }
  }
}

// ---------------------------------------------------------------- TMA
DEVI void tma_prefetch_desc(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

// 2-D tiled load into shared memory; completion is counted in bytes on `bar`.
// x (innermost) must be a multiple of 8 elements for 16-bit data.
DEVI void tma_load_2d(void* smem_dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled store from shared memory (bulk async-group completion).
// Brings one box of a 2-D tensor into L2 (no shared-memory destination, no
// completion to wait for).
DEVI void tma_prefetch_l2_2d(const CUtensorMap* tm, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(x), "r"(y)
               : "memory");
}
DEVI void tma_store_2d(const CUtensorMap* tm, int x, int y, const void* smem_src) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(x), "r"(y), "r"(smem_u32(smem_src))
      : "memory");
}
DEVI void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed bulk groups still read
// shared memory.
template <int N>
DEVI void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
DEVI void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core reads of operands written with st.shared).
DEVI void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
// The warp-collective tcgen05 instructions (.sync.aligned: alloc, dealloc,
// ld, st, wait) must be executed by all 32 lanes converged; each wrapper
// reconverges the warp first, since callers reach them after lane-dependent
// branches (ragged rows, lane-0 work).
DEVI void tmem_alloc(uint32_t* slot, uint32_t ncols) {  // whole warp
  __syncwarp();
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
DEVI void tmem_relinquish() {  // whole warp
  __syncwarp();
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
DEVI void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  __syncwarp();
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
DEVI void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DEVI void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on `bar` once every tcgen05 operation this thread issued so far
// has completed.
DEVI void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; fp16 or bf16 inputs (per the
// instruction descriptor), fp32 accumulator.
DEVI void tc_mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f16: A and B both fp16 (f16 = 1) or both
// bf16 (f16 = 0), fp32 D, M x N tile.  a_mn / b_mn select MN-major
// (transposed) operands.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, int a_mn, int b_mn, int f16) {
  return (1u << 4)                            // D format: f32
         | ((f16 ? 0u : 1u) << 7)             // A format: 0 f16, 1 bf16
         | ((f16 ? 0u : 1u) << 10)            // B format
         | ((uint32_t)a_mn << 15)             // A major
         | ((uint32_t)b_mn << 16)             // B major
         | ((uint32_t)(N >> 3) << 17)         // N / 8
         | ((uint32_t)(M >> 4) << 24);        // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle.  saddr: shared-window
// byte address of the first element (tile bases 1024-byte aligned); lbo/sbo
// in bytes.  K-major: sbo = distance between 8-row groups (lbo unused).
// MN-major: lbo = distance between 64-element MN chunks, sbo = distance
// between 8-row K groups.
DEVI uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version of tcgen05
  d |= 2ull << 61;  // SWIZZLE_128B
  return d;
}

// D[tmem] (+)= A[tmem] * B[smem desc]: A (M x K, one row per TMEM lane, two
// 16-bit K elements per 32-bit column, even K in the low half) read from TMEM.
DEVI void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---------------------------------------------------------------- CTA pairs
// A cluster of two CTAs on two SMs sharing one 256-row MMA (cta_group::2):
// rank 0 issues the MMAs, which read A's rows 0..127 and B's first half from
// its own shared memory and the rest from its peer's, at the same offsets, and
// write rows 0..127 of D to its tensor memory and rows 128..255 to the peer's.
// Every tcgen05 allocation, MMA and commit of such a kernel is of cta_group::2.
DEVI uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the variable at shared::cta address `addr`
// in the cluster's CTA `rank`.
DEVI uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// All threads of both CTAs (converged): earlier writes, shared-memory
// barrier initialisation included, are visible to the peer afterwards.
DEVI void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
DEVI void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// Arrive on an mbarrier of either CTA of the cluster.  CTA-scope release:
// what the waiter needs ordered is this thread's tensor-memory reads, which
// tcgen05.wait::ld has completed and tcgen05.fence::before_thread_sync orders
// before the arrive; a cluster-scope release would add a memory barrier that
// waits for all of the thread's outstanding memory operations.
DEVI void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Bounded wait, single thread, with cluster-scope acquire (arrivals that come
// from the peer CTA's threads).
DEVI bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
DEVI bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, AbortState* ab, int* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*((volatile int*)&ab->flag)) return false;
      if (global_timer_ns() - t0 > 1000ull * ab->limit_us) {
        *((volatile int*)&ab->flag) = 1;
        raise_status(status, HSTU_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
// 2-D tiled load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (`bar`: shared::cluster address).
DEVI void tma_load_2d_pair(void* smem_dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// One warp of EACH CTA of the pair executes these, converged; the pair's
// allocation sits at the same column in both CTAs' tensor memory.
DEVI void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  __syncwarp();
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
DEVI void tmem_relinquish_pair() {
  __syncwarp();
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
DEVI void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  __syncwarp();
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive on the mbarrier at the same shared offset in every CTA of `mask`
// once every pair MMA this thread issued so far has completed.
DEVI void tc_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}
DEVI void tc_mma_f16_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 registers per thread -> 32 lanes x 32 consecutive 32-bit TMEM columns.
DEVI void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  __syncwarp();  // .sync.aligned: the whole warp, converged
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
DEVI void tmem_st_wait() {
  __syncwarp();
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit TMEM columns -> 32 registers per thread.
DEVI void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  __syncwarp();  // .sync.aligned: the whole warp, converged
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit TMEM columns -> 16 registers per thread.
DEVI void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  __syncwarp();  // .sync.aligned: the whole warp, converged
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// 16 registers per thread -> 32 lanes x 16 consecutive 32-bit TMEM columns.
DEVI void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  __syncwarp();  // .sync.aligned: the whole warp, converged
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
DEVI void tmem_ld_wait() {
  __syncwarp();
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- score keys
// Order-preserving 32-bit key of an fp32 score with the order reversed (a
// smaller key is a larger score); -0 is folded into +0 so equal scores get
// equal keys.
DEVI uint32_t desc_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  const uint32_t asc = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ~asc;
}
DEVI float key_score(uint32_t k) {
  const uint32_t asc = ~k;
  return __uint_as_float((asc & 0x80000000u) ? (asc & 0x7fffffffu) : ~asc);
}

// ---------------------------------------------------------------- math
// SiLU(x) = x * sigmoid(x), sigmoid(x) = 0.5 + 0.5 * tanh(x / 2), one MUFU op.
DEVI float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
DEVI float silu_fast(float x) {
  const float hx = 0.5f * x;
  return fmaf(hx, tanh_approx(hx), hx);
}
// x / (1 + e^-x) with the fast exponential and reciprocal (relative error of
// a few fp32 ulps); saturates to -0 for x below about -88.
DEVI float silu_accurate(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

DEVI uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// fp16 pair with saturation to +-65504 (no infinities from in-range math).
DEVI uint32_t pack_f16x2_sat(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}
DEVI float f16lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu))); }
DEVI float f16hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }
DEVI float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
DEVI float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
// A packed pair in either 16-bit format of the tensor-core path (f16 != 0: fp16).
DEVI uint32_t pack16(int f16, float lo, float hi) {
  return f16 ? pack_f16x2_sat(lo, hi) : pack_bf16x2(lo, hi);
}
DEVI float lo16(int f16, uint32_t v) { return f16 ? f16lo(v) : bf16lo(v); }
DEVI float hi16(int f16, uint32_t v) { return f16 ? f16hi(v) : bf16hi(v); }

// Log-linear bucket of a non-negative distance (see hstu.h).
DEVI int log_bucket(int x, int S, int N) {
  int b;
  if (x < (1 << S)) {
    b = x;
  } else {
    const int e = 31 - __clz(x);
    b = ((e - S + 1) << S) + ((x >> (e - S)) - (1 << S));
  }
  return min(b, N - 1);
}
// log_bucket without branches (the same values; x >= 0): lanes of a warp
// whose distances fall on both sides of 2^S do not diverge.
// The same bucket without branches (x >= 0, S <= 20): for x >= 2^S the
// bucket (e - S + 1) 2^S + (top S bits below x's leading one) is read off the
// float x converted toward zero, whose exponent field is e + 127 and whose
// mantissa's top S bits are exactly those bits: (bits >> (23 - S)) - (126 + S) 2^S.
DEVI uint32_t log_bucket_nb(int x, int S, int N) {
  const int big = (int)(__float_as_uint(__int2float_rz(x)) >> (23 - S)) - ((126 + S) << S);
  const int b = x < (1 << S) ? x : big;
  return (uint32_t)min(b, N - 1);
}
// Smallest distance that falls in bucket b (b < N), saturated to int32.
DEVI int bucket_lo(int b, int S) {
  if (b < (1 << S)) return b;
  const int g = b >> S;  // e - S + 1
  const long long m = b & ((1 << S) - 1);
  const int sh = g - 1;
  if (sh >= 31) return 0x7fffffff;
  const long long v = ((1ll << S) + m) << sh;
  return v > 0x7fffffffll ? 0x7fffffff : (int)v;
}

}  // namespace hstu
