// device.cuh -- sm_100a building blocks shared by the kernels of libw8a8:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM allocation,
// INT8 MMA, commit, TMEM loads) and the exact fp32 helpers of the epilogue.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/w8a8.h"

namespace w8a8 {

// Default limit of every device-side wait (nanoseconds of %globaltimer).
// Far above any legitimate wait (microseconds), short enough that a stuck
// kernel returns with an error status instead of holding the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// First failure sticks: later codes do not overwrite an earlier one.
__device__ __forceinline__ void record_error(int32_t *status_word, int32_t code) {
  if (status_word) atomicCAS(status_word, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// try_wait that acquires at cluster scope: for a phase completed by arrivals
// of another CTA of the cluster (mbarrier.arrive.release.cluster) whose
// shared-memory writes the waiter then reads.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase of `bar` with the given parity to complete. Gives up
// after limit_ns, or as soon as *abort (shared) becomes non-zero; returns
// false when it gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  const volatile int *abort, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Non-blocking test of a phase completed by another CTA of the cluster
// (acquire at cluster scope; returns at once either way).
__device__ __forceinline__ bool mbar_test_wait_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// mbar_wait_bounded acquiring at cluster scope (see mbar_try_wait_cluster).
__device__ __forceinline__ bool mbar_wait_bounded_cluster(uint64_t *bar, uint32_t parity, const volatile int *abort,
                                                          uint64_t limit_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (abort && *abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory; completion
// is signalled on `bar` as transaction bytes. x is the inner (contiguous)
// coordinate in elements and must be a multiple of 16 bytes' worth.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint64_t *bar, void *dst,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

// 2-D tiled TMA store from this CTA's shared memory (one bulk group per
// commit). x must be a multiple of 16 bytes' worth of elements, x, y >= 0;
// rows and columns past the tensor's extent are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_addr(src)), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until no committed bulk store group of this thread still reads shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Wait until every committed bulk store group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 1-D bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global memory into this CTA's shared memory, completing on `bar` as
// transaction bytes. No multicast.
__device__ __forceinline__ void bulk_load_1d(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
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

// D[tmem] (+)= A[smem] * B[smem]^T, signed 8-bit inputs, int32 accumulator.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets the
// 32 columns of TMEM lane (lane base of its warp quarter) + i.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored in the
// 128-byte swizzled layout that TMA's SWIZZLE_128B writes: rows of 128 bytes,
// groups of 8 rows 1024 bytes apart (stride byte offset), tile base 1024-byte
// aligned. Layout type 2 = 128B swizzle; version field 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t smem_byte_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_byte_addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                            // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;                    // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                            // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                            // SWIZZLE_128B
  return d;
}

// Instruction descriptor of tcgen05.mma kind::i8: s8 x s8 -> s32, both
// operands K-major, shape M x N (x K = 32 bytes).
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4)                                  // D format: s32
         | (1u << 7)                                // A: signed 8-bit
         | (1u << 10)                               // B: signed 8-bit
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B (the
// same type on both sides), an fp32 accumulator, both operands K-major,
// shape M x N (x K = 16 elements).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                  // D format: f32
         | (1u << 7)                                // A: bf16
         | (1u << 10)                               // B: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// Make this thread's ordinary shared-memory stores visible to the async proxy
// (TMA, tcgen05.mma) before signalling a barrier the MMA thread waits on.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Ask L2 for `bytes` (a multiple of 16) from a 16-byte aligned global address,
// without waiting. L2 is where global memory is kept coherent, so this is
// safe even before the kernel that writes the range has finished: a line
// fetched early is updated by any later write.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream is still
// running; griddepcontrol.wait blocks until that kernel has completed and its
// memory is visible (a no-op when there is no such dependency).
__device__ __forceinline__ void pdl_wait_prerequisite() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allow the next kernel in the stream (if launched with programmatic stream
// serialization) to start launching now.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- CTA pairs
// Rank of this CTA in its cluster.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address, in the cluster's shared window, of the same shared-memory offset in
// CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(const void *p, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_addr(p)), "r"(rank));
  return out;
}

// All threads of all CTAs of the cluster (call it from every thread).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier given by its cluster-window address (another CTA's).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Store a 32-bit word to a shared::cluster address (from map_to_rank).
__device__ __forceinline__ void st_shared_cluster(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Make the cluster-scope writes that an acquired barrier phase guards visible
// (after a wait on a barrier another CTA arrived on with release.cluster).
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// Count `bytes` of the current phase's transactions as done without a copy
// (for a phase that expects bytes a copy will never bring).
__device__ __forceinline__ void mbar_complete_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// 2-D TMA load for a CTA pair: lands in this CTA's shared memory and signals
// the mbarrier at `bar_cluster_addr` (the pair leader's), no multicast.
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *map, uint32_t bar_cluster_addr, void *dst,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T over the pair
// (M = 256: each CTA holds 128 rows of A and of D; B's N rows are split
// between the two CTAs' shared memory). Issued by one thread of the leader.
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem of both CTAs] (+)= A * B^T over the pair with bf16 operands and an
// fp32 accumulator (tcgen05.mma kind::f16; A and B are both bf16, K = 16 per
// instruction). Issued by one thread of the leader.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at `bar_cluster_addr` (any CTA of the pair) when
// the pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar_cluster_addr) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar_cluster_addr)
               : "memory");
}

// ---------------------------------------------------------------- numerics
// bf16 <-> fp32 on raw bits.
__device__ __forceinline__ float bf16_lo(uint32_t two) { return __uint_as_float(two << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t two) { return __uint_as_float(two & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// round-half-even of an fp32 product, pre-clamped to [-1024, 1024] so that a
// zero point can be added without overflow (the int8 clamp that follows
// makes the pre-clamp invisible).
__device__ __forceinline__ int rne_clamped(float p) {
  int t = __float2int_rn(p);
  return min(max(t, -1024), 1024);
}

// Round to nearest even into int32 (out-of-range values saturate).
__device__ __forceinline__ int rne_s32(float p) {
  int r;
  asm("cvt.rni.s32.f32 %0, %1;" : "=r"(r) : "f"(p));
  return r;
}

// Four int32 saturated to [-128, 127] and packed, a in the lowest byte.
__device__ __forceinline__ uint32_t pack_sat_s8x4(int a, int b, int c, int d) {
  uint32_t hi, out;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(d), "r"(c));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(out) : "r"(b), "r"(a), "r"(hi));
  return out;
}

// Symmetric codes of the 8 bf16 values in one uint4: clamp(rne(x * r), -127, 127). With r = 127/absmax every |x * r|
// is at most 127 * (1 + 2^-23), so saturating to [-128, 127] equals that clamp.
// The two fp32 products x0 * r and x1 * r, each rounded to nearest even, in
// one packed fp32x2 multiply. Only for products that are rounded on their own:
// ptxas contracts a packed multiply followed by a packed add into a fused
// multiply-add, so no packed add may take these products.
__device__ __forceinline__ void mul_f32x2(float x0, float x1, float r, float &p0, float &p1) {
  asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %4};\n\t"
      "mul.rn.f32x2 pd, pa, pb;\n\t"
      "mov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(p0), "=f"(p1)
      : "f"(x0), "f"(x1), "f"(r));
}

__device__ __forceinline__ uint2 quant8_sym_sat(const uint4 &v, float r) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int q[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float p0, p1;
    mul_f32x2(bf16_lo(w[i]), bf16_hi(w[i]), r, p0, p1);
    q[2 * i] = rne_s32(p0);
    q[2 * i + 1] = rne_s32(p1);
  }
  return make_uint2(pack_sat_s8x4(q[0], q[1], q[2], q[3]), pack_sat_s8x4(q[4], q[5], q[6], q[7]));
}

// r = 127/a for a vector with absmax a, or 0 for a vector quantized as zero:
// a = 0 (or NaN), or a so small (below 127/FLT_MAX, about 3.7e-37) that 127/a
// overflows fp32 -- no finite scale resolves such values on the int8 grid.
__device__ __forceinline__ float sym_r(float a) {
  const float r = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
  return isinf(r) ? 0.0f : r;
}

// Its scale S = a/127, 0 where sym_r gave 0 for a finite a.
__device__ __forceinline__ float sym_S(float a, float r) {
  return r > 0.0f || isinf(a) ? __fdiv_rn(a, 127.0f) : 0.0f;
}

// The low bytes of four words, a in the lowest byte (two byte permutes).
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}


// Static asymmetric codes of the 8 bf16 values in one uint4:
// clamp(rne(x * r) + Z, -128, 127), Z in [-128, 127]. The product is held to the integer
// bounds [-128 - Z, 127 - Z] before it is rounded -- rounding is monotone,
// so holding to integer bounds before or after it gives the same integer --
// and then rounded to nearest, ties to even, by adding 1.5 * 2^23, which
// leaves rne(y) in the low mantissa bits (|y| <= 255 here). The code is the
// low byte of those bits plus Z - 0x4B400000. A NaN product is held to the
// lower bound (fmaxf returns the non-NaN operand): code -128.
__device__ __forceinline__ uint2 quant8_asym_sat(const uint4 &v, float r, int z) {
  const float lo = static_cast<float>(-128 - z), hi = static_cast<float>(127 - z);
  const int bias = z - 0x4B400000;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int q[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    q[2 * i] = __float_as_int(__fadd_rn(fminf(fmaxf(__fmul_rn(bf16_lo(w[i]), r), lo), hi), 12582912.0f)) + bias;
    q[2 * i + 1] = __float_as_int(__fadd_rn(fminf(fmaxf(__fmul_rn(bf16_hi(w[i]), r), lo), hi), 12582912.0f)) + bias;
  }
  return make_uint2(low_bytes4(q[0], q[1], q[2], q[3]), low_bytes4(q[4], q[5], q[6], q[7]));
}

// Byte b (0..3) of w sign-extended to 32 bits: one prmt whose selector copies
// byte b into the lowest byte and replicates its sign bit (selector nibble
// with the high bit set) into the other three.
template <int b>
__device__ __forceinline__ int sext_byte(uint32_t w) {
  constexpr uint32_t kSel = b | ((b | 8u) << 4) | ((b | 8u) << 8) | ((b | 8u) << 12);
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "n"(kSel));
  return static_cast<int>(r);
}

// S * (q - Z) for the 16 codes of one uint4 (code j in byte j), Z in
// [-128, 127]. q - Z is turned into fp32 without the conversion unit: the
// sign-extended code plus 0x4B400000 - Z is the bit pattern of
// 1.5 * 2^23 + (q - Z) (|q - Z| <= 255), from which 1.5 * 2^23 is subtracted
// exactly. The product is the one rounding, as in S * float(q - Z).
__device__ __forceinline__ void dequant16(const uint4 &v, float S, int z, float (&y)[16]) {
  const int bias = 0x4B400000 - z;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q[4] = {sext_byte<0>(w[i]), sext_byte<1>(w[i]), sext_byte<2>(w[i]), sext_byte<3>(w[i])};
#pragma unroll
    for (int b = 0; b < 4; ++b) y[4 * i + b] = __fmul_rn(S, __fsub_rn(__int_as_float(q[b] + bias), 12582912.0f));
  }
}

// Running absmax of the bf16 pairs of v, one packed max of magnitudes per
// word: each half of the result is max(|m2 half|, |v half|) with the sign bit
// meaningless (it is the xor of the operands' signs), so clear the sign bits
// (absmax2_halves) before reading it. A NaN operand gives the canonical NaN
// 0x7FFF, above every finite or infinite magnitude.
__device__ __forceinline__ uint32_t absmax2_bf16(const uint4 &v, uint32_t m2) {
  asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m2) : "r"(v.x));
  asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m2) : "r"(v.y));
  asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m2) : "r"(v.z));
  asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m2) : "r"(v.w));
  return m2;
}

// The larger magnitude of the two halves of a running absmax2_bf16 value.
__device__ __forceinline__ uint32_t absmax2_halves(uint32_t m2) {
  m2 &= 0x7FFF7FFFu;
  return max(m2 & 0xFFFFu, m2 >> 16);
}


}  // namespace w8a8
