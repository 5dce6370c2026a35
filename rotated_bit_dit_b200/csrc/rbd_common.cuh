// Shared device helpers of the rotated low-bit linear library (sm_100a only).
// Hand-written inline PTX for mbarriers, TMA, and the tcgen05 tensor-core /
// tensor-memory instructions, plus the bounded-wait and status machinery.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/rbd.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "rotated_bit_dit_b200 targets sm_100a only"
#endif

namespace rbd {

// ---------------------------------------------------------------- status word
// Device-side error record: 0 = fine, otherwise an rbd_status value.  Lives in
// the library's static device memory; read and cleared by rbd_check().  The
// library is one translation unit (rbd_lib.cu), so this is its only definition.
__device__ int g_device_status = 0;

// Default bound of a device-side wait (nanoseconds, measured with %globaltimer).
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;   // 2 s

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_status(int s) {
  atomicCAS(&g_device_status, 0, s);
}

__device__ __forceinline__ bool device_failed() {
  return *reinterpret_cast<volatile int*>(&g_device_status) != 0;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
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

// As mbar_try_wait, but the thread may sleep until the phase completes or about
// 20 us pass, so waiting warps do not take issue slots from working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
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

// Bounded wait for the phase with the given parity to complete.  Returns false
// (and records RBD_ERR_DEVICE_TIMEOUT) when the bound expires or another
// thread already recorded a failure; callers then leave their loops.
// The status word in global memory is read only after 50 us of waiting and
// then every 50 us, so a normal hand-off never waits behind a memory load.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t timeout_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint64_t next_check = t0 + 50000ull;
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait_sleep(bar, parity)) return true;
    const uint64_t now = globaltimer_ns();
    if (now >= next_check) {
      if (device_failed()) return false;
      if (now - t0 > timeout_ns) {
        record_status(RBD_ERR_DEVICE_TIMEOUT);
        return false;
      }
      next_check = now + 50000ull;
    }
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled bulk tensor load global -> shared, completing transaction bytes on `bar`.
// c0 is the innermost (contiguous) coordinate.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 2D tiled bulk tensor store shared -> global (tracked by this thread's bulk
// async-groups).  c0 is the innermost coordinate; rows outside the tensor are
// not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Contiguous bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- tcgen05
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
// Arrive on `bar` once every previously issued tcgen05.mma of this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, INT8 inputs, int32 accumulation.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, 8-bit float inputs (kind::f8f6f4, formats
// given by the instruction descriptor), fp32 accumulation, K = 32 per instruction.
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 lanes x 16 consecutive 32-bit columns, load + wait in one statement.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Asynchronous form: 32 lanes x 16 columns, no wait.  The registers may only be
// read after tmem_wait_ld() followed by tmem_reg_fence() on the same array.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Orders every later use of `r` after the preceding tcgen05.wait::ld (both are
// volatile asm statements, so they keep their relative order).
__device__ __forceinline__ void tmem_reg_fence(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]));
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (tcgen05 format, version 1): K-major operand
// whose rows are `row_bytes` long (32, 64 or 128 -> matching swizzle mode) and
// are stored contiguously, 8-row core groups `8*row_bytes` apart.
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t smem_addr, uint32_t row_bytes) {
  uint64_t layout;
  switch (row_bytes) {
    case 128: layout = 2; break;   // SWIZZLE_128B
    case 64: layout = 4; break;    // SWIZZLE_64B
    default: layout = 6; break;    // SWIZZLE_32B
  }
  const uint64_t sbo = (8u * row_bytes) >> 4;
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                  // leading byte offset (unused for swizzled K-major)
  d |= (sbo & 0x3FFFu) << 32;               // stride byte offset between 8-row groups
  d |= (uint64_t)1u << 46;                  // descriptor version for tcgen05
  d |= layout << 61;
  return d;
}

// Instruction descriptor: INT8 x INT8 -> S32, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_i8(uint32_t m, uint32_t n, bool a_signed = true, bool b_signed = true) {
  return (2u << 4)                          // D format: S32
         | ((a_signed ? 1u : 0u) << 7)       // A: s8 / u8
         | ((b_signed ? 1u : 0u) << 10)      // B: s8 / u8
         | ((n >> 3) << 17) | ((m >> 4) << 24);
}
// Instruction descriptor of kind::f8f6f4: E4M3 x E4M3 (format 0) -> F32, both
// K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3(uint32_t m, uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);
}
// Instruction descriptor: BF16 x BF16 -> F32, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t m, uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// Block-scaled FP4 MMA: D[tmem] (+)= (A * SFA) * (B * SFB)^T, E2M1 operands in
// shared memory, one E4M3 scale per 16 elements read from TMEM (sfa, sfb),
// float32 accumulation, K = 64 per instruction.
__device__ __forceinline__ void mma_nvf4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Copy 32 rows x 16 bytes of shared memory into TMEM lanes 0-31, 4 columns,
// replicated into all four lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory matrix descriptor of an unswizzled K-major matrix whose rows are
// 16 bytes (consecutive rows, 8-row groups 128 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_rows16(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;           // leading byte offset (one 16-byte column: unused)
  d |= (uint64_t)(128u >> 4) << 32;  // stride byte offset between 8-row groups
  d |= (uint64_t)1u << 46;           // descriptor version for tcgen05
  return d;                          // layout type 0: no swizzle
}

// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B (format 1), K-major,
// E4M3 scales (scale format 0), scale-factor byte offsets 0, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(uint32_t m, uint32_t n) {
  return (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// ---------------------------------------------------------------- misc
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before the preceding kernel of its stream has
// finished; pdl_wait() blocks until that kernel has completed and its memory
// operations are visible (a no-op for an ordinary launch).  A kernel calls
// pdl_launch_dependents() to let such a follower start early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Bulk prefetch of [p, p + bytes) into L2 (p 16-byte aligned, bytes a multiple
// of 16).  L2 is the point of coherence, so a prefetch never yields stale data.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight packed two's-complement nibbles (code k in bits 4k..4k+3) -> their eight
// E4M3 bytes, codes 0-3 in o0 and 4-7 in o1, in order.  Two byte-permute
// tables give the E4M3 byte of every non-negative nibble value (0..7) and of
// every negative one (-8..-1) from the nibble's low three bits; a third permute
// replicates each nibble's sign bit into a byte mask that selects between them.
constexpr uint32_t kE4Pos0 = 0x44403800u;   // E4M3 of 0, 1, 2, 3
constexpr uint32_t kE4Pos1 = 0x4E4C4A48u;   // E4M3 of 4, 5, 6, 7
constexpr uint32_t kE4Neg0 = 0xCACCCED0u;   // E4M3 of -8, -7, -6, -5
constexpr uint32_t kE4Neg1 = 0xB8C0C4C8u;   // E4M3 of -4, -3, -2, -1
__device__ __forceinline__ void nibbles_to_e4m3(uint32_t pw, uint32_t& o0, uint32_t& o1) {
  const uint32_t sel = pw & 0x77777777u;   // low three bits of every nibble
  const uint32_t sh4 = pw << 4;            // sign bits of the even nibbles at byte msbs
  const uint32_t selh = sel >> 16;
  const uint32_t m0 = prmt(sh4, pw, 0xD9C8u);   // 0xFF where codes 0..3 are negative
  const uint32_t m1 = prmt(sh4, pw, 0xFBEAu);   // likewise codes 4..7
  o0 = (prmt(kE4Pos0, kE4Pos1, sel) & ~m0) | (prmt(kE4Neg0, kE4Neg1, sel) & m0);
  o1 = (prmt(kE4Pos0, kE4Pos1, selh) & ~m1) | (prmt(kE4Neg0, kE4Neg1, selh) & m1);
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

}  // namespace rbd
