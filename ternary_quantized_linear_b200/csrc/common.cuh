// common.cuh -- device helpers shared by the sm_100a kernels: inline PTX for
// mbarriers, TMA, tcgen05 (TMEM allocation, MMA, loads), the bounded-wait
// discipline, and small reductions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnet {

// Kernel-side detail codes written to the device status word on a timeout.
enum DeviceDetail : int {
  DEV_OK = 0,
  DEV_TIMEOUT_PRODUCER = 1,
  DEV_TIMEOUT_UNPACK = 2,
  DEV_TIMEOUT_MMA = 3,
  DEV_TIMEOUT_EPILOGUE = 4,
  DEV_TIMEOUT_DRAIN = 5,
  DEV_TIMEOUT_SELFTEST = 6,
  DEV_TIMEOUT_GEMV = 7,
  DEV_TIMEOUT_QUANT = 8,  // activation-quant row copy
};

// Default limit of one on-chip wait (nanoseconds of %globaltimer).  Real
// waits last microseconds; this only bounds a wait that would never end.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Record the first failure of this launch sequence (later ones are dropped).
__device__ __forceinline__ void record_failure(int* status, int detail) {
  if (status) atomicCAS(status, 0, detail);
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait until the phase with the given parity of `bar` has completed.  Gives
// up (returns false) when *abort becomes non-zero or after limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  const volatile int* abort, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    if ((i & 31u) == 0u) {
      if (abort && *abort) return false;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
}

// One try with a suspend-time hint: the thread sleeps until the phase
// completes or about hint_ns pass, instead of spinning on the issue slots
// that the warps sharing its scheduler need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar_addr, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar_addr), "r"(parity), "r"(hint_ns)
      : "memory");
  return done != 0;
}

// mbar_wait_bounded with sleeping tries (the abort flag and the limit are
// looked at between tries).
__device__ __forceinline__ bool mbar_wait_bounded_sleep(uint64_t* bar, uint32_t parity,
                                                        const volatile int* abort,
                                                        uint64_t limit_ns) {
  constexpr uint32_t kHintNs = 20000;
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(a, parity, kHintNs)) return true;
    if (abort && *abort) return false;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// ----------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor load (no multicast) into this CTA's shared memory;
// completion is reported as transaction bytes on `bar`.  c0 is the innermost
// coordinate (elements), c1 the row.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int c0,
                                            int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 1-D bulk copy (no tensor map, no multicast) of `bytes` contiguous bytes
// from global memory into this CTA's shared memory, completing as
// transaction bytes on `bar`.  Both addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// -------------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
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

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, int8 x int8 -> int32, one CTA.
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on `bar` when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns: thread i of the warp gets
// columns [col, col+16) of TMEM lane (lane_base + i).
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand in the 128-byte
// swizzled canonical layout: rows of 128 bytes, 8-row atoms of 1024 bytes
// (stride byte offset), 16-byte chunk index XOR-ed with (row % 8).
__device__ __forceinline__ uint64_t umma_desc_sw128_kmajor(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1u) << 16;                     // leading byte offset (16 B)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;             // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;                     // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                     // SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::i8, s8 x s8 -> s32, both K-major, dense.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int M, int N) {
  return (2u << 4)                                 // D = S32
         | (1u << 7)                               // A = signed 8-bit
         | (1u << 10)                              // B = signed 8-bit
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// ------------------------------------------------- programmatic dependent launch

__device__ __forceinline__ void pdl_wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------------- mma.sync

// D = A(16x32, s8, row) * B(32x8, s8, col) + C, int32.
__device__ __forceinline__ void mma_m16n8k32_s8(int (&d)[4], uint32_t a0, uint32_t a1,
                                                uint32_t a2, uint32_t a3, uint32_t b0,
                                                uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = c + the dot product of the four unsigned bytes of a with the four
// signed bytes of b (exact, 32-bit wrap-around never reached by the callers).
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Barrier `id` (1..15) over `count` threads (a multiple of 32): lets a
// subset of a CTA's warps synchronise without the others.
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ------------------------------------------------------------ division

// a / b rounded to nearest even (binary32) through y = RN(1 / b):
// Markstein's method (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with y
// within half an ulp of 1/b and q within one ulp of a/b, the residual
// a - b q is exact under a fused multiply-add and RN(q + (a - b q) y) =
// RN(a / b).  One correction brings RN(a y) within one ulp; the second
// rounds correctly.  That holds for finite a and b whose quotient and
// numerator are zero or stay well inside the normal range.
//
// The dequant divides integers (|a| <= 2^31) by s_x * s_w.  For a divisor
// with 2^-95 <= |b| <= 2^100 every such quotient lies in [2^-100, 2^126],
// so the divisor alone decides: recip_for_div(b) returns RN(1 / b) for such
// divisors and 0 otherwise, computed once per token, and div_rn_int takes
// the IEEE division for a zero reciprocal (reachable only with extreme
// gains or weight magnitudes).  No test per output: an extra range check
// there cost the tensor-core prefill kernel a fifth of its throughput.
__device__ __forceinline__ float recip_for_div(float b) {
  const float ab = fabsf(b);
  return (ab >= 0x1p-95f && ab <= 0x1p100f) ? __frcp_rn(b) : 0.0f;
}

// Kept out of line: an inlined IEEE division in an unrolled epilogue
// multiplies the kernel's code size.
__device__ __noinline__ float div_rn_out_of_range(float a, float b) { return __fdiv_rn(a, b); }

// RN(a / b) for an integer-valued a with |a| <= 2^31 and y = recip_for_div(b)
// known to be non-zero (a kernel that checked all its divisors beforehand).
__device__ __forceinline__ float div_rn_int_fast(float a, float b, float y) {
  float q = __fmul_rn(a, y);
  float r = __fmaf_rn(-q, b, a);
  q = __fmaf_rn(r, y, q);
  r = __fmaf_rn(-q, b, a);
  return __fmaf_rn(r, y, q);
}

// RN(a / b) for an integer-valued a with |a| <= 2^31, y = recip_for_div(b).
__device__ __forceinline__ float div_rn_int(float a, float b, float y) {
  if (y == 0.0f) return div_rn_out_of_range(a, b);
  return div_rn_int_fast(a, b, y);
}

// ------------------------------------------------- decode activation order

// Decode-matmul block order: inside every 256-byte span of a token row of
// k-interleaved x_q, 16-byte block b is stored at block x_block_pos(b, m & 1).
// A lane (g, t) of the decode matmul reads blocks 4t + q of token g; with
// this order the eight lanes of a quarter warp (two tokens of opposite
// parity, t = 0..3) hit eight different 16-byte bank groups for every q.
__host__ __device__ __forceinline__ int x_block_pos(int b, int parity) {
  return b ^ (((b >> 3) & 1) << 1) ^ parity;
}

// ---------------------------------------------------------- float helpers

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
  return __uint_as_float(h << 16);
}

}  // namespace bitnet
