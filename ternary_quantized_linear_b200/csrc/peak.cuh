// peak.cuh -- a measurement kernel, not part of the forward: it keeps the
// int8 tensor cores of every SM busy with back-to-back
// tcgen05.mma.cta_group::1.kind::i8 instructions of shape M = 128,
// N = 256, K = 32 (the largest single-CTA tile), so that the caller can time
// it and derive the dense int8 rate of the GPU as it is clocked at the
// moment.  The prefill kernel's roofline is reported against that rate.
//
// Operands: A (128 x 32 int8) from shared memory or, like the forward's
// kernels, from tensor memory; B (256 x 32 int8) from shared memory; the
// int32 accumulators in tensor memory.  The values are zero: the rate of the
// instruction does not depend on them.  One thread per CTA issues every MMA;
// a commit at the end is waited for (bounded) before the TMEM is freed.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kPeakN = 256;
constexpr int kPeakSmem = (128 + kPeakN) * 128 + 1024;  // A and B, 128-byte rows, + alignment

template <bool kTmemA>
__global__ void __launch_bounds__(128, 1)
mma_i8_peak_kernel(int64_t iters, int* status, uint64_t wait_limit_ns) {
  extern __shared__ uint8_t pk_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(pk_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a = smem;                 // 128 rows x 128 bytes
  uint8_t* b = smem + 128 * 128;     // 256 rows x 128 bytes
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(8) uint64_t done;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (128 + kPeakN) * 128 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_slot;
  const uint32_t d_tmem = tmem;          // columns 0..255: accumulators
  const uint32_t a_tmem = tmem + 256;    // columns 256..263: A (kTmemA)
  if (kTmemA && warp < 4) {
    // Zero the A columns (32 lanes per warp quarter, 8 columns of 4 bytes).
    uint32_t z[16] = {};
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            a_tmem + (static_cast<uint32_t>(32 * warp) << 16)),
        "r"(z[0]), "r"(z[1]), "r"(z[2]), "r"(z[3]), "r"(z[4]), "r"(z[5]), "r"(z[6]), "r"(z[7]),
        "r"(z[8]), "r"(z[9]), "r"(z[10]), "r"(z[11]), "r"(z[12]), "r"(z[13]), "r"(z[14]),
        "r"(z[15])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (threadIdx.x == 0) {
    const uint32_t idesc = umma_idesc_i8(128, kPeakN);
    const uint64_t adesc = umma_desc_sw128_kmajor(smem_u32(a));
    const uint64_t bdesc = umma_desc_sw128_kmajor(smem_u32(b));
    for (int64_t i = 0; i < iters; ++i) {
      if (kTmemA) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
            "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(i > 0 ? 1u : 0u)
            : "memory");
      } else {
        tc_mma_i8(d_tmem, adesc, bdesc, idesc, i > 0 ? 1u : 0u);
      }
    }
    tc_commit(&done);
    if (!mbar_wait_bounded(&done, 0u, nullptr, wait_limit_ns))
      record_failure(status, DEV_TIMEOUT_MMA);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bitnet
