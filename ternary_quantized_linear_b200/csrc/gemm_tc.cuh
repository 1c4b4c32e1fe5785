// gemm_tc.cuh -- prefill-path ternary matmul on the 5th-generation tensor
// cores: tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// sections 計算パラダイム (integer matmul), 推論最適化とカスタムカーネル
// (weights unpacked on the fly inside the kernel), タイル化行列乗算 (tiles
// staged in fast shared memory to avoid redundant global traffic),
// 量子化の仕組み (rescale by both scales).
//
// One CTA computes a 128 (weight rows) x BN (tokens) tile of acc^T:
//   warp 0      TMA producer: per 128-k step, the activation tile
//               (BN x 128 int8, 128-byte swizzle, straight into the MMA's
//               canonical K-major layout) and the packed weight tile
//               (128 rows x 32 bytes) into a STAGES-deep ring;
//   warp 1      allocates TMEM; one thread issues 4 MMAs (K = 32 each) per
//               step with A = unpacked weights, B = activations, and
//               commits each stage back to the producer;
//   warps 4-7   unpack: thread i expands row i's 32 packed bytes to 128 int8
//               codes (shift + mask, no table) written into the swizzled A
//               tile, then fences the async proxy and arrives; after the last
//               step the same warps read TMEM (one lane = one weight row) and
//               write y = (acc - rowsum) / (s_x * s_w) coalesced along N.
// The unpacked codes are t+1 in {0,1,2}, in the same k-interleaved order as
// the activations (see act_quant.cuh), so the MMA pairs equal k and the row
// sum correction restores sum x*t exactly.
//
// Every wait is bounded: on a timeout the thread records the failure in the
// device status word, raises a CTA abort flag (so the other roles stop
// waiting), and the kernel drains in-flight copies and MMAs before it frees
// TMEM and exits without writing results.
#pragma once

#include "common.cuh"

namespace bitnet {

struct GemmParams {
  const int32_t* rowsum;  // [M]
  const float* s_x;       // [M] (null: no dequant)
  const float* s_w;       // [1]
  int M, N, K;
  void* y;                // [M][N] or null
  int y_bf16;
  int32_t* acc_out;       // [M][N] debug or null
  int* status;            // device status word
  uint64_t wait_limit_ns;
};

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;                 // weight rows per CTA (MMA M)
  static constexpr int BK = 128;                 // k per pipeline stage (one swizzle row)
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 5 : 4);
  static constexpr int X_BYTES = BN * BK;        // activation tile
  static constexpr int A_BYTES = BM * BK;        // unpacked weight tile
  static constexpr int WP_BYTES = BM * BK / 4;   // packed weight tile
  static constexpr int OFF_X = 0;
  static constexpr int OFF_A = OFF_X + STAGES * X_BYTES;
  static constexpr int OFF_WP = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_BAR = OFF_WP + STAGES * WP_BYTES;
  static constexpr int NBAR = 3 * STAGES + 1;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_DYN = BYTES + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = BN;      // power of two >= 32
  static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
  static_assert(SMEM_DYN <= 232448, "shared memory");
};

__device__ __forceinline__ void gemm_fail(volatile int* abort_flag, int* status, int detail) {
  *abort_flag = 1;
  record_failure(status, detail);
}

template <int BN>
__global__ void __launch_bounds__(256, 1)
ternary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_w, const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* xs = smem + C::OFF_X;
  uint8_t* as = smem + C::OFF_A;
  uint8_t* wps = smem + C::OFF_WP;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* aready = full + C::STAGES;
  uint64_t* empty = aready + C::STAGES;
  uint64_t* accfull = empty + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::BM;
  const int m0 = blockIdx.y * BN;
  const int nk = (p.K + C::BK - 1) / C::BK;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&aready[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accfull, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t use = static_cast<uint32_t>(kb / C::STAGES);
        if (kb >= C::STAGES && !mbar_wait_bounded(&empty[s], (use - 1u) & 1u, abort_flag, limit)) {
          gemm_fail(abort_flag, p.status, DEV_TIMEOUT_PRODUCER);
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::X_BYTES + C::WP_BYTES);
        tma_load_2d(xs + s * C::X_BYTES, &tmap_x, kb * C::BK, m0, &full[s]);
        tma_load_2d(wps + s * C::WP_BYTES, &tmap_w, kb * (C::BK / 4), n0, &full[s]);
        issued = kb + 1;
      }
      if (*abort_flag) {
        // Let the copies already in flight land before the CTA exits.
        const int first = issued > C::STAGES ? issued - C::STAGES : 0;
        for (int kb = first; kb < issued; ++kb) {
          const int s = kb % C::STAGES;
          if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>(kb / C::STAGES) & 1u, nullptr,
                                 limit))
            record_failure(p.status, DEV_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t idesc = umma_idesc_i8(C::BM, BN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t par = static_cast<uint32_t>(kb / C::STAGES) & 1u;
        if (!mbar_wait_bounded(&full[s], par, abort_flag, limit) ||
            !mbar_wait_bounded(&aready[s], par, abort_flag, limit)) {
          gemm_fail(abort_flag, p.status, DEV_TIMEOUT_MMA);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_base = smem_u32(as + s * C::A_BYTES);
        const uint32_t b_base = smem_u32(xs + s * C::X_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::BK / 32; ++kk) {
          tc_mma_i8(tmem_d, umma_desc_sw128_kmajor(a_base + 32 * kk),
                    umma_desc_sw128_kmajor(b_base + 32 * kk), idesc,
                    (kb > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      // Signals the epilogue; on an abort it still marks that every MMA
      // issued so far has finished with TMEM and shared memory.
      tc_commit(accfull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- unpack
    const int i = threadIdx.x - 128;  // weight row inside the tile
    const int sw = i & 7;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % C::STAGES;
      const uint32_t par = static_cast<uint32_t>(kb / C::STAGES) & 1u;
      if (!mbar_wait_bounded(&full[s], par, abort_flag, limit)) {
        gemm_fail(abort_flag, p.status, DEV_TIMEOUT_UNPACK);
        break;
      }
      const uint4* src = reinterpret_cast<const uint4*>(wps + s * C::WP_BYTES + i * 32);
      const uint4 q0 = src[0], q1 = src[1];
      uint8_t* dst = as + s * C::A_BYTES + i * 128;
      const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const uint32_t P = words[w];
        *reinterpret_cast<uint4*>(dst + ((w ^ sw) << 4)) =
            make_uint4(P & 0x03030303u, (P >> 2) & 0x03030303u, (P >> 4) & 0x03030303u,
                       (P >> 6) & 0x03030303u);
      }
      fence_proxy_async_smem();
      mbar_arrive(&aready[s]);
    }
    // ----------------------------------------------------------- epilogue
    const bool done = mbar_wait_bounded(accfull, 0u, nullptr, limit);
    if (!done) gemm_fail(abort_flag, p.status, DEV_TIMEOUT_EPILOGUE);
    tc_fence_after_sync();
    // tcgen05.ld is warp-collective: decide once per warp.
    const bool write = __all_sync(0xFFFFFFFFu, done && *abort_flag == 0);
    if (write) {
      const int wq = warp - 4;
      const int n = n0 + wq * 32 + lane;
      const float swv = (p.y && p.s_w) ? *p.s_w : 0.0f;
      for (int c0 = 0; c0 < BN; c0 += 16) {
        if (m0 + c0 >= p.M) break;  // uniform across the warp
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem_d + (static_cast<uint32_t>(wq * 32) << 16) + c0, r);
        tmem_ld_wait();
        if (n < p.N) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m0 + c0 + j;
            if (m < p.M) {
              const int acc = static_cast<int>(r[j]) - p.rowsum[m];
              const int64_t o = static_cast<int64_t>(m) * p.N + n;
              if (p.acc_out) p.acc_out[o] = acc;
              if (p.y) {
                const float yv = __fdiv_rn(__int2float_rn(acc), __fmul_rn(p.s_x[m], swv));
                if (p.y_bf16)
                  reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(yv);
                else
                  reinterpret_cast<float*>(p.y)[o] = yv;
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_d, C::TMEM_COLS);
  }
}

}  // namespace bitnet
