// warmup.cuh -- the training-time BitLinear forward with the quantization
// warm-up, and its straight-through backward.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// section 動的ウォームアップ量子化 (lambda = min(step / total_steps, 1) scales
// the difference between the full-precision and the quantized values, so
// fine-tuning moves from no quantization to full quantization), with the
// weight and activation quantizers of its section 量子化の仕組み and the
// straight-through estimator of the same page (the rounding passes the
// gradient through unchanged).
//
// Reading (the page gives the blend for "the" quantized value): the blend
// applies to both operands that the page quantizes, each quantized value
// being the rescaled fake-quant value, in rounded fp32 steps:
//   W_lam = W + lambda * (t / s_w - W)              t, s_w: the ternary quant
//   x_lam = x_n + lambda * (x_q / s_x - x_n)        x_n: RMSNorm of x
//   y     = x_lam W_lam^T                            bf16 operands, fp32 sums
// Both operands are rounded to bf16 (the training dtype) and multiplied on
// the tensor cores (tcgen05.mma kind::f16, fp32 accumulation in TMEM).  The
// straight-through backward treats the quantizers as the identity, so
// dL/dW = dY^T x_lam and dL/dx_n = dY W_lam: the same GEMM on transposed
// copies.
#pragma once

#include "act_quant.cuh"
#include "common.cuh"
#include "weight_quant.cuh"

namespace bitnet {

// --------------------------------------------------------- fake-quant inputs

__device__ __forceinline__ float warmup_blend(float v, float q, float lam) {
  return __fadd_rn(v, __fmul_rn(lam, __fsub_rn(q, v)));
}

// W_lam (bf16) from W (fp32) and the per-tensor scale s_w (written by the
// weight-scale kernels before this one).
__global__ void __launch_bounds__(256)
warmup_weights_kernel(const float* __restrict__ W, int64_t n4, const float* __restrict__ s_w,
                      float lam, __nv_bfloat16* __restrict__ W_lam) {
  const float sw = *s_w;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(W) + i);
    const float w[4] = {v.x, v.y, v.z, v.w};
    __nv_bfloat16 o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float t = static_cast<float>(static_cast<int>(ternary_code(w[j], sw)) - 1);
      o[j] = __float2bfloat16_rn(warmup_blend(w[j], __fdiv_rn(t, sw), lam));
    }
    uint2 packed;
    packed.x = static_cast<uint32_t>(__bfloat16_as_ushort(o[0])) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(o[1])) << 16);
    packed.y = static_cast<uint32_t>(__bfloat16_as_ushort(o[2])) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(o[3])) << 16);
    reinterpret_cast<uint2*>(W_lam)[i] = packed;
  }
}

// x_lam (bf16, [M][K]) of one token row per CTA: RMSNorm in the canonical
// order of the quantization kernel, the per-token absmax scale, then the
// blend.  The row is re-read in each pass (L1 serves the re-reads).
template <bool kBF16>
__global__ void __launch_bounds__(kActThreads)
warmup_act_kernel(const void* __restrict__ x, const float* __restrict__ gamma, float eps,
                  int64_t K, float lam, __nv_bfloat16* __restrict__ x_lam) {
  __shared__ float red[kActThreads];
  const int tid = threadIdx.x;
  const int64_t m = blockIdx.x;
  const int64_t nchunk = K >> 3;
  auto chunk = [&](int64_t c, float (&v)[8]) {
    widen8<kBF16>(load_raw8<kBF16>(x, m * K + 8 * c), v);
  };
  float p = 0.0f;
  for (int64_t c = tid; c < nchunk; c += kActThreads) {
    float v[8];
    chunk(c, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) p = __fmaf_rn(v[j], v[j], p);
  }
  const float ss = block_tree_sum_f32(p, red);
  const float d = __fadd_rn(__fdiv_rn(ss, static_cast<float>(K)), eps);
  const bool zero_row = (d == 0.0f);
  const float r = zero_row ? 0.0f : __fdiv_rn(1.0f, __fsqrt_rn(d));
  float a = 0.0f;
  for (int64_t c = tid; c < nchunk; c += kActThreads) {
    float v[8], g[8];
    chunk(c, v);
    load_gamma8(gamma, 8 * c, g);
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(__fmul_rn(__fmul_rn(v[j], r), g[j])));
  }
  const float amax = block_max_f32(a, red);
  const float sx = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
  for (int64_t c = tid; c < nchunk; c += kActThreads) {
    float v[8], g[8];
    chunk(c, v);
    load_gamma8(gamma, 8 * c, g);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      float o[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float xn = __fmul_rn(__fmul_rn(v[j + h], r), g[j + h]);
        const float qt = __fdiv_rn(static_cast<float>(quant_one(xn, sx)), sx);
        o[h] = warmup_blend(xn, qt, lam);
      }
      w[j >> 1] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[0]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[1]))) << 16);
    }
    reinterpret_cast<uint4*>(x_lam + m * K)[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// bf16 src [R][C] -> dst [C][ldd] (ldd >= R; entries R..ldd-1 of each dst row
// are zero) through 32 x 32 shared-memory tiles: the backward's K-major
// operands.  Grid: (ceil(C/32), ceil(ldd/32)), 256 threads.
__global__ void __launch_bounds__(256)
transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src, int64_t R, int64_t C,
                      __nv_bfloat16* __restrict__ dst, int64_t ldd) {
  __shared__ uint16_t tile[32][33];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = r0 + i, c = c0 + tx;
    tile[i][tx] = (r < R && c < C) ? __bfloat16_as_ushort(src[r * C + c]) : 0;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t c = c0 + i, r = r0 + tx;
    if (c < C && r < ldd) dst[c * ldd + r] = __ushort_as_bfloat16(tile[tx][i]);
  }
}

// ------------------------------------------------------------- bf16 GEMM

// C[m][n] = sum_k B[m][k] A[n][k] (both operands K-major bf16, fp32 sums):
// A rows are the output columns (128 per CTA, the MMA's M and TMEM lanes),
// B rows the output rows (BN per CTA, the MMA's N).  y [M][ldy] fp32 or bf16.
struct WgParams {
  int M, N, K;
  void* y;
  int64_t ldy;
  int y_bf16;
  int* status;
  uint64_t wait_limit_ns;
  int use_pdl;
};

template <int BN>
struct WgCfg {
  static constexpr int BM = 128;
  static constexpr int KSTEP = 64;                 // bf16 per step: one 128-byte swizzle row
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN >= 256 ? 4 : 6;
  static constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;  // one fp32 column per token
  static constexpr int THREADS = 256;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int NBAR = 2 * STAGES + 1;      // full, done, accfull
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int SMEM_DYN = OFF_MISC + 16 + 1024;
  static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(SMEM_DYN <= 232448, "shared memory");
};

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4)                                 // D = F32
         | (1u << 7)                               // A = BF16
         | (1u << 10)                              // B = BF16
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void tc_mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warps: 0 copies A, 2 copies B (one 2-D tensor copy each per 64-k step into
// a STAGES-deep ring), 1 allocates TMEM and issues the MMAs (four K = 16
// MMAs per step, then a commit that frees the stage), 4-7 read the
// accumulators back (warp 4 + q: TMEM lanes 32q..32q+31) and store y.
// Every wait is bounded; on a timeout the kernel records the failure, lets
// its copies land and exits without writing y.
template <int BN>
__global__ void __launch_bounds__(WgCfg<BN>::THREADS, 1)
bf16_gemm_nt_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b, const WgParams p) {
  using C = WgCfg<BN>;
  extern __shared__ uint8_t wg_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(wg_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* done = full + C::STAGES;
  uint64_t* accfull = done + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::BM, m0 = blockIdx.y * BN;
  const int nk = (p.K + C::KSTEP - 1) / C::KSTEP;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 2);    // the A and the B producer
      mbar_init(&done[s], 1);    // MMA commit
    }
    mbar_init(accfull, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  if (p.use_pdl) pdl_wait_prior_grid();

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      const bool is_a = warp == 0;
      const CUtensorMap* map = is_a ? &tmap_a : &tmap_b;
      const int off = is_a ? 0 : C::A_BYTES;
      const uint32_t bytes = is_a ? C::A_BYTES : C::B_BYTES;
      const int row0 = is_a ? n0 : m0;
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES &&
            !mbar_wait_bounded(&done[s], static_cast<uint32_t>(j / C::STAGES - 1) & 1u,
                               abort_flag, limit)) {
          *abort_flag = 1;
          record_failure(p.status, DEV_TIMEOUT_PRODUCER);
          break;
        }
        mbar_arrive_expect_tx(&full[s], bytes);
        tma_load_2d(smem + s * C::STAGE_BYTES + off, map, j * C::KSTEP, row0, &full[s]);
        issued = j + 1;
      }
      if (*abort_flag) {
        for (int j = (issued > C::STAGES ? issued - C::STAGES : 0); j < issued; ++j)
          if (!mbar_wait_bounded(&full[j % C::STAGES], static_cast<uint32_t>(j / C::STAGES) & 1u,
                                 nullptr, limit))
            record_failure(p.status, DEV_TIMEOUT_DRAIN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(C::BM, BN);
      for (int j = 0; j < nk; ++j) {
        const int s = j % C::STAGES;
        if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>(j / C::STAGES) & 1u, abort_flag,
                               limit)) {
          *abort_flag = 1;
          record_failure(p.status, DEV_TIMEOUT_MMA);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_base = smem_u32(smem + s * C::STAGE_BYTES);
        const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::KSTEP / 16; ++kk)   // 16 bf16 = 32 bytes per MMA
          tc_mma_f16_ss(tmem_base, umma_desc_sw128_kmajor(a_base + 32 * kk),
                        umma_desc_sw128_kmajor(b_base + 32 * kk), idesc,
                        (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&done[s]);
      }
      tc_commit(accfull);
    }
  } else if (warp >= 4) {
    const int q = warp - 4;
    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(accfull, 0u, nullptr, limit));
    if (!ok && lane == 0) record_failure(p.status, DEV_TIMEOUT_EPILOGUE);
    tc_fence_after_sync();
    const bool write = __all_sync(0xFFFFFFFFu, ok && *abort_flag == 0) && nk > 0;
    const int n = n0 + 32 * q + lane;
    if (write) {
      for (int c0 = 0; c0 < BN; c0 += 16) {
        if (m0 + c0 >= p.M) break;   // uniform across the warp
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + c0, r);
        tmem_ld_wait();
        if (n < p.N) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int m = m0 + c0 + jj;
            if (m < p.M) {
              const float v = __uint_as_float(r[jj]);
              const int64_t o = static_cast<int64_t>(m) * p.ldy + n;
              if (p.y_bf16)
                reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
              else
                reinterpret_cast<float*>(p.y)[o] = v;
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
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace bitnet
