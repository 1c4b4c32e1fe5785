// gemv.cuh -- decode-path ternary matmul (M <= 16 tokens): stream the packed
// 2-bit weights from HBM with 16-byte coalesced loads straight into registers,
// unpack them with one shift and one mask per 4 weights, and multiply on the
// tensor cores with warp-level int8 MMA (m16n8k32, s8 x s8 -> s32) in
// "swap-AB" form: 16 weight rows are the MMA's M side, the (at most 16)
// tokens its N side.  Dequantization is fused into the epilogue.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// sections 計算パラダイム (integer accumulation), 推論最適化とカスタムカーネル
// (weights unpacked on the fly inside the matmul) and タイル化行列乗算 (tiling
// to cut redundant global-memory traffic), 量子化の仕組み (rescale).
//
// Unpacking without a lookup: a 32-bit word P of packed codes holds k = 0..15
// of a 16-weight group (code of k in bits 2k, 2k+1).  (P >> 2r) & 0x03030303
// is a word of four int8 codes for k = r, 4+r, 8+r, 12+r.  The activations are
// stored k-interleaved (byte 4r+i of each 16-group holds k = 4i+r), so the
// activation word at byte offset 4r pairs with exactly those k.  Codes are
// t+1 in {0,1,2}; the kernel accumulates sum x*(t+1) and subtracts the token's
// row sum sum x at the end, which is exact integer arithmetic.
//
// Fragment mapping (lane = 4g + t): lane loads 16 bytes (64 k) of weight rows
// g and g+8 of each 16-row group at k offset 64t of the current 256-k step;
// word w of that load feeds MMAs 2w and 2w+1 (shifts 0,2 and 4,6); the B
// fragment for token g is the matching 8 bytes of the interleaved activation
// row, staged in shared memory.
//
// Split-K: a CTA covers ROWS weight rows and a contiguous range of 256-k
// steps.  With several K ranges, CTAs add their int32 partials into a
// workspace with atomics; the last CTA of a row block (found with a counter,
// no waiting) reads and re-zeroes the partials, and finishes the dequant.
#pragma once

#include "common.cuh"

namespace bitnet {

struct GemvParams {
  const uint8_t* Wp;      // [N][K/4]
  const int8_t* xi;       // [M][K] k-interleaved activations
  const int32_t* rowsum;  // [M]
  const float* s_x;       // [M] (null: no dequant)
  const float* s_w;       // [1] (null: no dequant)
  int M, N, K;
  int iters_per_split;    // 256-k steps per CTA
  int32_t* ws_acc;        // [M][N] zero-filled split-K partials (when gridDim.y > 1)
  unsigned* ws_cnt;       // [row blocks] zero-filled arrival counters
  void* y;                // [M][N] fp32 or bf16, may be null
  int y_bf16;
  int32_t* acc_out;       // [M][N] debug accumulators, may be null
  int use_pdl;            // wait for the preceding grid before reading activations
  int early_weights;      // prefetch weights before that wait (only when the preceding
                          // grid is known not to write them)
};

constexpr uint32_t kCodeMask = 0x03030303u;

__device__ __forceinline__ void finish_output(const GemvParams& p, float sw, int m, int n,
                                              int acc_codes) {
  const int acc = acc_codes - p.rowsum[m];
  const int64_t o = static_cast<int64_t>(m) * p.N + n;
  if (p.acc_out) p.acc_out[o] = acc;
  if (p.y) {
    const float yv = __fdiv_rn(__int2float_rn(acc), __fmul_rn(p.s_x[m], sw));
    if (p.y_bf16)
      reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(yv);
    else
      reinterpret_cast<float*>(p.y)[o] = yv;
  }
}

template <int RG>
__device__ __forceinline__ void gemv_load_weights(const GemvParams& p, int n0, int g, int t,
                                                  int it, uint4 (&pa)[RG], uint4 (&pb)[RG]) {
  const int64_t rowbytes = p.K >> 2;
  const int kseg = it * 256 + 64 * t;
  const bool kval = kseg < p.K;
#pragma unroll
  for (int rg = 0; rg < RG; ++rg) {
    const int ra = n0 + 16 * rg + g;
    const int rb = ra + 8;
    pa[rg] = make_uint4(0u, 0u, 0u, 0u);
    pb[rg] = make_uint4(0u, 0u, 0u, 0u);
    if (kval && ra < p.N) pa[rg] = ldg_stream_u4(p.Wp + ra * rowbytes + (kseg >> 2));
    if (kval && rb < p.N) pb[rg] = ldg_stream_u4(p.Wp + rb * rowbytes + (kseg >> 2));
  }
}

__device__ __forceinline__ uint32_t u4_word(const uint4& v, int w) {
  return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

template <int RG, int NT>
__global__ void __launch_bounds__(256)
ternary_gemv_kernel(const GemvParams p) {
  constexpr int ROWS = 16 * RG;
  constexpr int MT = 8 * NT;
  extern __shared__ __align__(16) uint8_t xs[];
  __shared__ int red[ROWS * MT];
  __shared__ int is_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * ROWS;
  const int total_iters = (p.K + 255) >> 8;
  const int it0 = blockIdx.y * p.iters_per_split;
  const int it1 = min(it0 + p.iters_per_split, total_iters);
  const int KC = p.iters_per_split * 256;
  const int XS = KC + 16;  // padded row stride: conflict-free 16-byte fragment loads

  for (int i = tid; i < ROWS * MT; i += blockDim.x) red[i] = 0;

  // Prefetch this warp's first weight step; weights do not depend on the
  // preceding kernel, so this overlaps it under programmatic launch.
  uint4 pa[RG], pb[RG];
  int it = it0 + warp;
  if (p.early_weights && it < it1) gemv_load_weights<RG>(p, n0, g, t, it, pa, pb);

  if (p.use_pdl) pdl_wait_prior_grid();
  if (!p.early_weights && it < it1) gemv_load_weights<RG>(p, n0, g, t, it, pa, pb);

  // Stage this CTA's slice of the interleaved activations, zero-padded.
  const int kbase = it0 * 256;
  const int cpr = KC >> 4;  // 16-byte chunks per row
  for (int idx = tid; idx < MT * cpr; idx += blockDim.x) {
    const int mm = idx / cpr, cc = idx - mm * cpr;
    const int k = kbase + 16 * cc;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (mm < p.M && k < p.K)
      v = *reinterpret_cast<const uint4*>(p.xi + static_cast<int64_t>(mm) * p.K + k);
    *reinterpret_cast<uint4*>(xs + mm * XS + 16 * cc) = v;
  }
  __syncthreads();

  int acc[RG][NT][4];
#pragma unroll
  for (int rg = 0; rg < RG; ++rg)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[rg][nt][j] = 0;

  for (; it < it1; it += nwarps) {
    uint4 na[RG], nb[RG];
    const int itn = it + nwarps;
    if (itn < it1) gemv_load_weights<RG>(p, n0, g, t, itn, na, nb);

    uint4 bx[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint8_t* src = xs + (8 * nt + g) * XS + (it - it0) * 256 + 64 * t;
#pragma unroll
      for (int q = 0; q < 4; ++q) bx[nt][q] = *reinterpret_cast<const uint4*>(src + 16 * q);
    }
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t Pa = u4_word(pa[rg], w);
        const uint32_t Pb = u4_word(pb[rg], w);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int sh = 4 * h;
          const uint32_t a0 = (Pa >> sh) & kCodeMask;
          const uint32_t a2 = (Pa >> (sh + 2)) & kCodeMask;
          const uint32_t a1 = (Pb >> sh) & kCodeMask;
          const uint32_t a3 = (Pb >> (sh + 2)) & kCodeMask;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint32_t b0 = h ? bx[nt][w].z : bx[nt][w].x;
            const uint32_t b1 = h ? bx[nt][w].w : bx[nt][w].y;
            mma_m16n8k32_s8(acc[rg][nt], a0, a1, a2, a3, b0, b1);
          }
        }
      }
    }
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) {
      pa[rg] = na[rg];
      pb[rg] = nb[rg];
    }
  }

  // Combine the warps' partials (integer sums: order does not matter).
#pragma unroll
  for (int rg = 0; rg < RG; ++rg)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int r0 = 16 * rg + g, r1 = r0 + 8;
      const int c0 = 8 * nt + 2 * t;
      atomicAdd(&red[r0 * MT + c0], acc[rg][nt][0]);
      atomicAdd(&red[r0 * MT + c0 + 1], acc[rg][nt][1]);
      atomicAdd(&red[r1 * MT + c0], acc[rg][nt][2]);
      atomicAdd(&red[r1 * MT + c0 + 1], acc[rg][nt][3]);
    }
  __syncthreads();

  const float sw = (p.y && p.s_w) ? __ldg(p.s_w) : 0.0f;
  const int nout = ROWS * p.M;
  if (gridDim.y == 1) {
    for (int idx = tid; idx < nout; idx += blockDim.x) {
      const int r = idx % ROWS, mm = idx / ROWS, n = n0 + r;
      if (n < p.N) finish_output(p, sw, mm, n, red[r * MT + mm]);
    }
    return;
  }
  for (int idx = tid; idx < nout; idx += blockDim.x) {
    const int r = idx % ROWS, mm = idx / ROWS, n = n0 + r;
    if (n < p.N) atomicAdd(p.ws_acc + static_cast<int64_t>(mm) * p.N + n, red[r * MT + mm]);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(p.ws_cnt + blockIdx.x, 1u) == gridDim.y - 1) ? 1 : 0;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int idx = tid; idx < nout; idx += blockDim.x) {
    const int r = idx % ROWS, mm = idx / ROWS, n = n0 + r;
    if (n < p.N) {
      const int v = atomicExch(p.ws_acc + static_cast<int64_t>(mm) * p.N + n, 0);
      finish_output(p, sw, mm, n, v);
    }
  }
  if (tid == 0) p.ws_cnt[blockIdx.x] = 0u;  // ready for the next call
}

}  // namespace bitnet
