// weight_quant.cuh -- absmean per-tensor ternary quantization and 2-bit
// packing of a weight matrix W [N][K] (offline, once per matrix).
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// section 量子化の仕組み (weights: per-tensor scale = 1/mean|W|, scale, round,
// clamp to [-1, 1]) and section 主な発見 (ternary weights packed into int8
// tensors); "[論文レビュー] The Era of 1-bit LLMs", section 提案手法 (absmean,
// values {-1, 0, 1}).
//
// Three kernels, all HBM-bound:
//   1. row_abs_sum_kernel: R_n = sum_k |W[n,k]| in fp64, element k feeding
//      partial (k/4) mod 256 (thread t owns the float4 chunks t, t+256, ...,
//      increasing k), partials combined by the tree i += i+s, s = 128..1.
//   2. abs_total_kernel (one CTA): S = tree over partials q_j = sum of R_n for
//      n = j mod 256 in increasing n; s_w = 1/max((float)(S/(N*K)), 1e-5).
//   3. pack_kernel: code = clamp(rint(W*s_w), -1, 1) + 1, four codes per
//      byte, weight k in bits [2(k%4), 2(k%4)+1] of byte k/4 of its row.
// The fixed orders make s_w (and hence every code) identical on every run.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kWqThreads = 256;

__device__ __forceinline__ double block_tree_sum_f64(double p, double* red) {
  const int tid = threadIdx.x;
  red[tid] = p;
  __syncthreads();
#pragma unroll
  for (int s = 128; s >= 32; s >>= 1) {
    if (tid < s) red[tid] = __dadd_rn(red[tid], red[tid + s]);
    __syncthreads();
  }
  if (tid < 32) {
    double v = red[tid];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v = __dadd_rn(v, __shfl_down_sync(0xFFFFFFFFu, v, s));
    if (tid == 0) red[0] = v;
  }
  __syncthreads();
  const double r = red[0];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float4 ldg_stream_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kWqThreads)
row_abs_sum_kernel(const float* __restrict__ W, int64_t K, double* __restrict__ R) {
  __shared__ double red[kWqThreads];
  const int64_t n = blockIdx.x;
  const float* row = W + n * K;
  const int64_t nchunk = K >> 2;
  double p = 0.0;
  for (int64_t c = threadIdx.x; c < nchunk; c += kWqThreads) {
    const float4 v = ldg_stream_f4(row + 4 * c);
    p = __dadd_rn(p, fabs(static_cast<double>(v.x)));
    p = __dadd_rn(p, fabs(static_cast<double>(v.y)));
    p = __dadd_rn(p, fabs(static_cast<double>(v.z)));
    p = __dadd_rn(p, fabs(static_cast<double>(v.w)));
  }
  const double rn = block_tree_sum_f64(p, red);
  if (threadIdx.x == 0) R[n] = rn;
}

__global__ void __launch_bounds__(kWqThreads)
abs_total_kernel(const double* __restrict__ R, int64_t N, int64_t K, float* __restrict__ s_w) {
  __shared__ double red[kWqThreads];
  double q = 0.0;
  for (int64_t n = threadIdx.x; n < N; n += kWqThreads) q = __dadd_rn(q, R[n]);
  const double S = block_tree_sum_f64(q, red);
  if (threadIdx.x == 0) {
    float mean = __double2float_rn(__ddiv_rn(S, static_cast<double>(N * K)));
    mean = fmaxf(mean, 1e-5f);
    *s_w = __fdiv_rn(1.0f, mean);
  }
}

__device__ __forceinline__ uint32_t ternary_code(float w, float sw) {
  float v = rintf(__fmul_rn(w, sw));
  v = fminf(fmaxf(v, -1.0f), 1.0f);
  return static_cast<uint32_t>(static_cast<int>(v) + 1);
}

// Each thread turns 16 consecutive weights (of the flattened [N*K] array)
// into one 32-bit word of packed codes; K % 64 == 0 so a word never straddles
// two rows.
__global__ void __launch_bounds__(kWqThreads)
pack_kernel(const float* __restrict__ W, int64_t nwords, const float* __restrict__ s_w,
            uint32_t* __restrict__ W_p) {
  const float sw = *s_w;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kWqThreads;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kWqThreads) + threadIdx.x; i < nwords;
       i += stride) {
    const float* src = W + 16 * i;
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src) + q);
      word |= ternary_code(v.x, sw) << (8 * q + 0);
      word |= ternary_code(v.y, sw) << (8 * q + 2);
      word |= ternary_code(v.z, sw) << (8 * q + 4);
      word |= ternary_code(v.w, sw) << (8 * q + 6);
    }
    W_p[i] = word;
  }
}

}  // namespace bitnet
