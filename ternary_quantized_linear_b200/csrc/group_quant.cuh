// group_quant.cuh -- group-wise scales: the weights and the activations are
// split into G = K / group_k contiguous groups along K that are quantized
// independently, each with its own scale.
//
// Method: bitnet.cpp article (unite.ai), section グループ量子化と正規化
// (weights and activations split into groups, each quantized on its own so
// that groups need no communication), applied to the scheme of "LLM を 1.58
// ビットにファインチューニング：BitNet による極端な量子化", section 量子化の仕組み
// (absmean weights, per-token absmax activations after a normalisation).
//
//   s_w[g]   = 1 / max(mean |W| over all rows and the group's columns, 1e-5)
//              (fp64 sum in the order of the per-tensor scale, applied to the
//              N x group_k block: element k - g*group_k of a row feeds partial
//              ((k - g*group_k)/4) mod 256, tree; rows feed partial n mod 256,
//              tree)
//   t        = clamp(rint(W * s_w[g(k)]), -1, 1), packed as the per-tensor codes
//   s_x[m,g] = 127 / max(max_{k in g} |x_n[m,k]|, 1e-5), x_n the RMSNorm of the
//              whole row
//   x_q      = clamp(rint(x_n * s_x[m,g(k)]), -128, 127)
//   acc_g    = sum_{k in g} x_q t (the matmul kernels write it per group)
//   y[m,n]   = sum_g (float)acc_g / (s_x[m,g] * s_w[g]), the fp32 terms summed
//              in fp64 and rounded once (group_combine_kernel).
// group_k is a multiple of 256 (one k chunk of the tiled weights).
#pragma once

#include "act_quant.cuh"
#include "common.cuh"
#include "weight_quant.cuh"

namespace bitnet {

constexpr int kGroupMaxG = 512;   // groups per row the activation kernel handles

// R[n*G + g] = sum of |W| over the group's columns of row n (canonical order).
__global__ void __launch_bounds__(kWqThreads)
group_row_abs_sum_kernel(const float* __restrict__ W, int64_t K, int64_t group_k,
                         double* __restrict__ R) {
  __shared__ double red[kWqThreads];
  const int64_t n = blockIdx.x;
  const int64_t G = K / group_k;
  const float* row = W + n * K;
  for (int64_t g = 0; g < G; ++g) {
    const float* grp = row + g * group_k;
    double p = 0.0;
    for (int64_t c = threadIdx.x; c < group_k / 4; c += kWqThreads) {
      const float4 v = ldg_stream_f4(grp + 4 * c);
      p = __dadd_rn(p, fabs(static_cast<double>(v.x)));
      p = __dadd_rn(p, fabs(static_cast<double>(v.y)));
      p = __dadd_rn(p, fabs(static_cast<double>(v.z)));
      p = __dadd_rn(p, fabs(static_cast<double>(v.w)));
    }
    const double rg = block_tree_sum_f64(p, red);
    if (threadIdx.x == 0) R[n * G + g] = rg;
  }
}

// One CTA per group: s_w[g] from the row sums of the group.
__global__ void __launch_bounds__(kWqThreads)
group_abs_total_kernel(const double* __restrict__ R, int64_t N, int64_t G, int64_t group_k,
                       float* __restrict__ s_w) {
  __shared__ double red[kWqThreads];
  const int64_t g = blockIdx.x;
  double q = 0.0;
  for (int64_t n = threadIdx.x; n < N; n += kWqThreads) q = __dadd_rn(q, R[n * G + g]);
  const double S = block_tree_sum_f64(q, red);
  if (threadIdx.x == 0) {
    float mean = __double2float_rn(__ddiv_rn(S, static_cast<double>(N * group_k)));
    mean = fmaxf(mean, 1e-5f);
    s_w[g] = __fdiv_rn(1.0f, mean);
  }
}

// Pack with the scale of each word's group (a word = 16 weights of one row,
// never straddling a group since group_k % 256 == 0).
__global__ void __launch_bounds__(kWqThreads)
group_pack_kernel(const float* __restrict__ W, int64_t nwords, int64_t K, int64_t group_k,
                  const float* __restrict__ s_w, uint32_t* __restrict__ W_p) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kWqThreads;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kWqThreads) + threadIdx.x; i < nwords;
       i += stride) {
    const float sw = s_w[((16 * i) % K) / group_k];
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

// RMSNorm + group-wise absmax quantization of one token row per CTA (the row
// re-read from global memory in each pass; L1 serves the re-reads).  Writes
// x_q k-interleaved in the decode-tiled order (tiled), row-major
// interleaved (for the tensor-core kernel) or in natural order (natural, a
// debug export), s_x [M][G] and the group row sums rowsum [M][G] (may be
// null).
template <bool kBF16>
__global__ void __launch_bounds__(kActThreads)
group_rmsnorm_quant_kernel(const void* __restrict__ x, const float* __restrict__ gamma,
                           float eps, int64_t M, int64_t K, int64_t group_k,
                           int8_t* __restrict__ x_q, float* __restrict__ s_x,
                           int32_t* __restrict__ rowsum, int tiled, int perm, int natural,
                           uint4* __restrict__ zero16, int64_t n_zero16, int trigger) {
  __shared__ float redf[kActThreads];
  __shared__ unsigned gmax[kGroupMaxG];
  __shared__ float gsx[kGroupMaxG];
  __shared__ int gsum[kGroupMaxG];
  if (trigger) pdl_launch_dependents();
  if (static_cast<int64_t>(blockIdx.x) >= M) {
    zero_fill_blocks(zero16, n_zero16, static_cast<int64_t>(blockIdx.x) - M,
                     static_cast<int64_t>(gridDim.x) - M);
    return;
  }
  const int tid = threadIdx.x;
  const int64_t m = blockIdx.x;
  const int64_t G = K / group_k;
  const int64_t nchunk = K >> 3;
  for (int64_t g = tid; g < G; g += kActThreads) {
    gmax[g] = 0u;
    gsum[g] = 0;
  }
  auto chunk = [&](int64_t c, float (&v)[8]) {
    widen8<kBF16>(load_raw8<kBF16>(x, m * K + 8 * c), v);
  };
  // Pass 1: sum of squares in the canonical order.
  float p = 0.0f;
  for (int64_t c = tid; c < nchunk; c += kActThreads) {
    float v[8];
    chunk(c, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) p = __fmaf_rn(v[j], v[j], p);
  }
  const float ss = block_tree_sum_f32(p, redf);   // its barriers also order the clears
  const float ms = __fdiv_rn(ss, static_cast<float>(K));
  const float d = __fadd_rn(ms, eps);
  const bool zero_row = (d == 0.0f);
  const float r = zero_row ? 0.0f : __fdiv_rn(1.0f, __fsqrt_rn(d));
  // Pass 2: max |x_n| per group (non-negative floats order like their bits).
  if (!zero_row) {
    for (int64_t c = tid; c < nchunk; c += kActThreads) {
      float v[8], gm[8];
      chunk(c, v);
      load_gamma8(gamma, 8 * c, gm);
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(__fmul_rn(__fmul_rn(v[j], r), gm[j])));
      atomicMax(&gmax[(8 * c) / group_k], __float_as_uint(a));
    }
  }
  __syncthreads();
  for (int64_t g = tid; g < G; g += kActThreads) {
    const float sx = __fdiv_rn(127.0f, fmaxf(__uint_as_float(gmax[g]), 1e-5f));
    gsx[g] = sx;
    s_x[m * G + g] = sx;
  }
  __syncthreads();
  // Pass 3: quantize with the group's scale, store, group row sums.
  const bool tl = tiled != 0;
  int8_t* xq_row = tl ? x_q + m * 256 : x_q + m * K;
  const int64_t cs = tl ? M * 256 : 256;
  const int64_t nstore = tl ? ((K + 255) >> 8) << 5 : nchunk;
  const int iters = static_cast<int>((nstore + kActThreads - 1) / kActThreads);
  for (int it = 0; it < iters; ++it) {
    const int64_t c = tid + static_cast<int64_t>(kActThreads) * it;
    int8_t q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (c < nchunk && !zero_row) {
      float v[8], gm[8];
      chunk(c, v);
      load_gamma8(gamma, 8 * c, gm);
      const int64_t g = (8 * c) / group_k;
      const float sx = gsx[g];
      int sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        q[j] = quant_one(__fmul_rn(__fmul_rn(v[j], r), gm[j]), sx);
        sum += q[j];
      }
      atomicAdd(&gsum[g], sum);
    }
    Chunk8 ch{pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7])};
    if (natural)
      store_chunk8<false>(xq_row, 8 * c, ch, c < nstore);
    else
      store_chunk8<true>(xq_row, 8 * c, ch, c < nstore, perm ? static_cast<int>(m & 1) : -1,
                         cs);
  }
  __syncthreads();
  if (rowsum)
    for (int64_t g = tid; g < G; g += kActThreads) rowsum[m * G + g] = gsum[g];
}

// y[m][n] = sum_g (float)acc[g][m][n] / (s_x[m][g] * s_w[g]): each term one
// correctly rounded fp32 division, the terms summed in fp64 in group order,
// the sum rounded once.  acc holds the group sums of x_q * t (row sums
// already subtracted).
__global__ void __launch_bounds__(256)
group_combine_kernel(const int32_t* __restrict__ acc, const float* __restrict__ s_x,
                     const float* __restrict__ s_w, int64_t M, int64_t N, int64_t G,
                     void* __restrict__ y, int y_bf16) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N;
    double s = 0.0;
    for (int64_t g = 0; g < G; ++g) {
      const float d = __fmul_rn(s_x[m * G + g], s_w[g]);
      s = __dadd_rn(s, static_cast<double>(__fdiv_rn(__int2float_rn(acc[g * total + i]), d)));
    }
    const float yv = __double2float_rn(s);
    if (y_bf16)
      reinterpret_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(yv);
    else
      reinterpret_cast<float*>(y)[i] = yv;
  }
}

}  // namespace bitnet
