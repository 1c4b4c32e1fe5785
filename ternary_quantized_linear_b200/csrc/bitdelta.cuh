// bitdelta.cuh -- 1-bit deltas of fine-tuned weights and the batched
// multi-tenant decode forward that applies them.
//
// Method: "【論文要約】BitDelta: Your Fine-Tune May Only Be Worth One Bit",
// Eq. 1-4 (Delta = W_fine - W_base, its sign and one scale per matrix,
// alpha = mean |Delta|, the scale that minimises the L2 error of
// alpha * Sign(Delta)) and Eq. 6 with its multi-tenant serving setting (one
// shared base matrix, a packed 1-bit delta per tenant, every tenant's token
// multiplied by base + its own delta in one pass; decode latency measured for
// a 8192 x 8192 linear layer and 8 tenants, Fig. 4).
//
// Readings (the page leaves them open):
//   * Sign(0) = -1 (Eq. 2 maps positive differences to +1, the rest to -1).
//   * The page's kernel packs the sign bits 32 per integer without a bit
//     order: here bit j (least significant first) of word w of row n holds
//     the sign of Delta[n, 32 w + j] (1 = +1), rows back to back, K/32
//     words each; tenants back to back ([B][N][K/32]).
//   * alpha is summed in fp64 in the fixed order of the weight scale (row n:
//     element k into partial (k/4) mod 256, tree; rows into partial
//     n mod 256, tree) and rounded once to fp32.
//   * y[b][n] = sum_k x[b][k] W_base[n][k] + alpha_b sum_k x[b][k] s_b[n][k]
//     with bf16 x and W_base, fp32 sums on the tensor cores.
#pragma once

#include "common.cuh"
#include "weight_quant.cuh"

namespace bitnet {

// One CTA per row n: the row's sign words and its fp64 sum of |Delta|.
__global__ void __launch_bounds__(kWqThreads)
bitdelta_row_kernel(const __nv_bfloat16* __restrict__ Wb, const __nv_bfloat16* __restrict__ Wf,
                    int64_t K, uint32_t* __restrict__ signs, double* __restrict__ R) {
  __shared__ double red[kWqThreads];
  const int64_t n = blockIdx.x;
  const uint16_t* b = reinterpret_cast<const uint16_t*>(Wb) + n * K;
  const uint16_t* f = reinterpret_cast<const uint16_t*>(Wf) + n * K;
  const int64_t nw = K >> 5;
  for (int64_t w = threadIdx.x; w < nw; w += kWqThreads) {
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 vb = __ldg(reinterpret_cast<const uint4*>(b + 32 * w) + q);
      const uint4 vf = __ldg(reinterpret_cast<const uint4*>(f + 32 * w) + q);
      const uint32_t eb[4] = {vb.x, vb.y, vb.z, vb.w}, ef[4] = {vf.x, vf.y, vf.z, vf.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float xb = bf16_bits_to_f32((eb[e] >> (16 * hh)) & 0xFFFFu);
          const float xf = bf16_bits_to_f32((ef[e] >> (16 * hh)) & 0xFFFFu);
          if (xf > xb) word |= 1u << (8 * q + 2 * e + hh);
        }
      }
    }
    signs[n * nw + w] = word;
  }
  double p = 0.0;
  for (int64_t c = threadIdx.x; c < (K >> 2); c += kWqThreads) {
    const uint2 vb = __ldg(reinterpret_cast<const uint2*>(b) + c);
    const uint2 vf = __ldg(reinterpret_cast<const uint2*>(f) + c);
    const uint32_t eb[2] = {vb.x, vb.y}, ef[2] = {vf.x, vf.y};
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const double db = static_cast<double>(bf16_bits_to_f32((eb[e] >> (16 * hh)) & 0xFFFFu));
        const double df = static_cast<double>(bf16_bits_to_f32((ef[e] >> (16 * hh)) & 0xFFFFu));
        p = __dadd_rn(p, fabs(__dsub_rn(df, db)));
      }
  }
  const double rn = block_tree_sum_f64(p, red);
  if (threadIdx.x == 0) R[n] = rn;
}

// One CTA: alpha = (float)(S / (N K)), S the tree over q_j = sum of R_n for
// n = j mod 256 in increasing n.
__global__ void __launch_bounds__(kWqThreads)
bitdelta_alpha_kernel(const double* __restrict__ R, int64_t N, int64_t K,
                      float* __restrict__ alpha) {
  __shared__ double red[kWqThreads];
  double q = 0.0;
  for (int64_t n = threadIdx.x; n < N; n += kWqThreads) q = __dadd_rn(q, R[n]);
  const double S = block_tree_sum_f64(q, red);
  if (threadIdx.x == 0) *alpha = __double2float_rn(__ddiv_rn(S, static_cast<double>(N * K)));
}

// ------------------------------------------------------- batched forward

constexpr int kBdMaxTenants = 8;
constexpr int kBdWarps = 4;          // warps of a CTA, each a quarter of K

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ldg_stream_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// Two bf16 +-1 in one register from the spread sign bits v (see below):
// bit i of the thread's byte to the low half's sign, bit i+1 to the high
// half's, a set bit meaning +1.
__device__ __forceinline__ uint32_t sign_pair(uint32_t spread_not, int i) {
  return ((spread_not << (15 - i)) & 0x80008000u) | 0x3F803F80u;
}

// Byte i of a sign word, inverted (a clear bit -- Sign = -1 -- sets the
// bf16 sign), with its odd bits moved up by 15 so that one shift puts bit
// 2p at bit 15 and bit 2p+1 at bit 31 (sign_pair).
__device__ __forceinline__ uint32_t spread_byte(uint32_t inv_word, int i) {
  const uint32_t v = (inv_word >> (8 * i)) & 0xFFu;
  return (v & 0x55u) | ((v & 0xAAu) << 15);
}

// Grid: ceil(N/16) CTAs of kBdWarps warps; CTA r owns rows 16r..16r+15,
// warp w the words [w*nw/kBdWarps, (w+1)*nw/kBdWarps) of K, taken four at a
// time (128 k).  For quarter q of such a group (word 4U + q), lane (g, t)
// holds k = 32 (4U + q) + 8 t .. +7 of rows g and g+8 (one 16-byte load
// each; the four lanes of a row read 64 contiguous bytes), the same k of
// every token, and bits 8t..8t+7 of each tenant's sign word (the four words
// of a group come in one 16-byte load per row and tenant).  Two m16n8k16
// MMAs consume a quarter: MMA h takes k + 4h + {0,1} as the MMA's k
// positions 2t, 2t+1 and k + 4h + {2,3} as 2t+8, 2t+9 (any assignment works
// as long as both operands use it).  The tokens (the MMA's N = 8 = the
// tenants) read x at the same k; the base MMA multiplies W_base, tenant b's
// MMA its signs as bf16 +-1, keeping column b.  The warps' partial sums meet
// in shared memory, added in warp order.
__global__ void __launch_bounds__(32 * kBdWarps)
bitdelta_forward_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wb,
                        const uint32_t* __restrict__ signs, const float* __restrict__ alpha,
                        int B, int64_t N, int64_t K, void* __restrict__ y, int y_bf16) {
  __shared__ float part[kBdWarps][2][16][kBdMaxTenants];   // [warp][base, delta][row][tenant]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t nw = K >> 5;
  // Warp ranges start on 4-word boundaries, so every group but the last
  // is four whole words.
  const int64_t w0 = (nw * warp / kBdWarps) & ~static_cast<int64_t>(3);
  const int64_t w1 = warp == kBdWarps - 1 ? nw : (nw * (warp + 1) / kBdWarps) & ~static_cast<int64_t>(3);
  // 16-byte sign loads need 16-byte aligned rows and tenants.
  const bool vec_ok = (reinterpret_cast<uintptr_t>(signs) & 15) == 0 && (nw & 3) == 0;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 16;
  const int64_t ra = r0 + g, rb = r0 + g + 8;
  const bool va = ra < N, vb = rb < N;
  const bool vx = g < B;
  const uint8_t* pa = reinterpret_cast<const uint8_t*>(Wb + (va ? ra : 0) * K) + 16 * t;
  const uint8_t* pb = reinterpret_cast<const uint8_t*>(Wb + (vb ? rb : 0) * K) + 16 * t;
  const uint8_t* px = reinterpret_cast<const uint8_t*>(x + (vx ? g : 0) * K) + 16 * t;
  const uint32_t* sa = signs + (va ? ra : 0) * nw;
  const uint32_t* sb = signs + (vb ? rb : 0) * nw;
  const int64_t tstride = N * nw;   // words from one tenant's signs to the next
  float base[4] = {0.f, 0.f, 0.f, 0.f};
  float dl[kBdMaxTenants][4];
#pragma unroll
  for (int b = 0; b < kBdMaxTenants; ++b)
#pragma unroll
    for (int e = 0; e < 4; ++e) dl[b][e] = 0.f;

  for (int64_t u0 = w0; u0 < w1; u0 += 4) {
    const bool full = vec_ok && u0 + 4 <= w1;   // u0 is a multiple of 4
    uint4 wa[4], wbv[4], xv[4];
    uint4 s_a[kBdMaxTenants], s_b[kBdMaxTenants];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t u = u0 + q;
      const bool in = u < w1;
      wa[q] = (in && va) ? ldg_stream_u4(pa + 64 * u) : make_uint4(0u, 0u, 0u, 0u);
      wbv[q] = (in && vb) ? ldg_stream_u4(pb + 64 * u) : make_uint4(0u, 0u, 0u, 0u);
      xv[q] = (in && vx) ? __ldg(reinterpret_cast<const uint4*>(px + 64 * u))
                         : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int b = 0; b < kBdMaxTenants; ++b) {
      const bool tb = b < B;
      if (full) {
        s_a[b] = (tb && va) ? __ldg(reinterpret_cast<const uint4*>(sa + b * tstride + u0))
                            : make_uint4(0u, 0u, 0u, 0u);
        s_b[b] = (tb && vb) ? __ldg(reinterpret_cast<const uint4*>(sb + b * tstride + u0))
                            : make_uint4(0u, 0u, 0u, 0u);
      } else {
        uint32_t ea[4], eb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool in = tb && u0 + q < w1;
          ea[q] = (in && va) ? __ldg(sa + b * tstride + u0 + q) : 0u;
          eb[q] = (in && vb) ? __ldg(sb + b * tstride + u0 + q) : 0u;
        }
        s_a[b] = make_uint4(ea[0], ea[1], ea[2], ea[3]);
        s_b[b] = make_uint4(eb[0], eb[1], eb[2], eb[3]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      mma_m16n8k16_bf16(base, wa[q].x, wbv[q].x, wa[q].y, wbv[q].y, xv[q].x, xv[q].y);
      mma_m16n8k16_bf16(base, wa[q].z, wbv[q].z, wa[q].w, wbv[q].w, xv[q].z, xv[q].w);
#pragma unroll
      for (int b = 0; b < kBdMaxTenants; ++b) {
        if (b < B) {   // uniform across the CTA
          const uint32_t wda = q == 0 ? s_a[b].x : q == 1 ? s_a[b].y : q == 2 ? s_a[b].z : s_a[b].w;
          const uint32_t wdb = q == 0 ? s_b[b].x : q == 1 ? s_b[b].y : q == 2 ? s_b[b].z : s_b[b].w;
          const uint32_t ga = spread_byte(~wda, t), gb = spread_byte(~wdb, t);
          mma_m16n8k16_bf16(dl[b], sign_pair(ga, 0), sign_pair(gb, 0), sign_pair(ga, 2),
                            sign_pair(gb, 2), xv[q].x, xv[q].y);
          mma_m16n8k16_bf16(dl[b], sign_pair(ga, 4), sign_pair(gb, 4), sign_pair(ga, 6),
                            sign_pair(gb, 6), xv[q].z, xv[q].w);
        }
      }
    }
  }
  // D fragment: lane (g, t) holds rows g, g+8 and columns (tenants) 2t, 2t+1.
  part[warp][0][g][2 * t] = base[0];
  part[warp][0][g][2 * t + 1] = base[1];
  part[warp][0][g + 8][2 * t] = base[2];
  part[warp][0][g + 8][2 * t + 1] = base[3];
#pragma unroll
  for (int b = 0; b < kBdMaxTenants; ++b) {
    if ((b >> 1) == t) {
      const int e = b & 1;
      part[warp][1][g][b] = dl[b][e];
      part[warp][1][g + 8][b] = dl[b][2 + e];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 16 * B; idx += blockDim.x) {
    const int r = idx & 15, b = idx >> 4;
    const int64_t n = r0 + r;
    if (n >= N) continue;
    float sb_ = 0.f, sd = 0.f;
#pragma unroll
    for (int w = 0; w < kBdWarps; ++w) {
      sb_ = __fadd_rn(sb_, part[w][0][r][b]);
      sd = __fadd_rn(sd, part[w][1][r][b]);
    }
    const float v = __fmaf_rn(alpha[b], sd, sb_);
    const int64_t o = static_cast<int64_t>(b) * N + n;
    if (y_bf16)
      reinterpret_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(y)[o] = v;
  }
}

}  // namespace bitnet
