// act_quant.cuh -- fused RMSNorm + per-token absmax int8 activation
// quantization, one CTA of 256 threads per token row.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// section 量子化の仕組み (activations: per-token absmax to 8 bits in
// [-128, 127] after a normalisation); "[論文レビュー] The Era of 1-bit LLMs",
// section 提案手法 (RMSNorm); bitnet.cpp article (unite.ai), section 数学的基礎
// item 2 (infinity-norm scale; its epsilon has no value on the page, read here
// as a 1e-5 floor on max|x_n|).
//
// Bit-exactness: the row's sum of squares uses a fixed order -- element k
// feeds partial (k/8) mod 256 through a fused multiply-add in increasing k
// (thread t owns the 8-element chunks t, t+256, ...), then partial i absorbs
// partial i+s for s = 128, ..., 1 -- and every other step is one correctly
// rounded IEEE operation (explicit _rn intrinsics; no fast-math).  The max
// and the integer row sum do not depend on order.
//
// Outputs: x_q in natural k order, or "k-interleaved" for the matmul kernels:
// inside every 16-element group G the byte at 16G + 4r + i holds x_q at
// k = 16G + 4i + r.  That matches how the matmul kernels unpack 2-bit codes
// (mask-and-shift of a 32-bit word of 16 codes yields four words holding the
// codes with k = 4i + r for a fixed r), so integer dot products pair the same
// k on both sides.  rowsum[m] = sum_k x_q[m,k] lets the matmul use the raw
// codes t+1 in {0,1,2} and subtract rowsum afterwards.  The decode matmul
// additionally wants its 16-byte blocks permuted inside every 256-byte span
// (see x_block_pos) so that its shared-memory reads hit distinct banks.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kActThreads = 256;

__device__ __forceinline__ void load_gamma8(const float* gamma, int64_t k, float (&g)[8]) {
  if (gamma) {
    const float4* p = reinterpret_cast<const float4*>(gamma + k);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
    g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) g[j] = 1.0f;
  }
}

// Quantized bytes of one 8-element chunk packed little-endian into two words.
struct Chunk8 {
  uint32_t lo, hi;  // bytes k+0..3, k+4..7
};

// Store one chunk of quantized values.  In interleaved mode the two threads
// (lanes l and l^1) holding the halves of a 16-element group swap four bytes
// each so that every lane writes 8 contiguous output bytes.  All 32 lanes of
// the warp must call this (valid or not).
// perm: -1 keeps the block order; 0 / 1 applies x_block_pos with that
// token parity.
// cs: bytes from one 256-element chunk of the row to the next (256 for a
// plain row; M * 256 for the decode-tiled layout, where chunk c of every
// token row sits together).
template <bool kInterleave>
__device__ __forceinline__ void store_chunk8(int8_t* xq_row, int64_t k, Chunk8 c, bool valid,
                                             int perm = -1, int64_t cs = 256) {
  if (!kInterleave) {
    if (valid) *reinterpret_cast<uint2*>(xq_row + k) = make_uint2(c.lo, c.hi);
    return;
  }
  if (perm >= 0)
    k = (k & ~static_cast<int64_t>(255)) +
        16 * x_block_pos(static_cast<int>((k & 255) >> 4), perm) + (k & 15);
  k = (k >> 8) * cs + (k & 255);
  const int h = static_cast<int>((k >> 3) & 1);   // which half of the 16-group
  // A = bytes (q0, q4, q1, q5), B = (q2, q6, q3, q7) of this half.
  const uint32_t A = __byte_perm(c.lo, c.hi, 0x5140);
  const uint32_t B = __byte_perm(c.lo, c.hi, 0x7362);
  const uint32_t send = h ? A : B;
  const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
  const uint32_t lo = h ? recv : A;   // half 0 contribution
  const uint32_t hi = h ? B : recv;   // half 1 contribution
  const uint32_t w0 = __byte_perm(lo, hi, 0x5410);
  const uint32_t w1 = __byte_perm(lo, hi, 0x7632);
  // half h writes bytes [8h, 8h+8) of the group, which start at element k
  if (valid) *reinterpret_cast<uint2*>(xq_row + k) = make_uint2(w0, w1);
}

__device__ __forceinline__ int8_t quant_one(float xn, float sx) {
  float q = rintf(__fmul_rn(xn, sx));
  q = fminf(fmaxf(q, -128.0f), 127.0f);
  return static_cast<int8_t>(static_cast<int>(q));
}

__device__ __forceinline__ uint32_t pack4(int8_t a, int8_t b, int8_t c, int8_t d) {
  return (static_cast<uint32_t>(static_cast<uint8_t>(a))) |
         (static_cast<uint32_t>(static_cast<uint8_t>(b)) << 8) |
         (static_cast<uint32_t>(static_cast<uint8_t>(c)) << 16) |
         (static_cast<uint32_t>(static_cast<uint8_t>(d)) << 24);
}

// Block-wide sum of squares in the canonical tree order; result valid in
// all threads.
__device__ __forceinline__ float block_tree_sum_f32(float p, float* red) {
  const int tid = threadIdx.x;
  red[tid] = p;
  __syncthreads();
#pragma unroll
  for (int s = 128; s >= 32; s >>= 1) {
    if (tid < s) red[tid] = __fadd_rn(red[tid], red[tid + s]);
    __syncthreads();
  }
  if (tid < 32) {
    float v = red[tid];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v = __fadd_rn(v, __shfl_down_sync(0xFFFFFFFFu, v, s));
    if (tid == 0) red[0] = v;
  }
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_max_f32(float v, float* red) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, s));
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  if (tid < 32) {
    float w = (tid < kActThreads / 32) ? red[tid] : 0.0f;
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) w = fmaxf(w, __shfl_xor_sync(0xFFFFFFFFu, w, s));
    if (tid == 0) red[0] = w;
  }
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

// block_tree_sum_f32 of p (same order, same result) and the block max of m
// through the same barriers.
__device__ __forceinline__ float2 block_sum_max_f32(float p, float m, float* red, int* redm) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));
  red[tid] = p;
  if ((tid & 31) == 0) redm[tid >> 5] = __float_as_int(m);
  __syncthreads();
#pragma unroll
  for (int s = 128; s >= 32; s >>= 1) {
    if (tid < s) red[tid] = __fadd_rn(red[tid], red[tid + s]);
    __syncthreads();
  }
  if (tid < 32) {
    float v = red[tid];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v = __fadd_rn(v, __shfl_down_sync(0xFFFFFFFFu, v, s));
    float w = (tid < kActThreads / 32) ? __int_as_float(redm[tid]) : 0.0f;
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) w = fmaxf(w, __shfl_xor_sync(0xFFFFFFFFu, w, s));
    if (tid == 0) {
      red[0] = v;
      redm[0] = __float_as_int(w);
    }
  }
  __syncthreads();
  const float2 r = make_float2(red[0], __int_as_float(redm[0]));
  __syncthreads();
  return r;
}

__device__ __forceinline__ int block_sum_i32(int v, int* red) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, s);
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  int r = 0;
#pragma unroll
  for (int i = 0; i < kActThreads / 32; ++i) r += red[i];
  __syncthreads();
  return r;
}

// Clear n16 16-byte words at dst using `nblocks` CTAs; this CTA is number
// `block` among them.  Used by blocks appended to a row-per-block launch to
// zero the matmul's split-K partials and counters without a memset launch.
__device__ __forceinline__ void zero_fill_blocks(uint4* __restrict__ dst, int64_t n16,
                                                 int64_t block, int64_t nblocks) {
  for (int64_t i = block * kActThreads + threadIdx.x; i < n16; i += nblocks * kActThreads)
    dst[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Raw bytes of one 8-element chunk (bf16: one 16-byte word; fp32: two).
template <bool kBF16>
struct RawChunk {
  uint4 w[kBF16 ? 1 : 2];
};

template <bool kBF16>
__device__ __forceinline__ RawChunk<kBF16> load_raw8(const void* x, int64_t elem) {
  RawChunk<kBF16> r;
  if (kBF16) {
    r.w[0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + elem));
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(x) + elem);
    r.w[0] = __ldg(p);
    r.w[kBF16 ? 0 : 1] = __ldg(p + 1);
  }
  return r;
}

template <bool kBF16>
__device__ __forceinline__ void widen8(const RawChunk<kBF16>& r, float (&v)[8]) {
  if (kBF16) {
    const uint32_t w[4] = {r.w[0].x, r.w[0].y, r.w[0].z, r.w[0].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
    const uint4 a = r.w[0], b = r.w[kBF16 ? 0 : 1];
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
    v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
    v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
  }
}

// RMSNorm + absmax quantization of row m of x [M][K] by the whole CTA.
// Thread t owns the 8-element chunks t, t+256, ...; with CACHE > 0 (and at
// most CACHE chunks per thread) the row is loaded once into registers with
// all loads in flight together, otherwise each pass re-reads it (L1 hits).
template <bool kBF16, bool kInterleave, int CACHE>
__device__ __forceinline__ void quant_row(const void* __restrict__ x,
                                          const float* __restrict__ gamma, float eps, int64_t m,
                                          int64_t K, int8_t* __restrict__ x_q,
                                          float* __restrict__ s_x, int32_t* __restrict__ rowsum,
                                          float* redf, int* redi, bool perm = false,
                                          int64_t M_tiled = 0) {
  const int tid = threadIdx.x;
  const int64_t nchunk = K >> 3;
  const int iters = static_cast<int>((nchunk + kActThreads - 1) / kActThreads);
  const int64_t row = m * K;
  constexpr int CN = CACHE > 0 ? CACHE : 1;
  RawChunk<kBF16> cache[CN];
  if (CACHE > 0) {
#pragma unroll
    for (int it = 0; it < CN; ++it) {
      const int64_t c = tid + static_cast<int64_t>(kActThreads) * it;
      if (it < iters && c < nchunk) cache[it] = load_raw8<kBF16>(x, row + 8 * c);
    }
  }
  auto chunk = [&](int it, int64_t c, float (&v)[8]) {
    if (CACHE > 0) {
#pragma unroll
      for (int u = 0; u < CN; ++u)
        if (u == it) widen8<kBF16>(cache[u], v);
    } else {
      widen8<kBF16>(load_raw8<kBF16>(x, row + 8 * c), v);
    }
  };

  // Pass 1: sum of squares, partial = this thread's chunks in increasing k.
  float p = 0.0f;
#pragma unroll
  for (int it = 0; it < (CACHE > 0 ? CN : 1); ++it) {
    for (int it2 = it; it2 < (CACHE > 0 ? it + 1 : iters); ++it2) {
      const int64_t c = tid + static_cast<int64_t>(kActThreads) * it2;
      if (it2 < iters && c < nchunk) {
        float v[8];
        chunk(it2, c, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) p = __fmaf_rn(v[j], v[j], p);
      }
    }
  }
  const float ss = block_tree_sum_f32(p, redf);
  const float ms = __fdiv_rn(ss, static_cast<float>(K));
  const float d = __fadd_rn(ms, eps);
  const bool zero_row = (d == 0.0f);
  const float r = zero_row ? 0.0f : __fdiv_rn(1.0f, __fsqrt_rn(d));

  // Pass 2: max |x_n|.
  float amax = 0.0f;
#pragma unroll
  for (int it = 0; it < (CACHE > 0 ? CN : 1); ++it) {
    for (int it2 = it; it2 < (CACHE > 0 ? it + 1 : iters); ++it2) {
      const int64_t c = tid + static_cast<int64_t>(kActThreads) * it2;
      if (it2 < iters && c < nchunk && !zero_row) {
        float v[8], g[8];
        chunk(it2, c, v);
        load_gamma8(gamma, 8 * c, g);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(v[j], r), g[j])));
      }
    }
  }
  amax = block_max_f32(amax, redf);
  amax = fmaxf(amax, 1e-5f);
  const float sx = __fdiv_rn(127.0f, amax);

  // Pass 3: quantize, store, row sum (every lane runs every iteration: the
  // interleaved store exchanges bytes between lane pairs).
  int sum = 0;
  const bool tiled = M_tiled > 0;   // decode-tiled layout, as in quant_row_staged
  int8_t* xq_row = tiled ? x_q + m * 256 : x_q + row;
  const int64_t cs = tiled ? M_tiled * 256 : 256;
  const int64_t nstore = tiled ? ((K + 255) >> 8) << 5 : nchunk;
  const int store_iters = static_cast<int>((nstore + kActThreads - 1) / kActThreads);
#pragma unroll
  for (int it = 0; it < (CACHE > 0 ? CN : 1); ++it) {
    for (int it2 = it; it2 < (CACHE > 0 ? it + 1 : store_iters); ++it2) {
      if (it2 >= store_iters) continue;  // uniform over the CTA
      const int64_t c = tid + static_cast<int64_t>(kActThreads) * it2;
      const bool valid = c < nstore;
      int8_t q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (c < nchunk && !zero_row) {
        float v[8], g[8];
        chunk(it2, c, v);
        load_gamma8(gamma, 8 * c, g);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          q[j] = quant_one(__fmul_rn(__fmul_rn(v[j], r), g[j]), sx);
          sum += q[j];
        }
      }
      Chunk8 ch{pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7])};
      store_chunk8<kInterleave>(xq_row, 8 * c, ch, valid, perm ? static_cast<int>(m & 1) : -1,
                                cs);
    }
  }
  sum = block_sum_i32(sum, redi);
  if (tid == 0) {
    if (s_x) s_x[m] = sx;
    if (rowsum) rowsum[m] = sum;
  }
}

// Shared-memory bytes to stage a row (and gamma) of K elements; rows above
// kQuantStageMax take the re-reading path instead.
constexpr uint32_t kQuantStageMax = 160u << 10;
__host__ __device__ constexpr uint32_t quant_stage_bytes(int64_t K, bool bf16, bool gamma) {
  return static_cast<uint32_t>(K * ((bf16 ? 2 : 4) + (gamma ? 4 : 0)));
}

// RMSNorm + absmax quantization of row m, staged: one thread brings the row
// (and gamma) into shared memory with bulk asynchronous copies, then three
// short loops read it there.  The executed code stays small, which matters:
// each row's CTA usually runs alone on an SM with a cold instruction cache.
// Same arithmetic and reduction order as quant_row.  Returns false (nothing
// written) when the copy did not land within the wait limit.
template <bool kBF16, bool kInterleave>
__device__ bool quant_row_staged(const void* __restrict__ x, const float* __restrict__ gamma,
                                 float eps, int64_t m, int64_t K, int8_t* __restrict__ x_q,
                                 float* __restrict__ s_x, int32_t* __restrict__ rowsum,
                                 float* redf, int* redi, uint8_t* stage, uint64_t* bar,
                                 uint64_t wait_limit_ns, bool perm, int64_t M_tiled = 0) {
  constexpr int ES = kBF16 ? 2 : 4;
  const int tid = threadIdx.x;
  const uint32_t xbytes = static_cast<uint32_t>(K * ES);
  const float* sg = reinterpret_cast<const float*>(stage + xbytes);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, xbytes + (gamma ? static_cast<uint32_t>(K * 4) : 0u));
    bulk_load(stage, static_cast<const uint8_t*>(x) + m * K * ES, xbytes, bar);
    if (gamma) bulk_load(stage + xbytes, gamma, static_cast<uint32_t>(K * 4), bar);
  }
  const bool landed = mbar_wait_bounded(bar, 0u, nullptr, wait_limit_ns);
  if (!__syncthreads_and(landed ? 1 : 0)) return false;

  const int64_t nchunk = K >> 3;
  auto chunk = [&](int64_t c, float (&v)[8]) {
    RawChunk<kBF16> r;
    const uint4* src = reinterpret_cast<const uint4*>(stage + c * 8 * ES);
    r.w[0] = src[0];
    if (!kBF16) r.w[kBF16 ? 0 : 1] = src[1];
    widen8<kBF16>(r, v);
  };
  auto gam = [&](int64_t c, float (&g)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) g[j] = gamma ? sg[8 * c + j] : 1.0f;
  };

  // Pass 1: sum of squares, partial = this thread's chunks in increasing k;
  // without gamma also max |x| (then max |x_n| = max |x| * r exactly: a
  // correctly rounded product is monotonic in |x|).
  float p = 0.0f, xmax = 0.0f;
#pragma unroll 1
  for (int64_t c = tid; c < nchunk; c += kActThreads) {
    float v[8];
    chunk(c, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      p = __fmaf_rn(v[j], v[j], p);
      xmax = fmaxf(xmax, fabsf(v[j]));
    }
  }
  float ss;
  if (gamma) {
    ss = block_tree_sum_f32(p, redf);
  } else {
    const float2 sm = block_sum_max_f32(p, xmax, redf, redi);
    ss = sm.x;
    xmax = sm.y;
  }
  const float ms = __fdiv_rn(ss, static_cast<float>(K));
  const float d = __fadd_rn(ms, eps);
  const bool zero_row = (d == 0.0f);
  const float r = zero_row ? 0.0f : __fdiv_rn(1.0f, __fsqrt_rn(d));

  // Pass 2 (with gamma): max |x_n|.
  float amax = 0.0f;
  if (!gamma) {
    amax = zero_row ? 0.0f : __fmul_rn(xmax, r);
  } else {
    if (!zero_row) {
#pragma unroll 1
      for (int64_t c = tid; c < nchunk; c += kActThreads) {
        float v[8], g[8];
        chunk(c, v);
        gam(c, g);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(v[j], r), g[j])));
      }
    }
    amax = block_max_f32(amax, redf);
  }
  amax = fmaxf(amax, 1e-5f);
  const float sx = __fdiv_rn(127.0f, amax);

  // Pass 3: quantize, store, row sum (every lane runs every iteration: the
  // interleaved store exchanges bytes between lane pairs).  In the
  // decode-tiled layout (M_tiled > 0) the row is stored as 256-element
  // chunks M_tiled * 256 bytes apart, its last chunk zero-padded past K.
  int sum = 0;
  const bool tiled = M_tiled > 0;
  int8_t* xq_row = tiled ? x_q + m * 256 : x_q + m * K;
  const int64_t cs = tiled ? M_tiled * 256 : 256;
  const int64_t nstore = tiled ? ((K + 255) >> 8) << 5 : nchunk;   // 8-element chunks
  const int store_iters = static_cast<int>((nstore + kActThreads - 1) / kActThreads);
#pragma unroll 1
  for (int it = 0; it < store_iters; ++it) {
    const int64_t c = tid + static_cast<int64_t>(kActThreads) * it;
    int8_t q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (c < nchunk && !zero_row) {
      float v[8], g[8];
      chunk(c, v);
      gam(c, g);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        q[j] = quant_one(__fmul_rn(__fmul_rn(v[j], r), g[j]), sx);
        sum += q[j];
      }
    }
    Chunk8 ch{pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7])};
    store_chunk8<kInterleave>(xq_row, 8 * c, ch, c < nstore, perm ? static_cast<int>(m & 1) : -1,
                              cs);
  }
  sum = block_sum_i32(sum, redi);
  if (tid == 0) {
    if (s_x) s_x[m] = sx;
    if (rowsum) rowsum[m] = sum;
  }
  return true;
}

// One CTA per row (blocks >= M zero `zero16` instead).  x: [M][K] (fp32 or
// bf16 bits), gamma: [K] or null.  STAGED: the row goes through shared
// memory (dynamic, quant_stage_bytes); otherwise each pass re-reads it.
template <bool kBF16, bool kInterleave, bool STAGED>
__global__ void __launch_bounds__(kActThreads)
rmsnorm_quant_kernel(const void* __restrict__ x, const float* __restrict__ gamma, float eps,
                     int64_t M, int64_t K, int8_t* __restrict__ x_q, float* __restrict__ s_x,
                     int32_t* __restrict__ rowsum, uint4* __restrict__ zero16, int64_t n_zero16,
                     int trigger_dependents, int* status, uint64_t wait_limit_ns, int perm,
                     int tiled) {
  __shared__ float redf[kActThreads];
  __shared__ int redi[kActThreads / 32];
  __shared__ __align__(8) uint64_t bar;
  extern __shared__ __align__(16) uint8_t stage[];
  if (trigger_dependents) pdl_launch_dependents();
  if (static_cast<int64_t>(blockIdx.x) >= M) {
    zero_fill_blocks(zero16, n_zero16, static_cast<int64_t>(blockIdx.x) - M,
                     static_cast<int64_t>(gridDim.x) - M);
    return;
  }
  if (STAGED) {
    if (!quant_row_staged<kBF16, kInterleave>(x, gamma, eps, blockIdx.x, K, x_q, s_x, rowsum,
                                              redf, redi, stage, &bar, wait_limit_ns, perm != 0,
                                              tiled ? M : 0) &&
        threadIdx.x == 0)
      record_failure(status, DEV_TIMEOUT_QUANT);
  } else {
    quant_row<kBF16, kInterleave, 0>(x, gamma, eps, blockIdx.x, K, x_q, s_x, rowsum, redf, redi,
                                     perm != 0, tiled ? M : 0);
  }
}

constexpr int kQuantMaxGroup = 16;

struct QuantProblem {
  const void* x;          // [M][K] fp32 or bf16
  const float* gamma;     // [K] or null
  int8_t* xi;             // [M][K] k-interleaved out
  float* s_x;             // [M]
  int32_t* rowsum;        // [M]
  uint4* zero16;          // region to clear (null: none)
  int64_t n_zero16;
  float eps;
  int M, K;
  int x_bf16;
  int perm;               // decode-matmul block order (x_block_pos)
  int tiled;              // decode-tiled layout: x_q [ceil(K/256)][M][256]
  int block_begin;        // first block of this problem
  int zero_blocks;        // blocks after the M row blocks that clear zero16
};

struct QuantLaunch {
  int count;
  int trigger_dependents;
  int* status;              // device status word (bounded waits)
  uint64_t wait_limit_ns;
  QuantProblem prob[kQuantMaxGroup];
};

// Several independent problems in one launch: rows of every problem, then
// each problem's zero-fill blocks, laid out by block_begin.  STAGED: every
// row of the launch fits the dynamic shared-memory stage.
template <bool STAGED>
__global__ void __launch_bounds__(kActThreads)
rmsnorm_quant_grouped_kernel(const __grid_constant__ QuantLaunch L) {
  __shared__ float redf[kActThreads];
  __shared__ int redi[kActThreads / 32];
  __shared__ __align__(8) uint64_t bar;
  extern __shared__ __align__(16) uint8_t stage[];
  if (L.trigger_dependents) pdl_launch_dependents();
  int pi = 0;
  for (int i = 1; i < L.count; ++i)
    if (static_cast<int>(blockIdx.x) >= L.prob[i].block_begin) pi = i;
  const QuantProblem& q = L.prob[pi];
  const int local = static_cast<int>(blockIdx.x) - q.block_begin;
  if (local >= q.M) {
    zero_fill_blocks(q.zero16, q.n_zero16, local - q.M, q.zero_blocks);
    return;
  }
  if (STAGED) {
    const int64_t mt = q.tiled ? q.M : 0;
    const bool ok =
        q.x_bf16 ? quant_row_staged<true, true>(q.x, q.gamma, q.eps, local, q.K, q.xi, q.s_x,
                                                q.rowsum, redf, redi, stage, &bar, L.wait_limit_ns,
                                                q.perm != 0, mt)
                 : quant_row_staged<false, true>(q.x, q.gamma, q.eps, local, q.K, q.xi, q.s_x,
                                                 q.rowsum, redf, redi, stage, &bar,
                                                 L.wait_limit_ns, q.perm != 0, mt);
    if (!ok && threadIdx.x == 0) record_failure(L.status, DEV_TIMEOUT_QUANT);
  } else if (q.x_bf16) {
    quant_row<true, true, 0>(q.x, q.gamma, q.eps, local, q.K, q.xi, q.s_x, q.rowsum, redf, redi,
                             q.perm != 0, q.tiled ? q.M : 0);
  } else {
    quant_row<false, true, 0>(q.x, q.gamma, q.eps, local, q.K, q.xi, q.s_x, q.rowsum, redf, redi,
                              q.perm != 0, q.tiled ? q.M : 0);
  }
}

// Natural-order x_q -> k-interleaved copy plus per-row sums (used when the
// caller hands in already-quantized activations).
__global__ void __launch_bounds__(kActThreads)
interleave_rowsum_kernel(const int8_t* __restrict__ x_q, int64_t M, int64_t K,
                         int8_t* __restrict__ xi, int32_t* __restrict__ rowsum,
                         uint4* __restrict__ zero16, int64_t n_zero16, int perm) {
  __shared__ int redi[kActThreads / 32];
  if (static_cast<int64_t>(blockIdx.x) >= M) {
    zero_fill_blocks(zero16, n_zero16, static_cast<int64_t>(blockIdx.x) - M,
                     static_cast<int64_t>(gridDim.x) - M);
    return;
  }
  const int tid = threadIdx.x;
  const int64_t m = blockIdx.x;
  const int64_t nchunk = K >> 3;
  const int iters = static_cast<int>((nchunk + kActThreads - 1) / kActThreads);
  int sum = 0;
  for (int it = 0; it < iters; ++it) {
    const int64_t c = tid + static_cast<int64_t>(kActThreads) * it;
    const bool valid = c < nchunk;
    Chunk8 ch{0u, 0u};
    if (valid) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(x_q + m * K + 8 * c));
      ch.lo = u.x;
      ch.hi = u.y;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sum += static_cast<int8_t>((u.x >> (8 * j)) & 0xFF);
        sum += static_cast<int8_t>((u.y >> (8 * j)) & 0xFF);
      }
    }
    store_chunk8<true>(xi + m * K, 8 * c, ch, valid, perm ? static_cast<int>(m & 1) : -1);
  }
  sum = block_sum_i32(sum, redi);
  if (tid == 0) rowsum[m] = sum;
}

}  // namespace bitnet
