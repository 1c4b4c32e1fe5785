// gemv.cuh -- decode-path ternary matmul (M <= 16 tokens) plus fused dequant,
// for one problem or a group of independent problems in a single launch.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// sections 計算パラダイム (integer accumulation), 推論最適化とカスタムカーネル
// (weights unpacked on the fly inside the matmul) and タイル化行列乗算 (tiles
// staged in fast shared memory so global memory is read once), 量子化の仕組み
// (rescale by both scales).
//
// Design (HBM-bound: the packed weights are the traffic):
//   * A CTA owns 16 consecutive weight rows and a range of K.  At entry one
//     thread issues one 1-D bulk async copy per row, straight from HBM into
//     shared memory (rows padded by 16 bytes so fragment reads are
//     conflict-free) -- before waiting on the preceding activation-quant
//     grid, so the weight stream overlaps it (programmatic dependent launch).
//   * Four warps split the CTA's 256-k steps.  A lane (4g + t) takes the
//     16 packed bytes (64 k) of rows g and g+8 at offset 64t of a step, and
//     unpacks them in registers with shift + mask: (P >> 2r) & 0x03030303 is
//     a word of four int8 codes t+1 for k = 4i + r of a 16-k group.  The
//     activations are stored k-interleaved (byte 4r+i of each 16-group holds
//     k = 4i+r), so the matching activation word is a plain 4-byte load.
//   * Tensor cores via warp-level int8 MMA m16n8k32 in swap-AB form: the 16
//     weight rows are the MMA's M, up to 16 tokens its N (one or two n8
//     tiles).  sum x*(t+1) minus the token's row sum sum x gives sum x*t.
//   * Warps combine through shared memory; the CTA writes
//     y = acc / (s_x * s_w) directly.  Only when a problem has too few row
//     blocks to fill the GPU is K split across CTAs: partials go to an int32
//     workspace with atomics and the last CTA of a row block (arrival counter,
//     no waiting) reads them back, re-zeroes them and finishes.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kGemvRows = 16;        // weight rows per CTA
constexpr int kGemvWarps = 4;        // warps per CTA
constexpr int kGemvMaxIps = 64;      // max 256-k steps per CTA (16 Ki of k)
constexpr int kGemvMaxGroup = 16;    // problems per grouped launch
constexpr uint32_t kCodeMask = 0x03030303u;

struct GemvProblem {
  const uint8_t* Wp;      // [N][K/4]
  const int8_t* xi;       // [M][K] k-interleaved activations
  const int32_t* rowsum;  // [M]
  const float* s_x;       // [M] (null: no dequant)
  const float* s_w;       // [1] (null: no dequant)
  void* y;                // [M][N] fp32 or bf16, may be null
  int32_t* acc_out;       // [M][N] debug accumulators, may be null
  int32_t* ws_acc;        // [M][N] split-K partials, zero on entry (ksplit > 1)
  unsigned* ws_cnt;       // [rb] arrival counters, zero on entry (ksplit > 1)
  int M, N, K;
  int y_bf16;
  int rb;                 // row blocks = ceil(N / 16)
  int ksplit;             // CTAs along K
  int ips;                // 256-k steps per CTA
  int block_begin;        // first block of this problem in the launch
};

struct GemvLaunch {
  int count;              // problems in this launch
  int use_pdl;            // wait for the preceding grid before reading activations
  int early_weights;      // start the weight copies before that wait
  int* status;            // device status word (bounded waits)
  uint64_t wait_limit_ns;
  GemvProblem prob[kGemvMaxGroup];
};

// Shared-memory row stride (bytes) of a problem's weight slice.
__host__ __device__ constexpr int gemv_row_stride(int ips) { return ips * 64 + 16; }

__device__ __forceinline__ void gemv_finish(const GemvProblem& p, float sw, int m, int n,
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

// Issue the bulk copies of this CTA's weight slice (one per existing row).
__device__ __forceinline__ void gemv_issue_weights(const GemvProblem& p, uint8_t* wt, int n0,
                                                   int k0, int k1, uint64_t* bar) {
  const int64_t rowbytes = p.K >> 2;
  const uint32_t slice = static_cast<uint32_t>((k1 - k0) >> 2);
  const int rows = min(kGemvRows, p.N - n0);
  mbar_arrive_expect_tx(bar, slice * static_cast<uint32_t>(rows));
  const int stride = gemv_row_stride(p.ips);
  for (int r = 0; r < rows; ++r)
    bulk_load(wt + r * stride, p.Wp + (n0 + r) * rowbytes + (k0 >> 2), slice, bar);
}

__global__ void __launch_bounds__(kGemvWarps * 32)
ternary_gemv_kernel(const __grid_constant__ GemvLaunch L) {
  extern __shared__ __align__(16) uint8_t wt[];  // [16][row stride]
  __shared__ int red[kGemvRows * 16];            // [row][token]
  __shared__ __align__(8) uint64_t bar;
  __shared__ int is_last;

  // Which problem and tile this CTA works on.
  int pi = 0;
  for (int i = 1; i < L.count; ++i)
    if (static_cast<int>(blockIdx.x) >= L.prob[i].block_begin) pi = i;
  const GemvProblem& p = L.prob[pi];
  const int local = static_cast<int>(blockIdx.x) - p.block_begin;
  const int rbi = local % p.rb, ks = local / p.rb;
  const int n0 = rbi * kGemvRows;
  const int total_iters = (p.K + 255) >> 8;
  const int it0 = ks * p.ips;
  const int it1 = min(it0 + p.ips, total_iters);
  const int k0 = it0 * 256, k1 = min(it1 * 256, p.K);
  const int stride = gemv_row_stride(p.ips);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  for (int i = tid; i < kGemvRows * 16; i += blockDim.x) red[i] = 0;
  __syncthreads();
  // The preceding grid never writes the weights when early_weights is set.
  if (tid == 0 && L.early_weights) gemv_issue_weights(p, wt, n0, k0, k1, &bar);
  if (L.use_pdl) pdl_wait_prior_grid();
  if (tid == 0 && !L.early_weights) gemv_issue_weights(p, wt, n0, k0, k1, &bar);

  const int ntiles = (p.M + 7) >> 3;  // 1 or 2 token tiles
  int acc[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[nt][j] = 0;

  bool weights_ready = false;
  bool ok = true;
  for (int it = it0 + warp; it < it1; it += kGemvWarps) {
    const int kseg = it * 256 + 64 * t;  // first k of this lane's 64-k segment
    const bool kval = kseg < p.K;        // K % 64 == 0: a segment is all in or all out
    // Activation fragments for tokens g and 8+g straight from L2.
    uint4 bx[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int tok = 8 * nt + g;
      const bool v = kval && nt < ntiles && tok < p.M;
      const int8_t* src = p.xi + static_cast<int64_t>(tok) * p.K + kseg;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        bx[nt][q] = v ? ldg_u4(src + 16 * q) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (!weights_ready) {
      if (!mbar_wait_bounded(&bar, 0u, nullptr, L.wait_limit_ns)) {
        record_failure(L.status, DEV_TIMEOUT_GEMV);
        ok = false;
        break;
      }
      weights_ready = true;
    }
    uint4 pa = make_uint4(0u, 0u, 0u, 0u), pb = make_uint4(0u, 0u, 0u, 0u);
    if (kval) {
      const uint8_t* wrow = wt + (it - it0) * 64 + 16 * t;
      pa = *reinterpret_cast<const uint4*>(wrow + g * stride);
      pb = *reinterpret_cast<const uint4*>(wrow + (g + 8) * stride);
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t Pa = w == 0 ? pa.x : (w == 1 ? pa.y : (w == 2 ? pa.z : pa.w));
      const uint32_t Pb = w == 0 ? pb.x : (w == 1 ? pb.y : (w == 2 ? pb.z : pb.w));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int sh = 4 * h;
        const uint32_t a0 = (Pa >> sh) & kCodeMask;
        const uint32_t a2 = (Pa >> (sh + 2)) & kCodeMask;
        const uint32_t a1 = (Pb >> sh) & kCodeMask;
        const uint32_t a3 = (Pb >> (sh + 2)) & kCodeMask;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          if (nt < ntiles) {
            const uint32_t b0 = h ? bx[nt][w].z : bx[nt][w].x;
            const uint32_t b1 = h ? bx[nt][w].w : bx[nt][w].y;
            mma_m16n8k32_s8(acc[nt], a0, a1, a2, a3, b0, b1);
          }
        }
      }
    }
  }
  // A warp with no steps never waited: make sure the copies have landed
  // before the CTA may exit.
  if (ok && !weights_ready && it0 < it1) {
    if (!mbar_wait_bounded(&bar, 0u, nullptr, L.wait_limit_ns)) {
      record_failure(L.status, DEV_TIMEOUT_GEMV);
      ok = false;
    }
  }

  // Combine the warps' partials (integer sums: order does not matter).
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    if (nt < ntiles) {
      const int c0 = 8 * nt + 2 * t;
      atomicAdd(&red[g * 16 + c0], acc[nt][0]);
      atomicAdd(&red[g * 16 + c0 + 1], acc[nt][1]);
      atomicAdd(&red[(g + 8) * 16 + c0], acc[nt][2]);
      atomicAdd(&red[(g + 8) * 16 + c0 + 1], acc[nt][3]);
    }
  }
  const int all_ok = __syncthreads_and(ok ? 1 : 0);
  if (!all_ok) return;  // a timed-out copy: results would be garbage

  const float sw = (p.y && p.s_w) ? __ldg(p.s_w) : 0.0f;
  const int nout = kGemvRows * p.M;
  if (p.ksplit == 1) {
    for (int idx = tid; idx < nout; idx += blockDim.x) {
      const int r = idx % kGemvRows, mm = idx / kGemvRows, n = n0 + r;
      if (n < p.N) gemv_finish(p, sw, mm, n, red[r * 16 + mm]);
    }
    return;
  }
  for (int idx = tid; idx < nout; idx += blockDim.x) {
    const int r = idx % kGemvRows, mm = idx / kGemvRows, n = n0 + r;
    if (n < p.N) atomicAdd(p.ws_acc + static_cast<int64_t>(mm) * p.N + n, red[r * 16 + mm]);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0)
    is_last = (atomicAdd(p.ws_cnt + rbi, 1u) == static_cast<unsigned>(p.ksplit - 1)) ? 1 : 0;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int idx = tid; idx < nout; idx += blockDim.x) {
    const int r = idx % kGemvRows, mm = idx / kGemvRows, n = n0 + r;
    if (n < p.N) {
      const int v = atomicExch(p.ws_acc + static_cast<int64_t>(mm) * p.N + n, 0);
      gemv_finish(p, sw, mm, n, v);
    }
  }
  if (tid == 0) p.ws_cnt[rbi] = 0u;  // ready for the next call
}

}  // namespace bitnet
