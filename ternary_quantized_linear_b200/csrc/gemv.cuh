// gemv.cuh -- decode-path ternary matmul (M <= 16 tokens) plus fused dequant,
// for one problem or a group of independent problems in a single launch.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// sections 計算パラダイム (integer accumulation), 推論最適化とカスタムカーネル
// (weights unpacked on the fly inside the matmul) and タイル化行列乗算 (tiles
// staged in fast shared memory so global memory is read once), 量子化の仕組み
// (rescale by both scales).
//
// The decode matmul is HBM-bound: the packed weights are the traffic.
//   * A CTA owns 64 consecutive weight rows and a range of K, streamed in
//     512-k steps through a STAGES-deep shared-memory ring by one producer
//     thread with TMA: the packed weight tile (64 rows x 128 bytes, 128-byte
//     swizzle) and the k-interleaved activation tile (MT tokens x 512 bytes as
//     four 128-byte swizzle atoms).  The weight copies of the first stages are
//     issued before waiting on the preceding activation-quant grid
//     (programmatic dependent launch), so the weight stream overlaps it.
//   * Eight compute warps touch only shared memory: warp w takes row group
//     w % 4 (16 rows) and half w / 4 (256 k) of every step.  A lane (4g + t)
//     reads 16 packed bytes (64 k) of rows g and g+8 and unpacks them in
//     registers with shift + mask: (P >> 2r) & 0x03030303 is a word of four
//     int8 codes t+1 for k = 4i + r of a 16-k group.  The activations are
//     stored k-interleaved (byte 4r+i of each 16-group holds k = 4i+r), so
//     the matching activation word is a plain 4-byte read.
//   * Warp-level int8 MMA m16n8k32 in swap-AB form: 16 weight rows are the
//     MMA's M, up to 16 tokens its N (one or two n8 tiles).  sum x*(t+1) minus
//     the token's row sum sum x gives sum x*t exactly.
//   * The two halves combine through shared memory; the CTA writes
//     y = acc / (s_x * s_w).  Only when the launch has too few row blocks to
//     fill the GPU is K split across CTAs: partials go to an int32 workspace
//     with atomics and the last CTA of a row block (arrival counter, no
//     waiting) reads them back, re-zeroes them and finishes.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kGemvRows = 64;        // weight rows per CTA
constexpr int kGemvComputeWarps = 8;
constexpr int kGemvThreads = 32 * (kGemvComputeWarps + 1);  // + producer warp
constexpr int kGemvKStep = 512;      // k per pipeline step
constexpr int kGemvStages = 6;
constexpr int kGemvMaxGroup = 16;    // problems per grouped launch
constexpr int kGemvWBytes = kGemvRows * (kGemvKStep / 4);   // 8 KiB packed weights / step
constexpr uint32_t kCodeMask = 0x03030303u;

// Shared memory of one CTA for MT token rows (8 or 16).
__host__ __device__ constexpr int gemv_x_bytes(int mt) { return mt * kGemvKStep; }
__host__ __device__ constexpr int gemv_smem_bytes(int mt) {
  return kGemvStages * (kGemvWBytes + gemv_x_bytes(mt)) + 1024;  // + alignment slack
}

struct GemvProblem {
  CUtensorMap tmap_w;     // W_packed [N][K/4] bytes, box 128 x 64 rows, 128-byte swizzle
  CUtensorMap tmap_x;     // x_q interleaved [M][K], box 128 x MT rows, 128-byte swizzle
  const int32_t* rowsum;  // [M]
  const float* s_x;       // [M] (null: no dequant)
  const float* s_w;       // [1] (null: no dequant)
  void* y;                // [M][N] fp32 or bf16, may be null
  int32_t* acc_out;       // [M][N] debug accumulators, may be null
  int32_t* ws_acc;        // [M][N] split-K partials, zero on entry (ksplit > 1)
  unsigned* ws_cnt;       // [rb] arrival counters, zero on entry (ksplit > 1)
  int M, N, K;
  int y_bf16;
  int rb;                 // row blocks = ceil(N / 64)
  int ksplit;             // CTAs along K
  int steps;              // 512-k steps per CTA
  int block_begin;        // first block of this problem in the launch
};

struct GemvLaunch {
  GemvProblem prob[kGemvMaxGroup];
  int count;              // problems in this launch
  int mt;                 // token rows per activation tile (8 or 16)
  int use_pdl;            // wait for the preceding grid before reading activations
  int early_weights;      // start the weight copies before that wait
  int* status;            // device status word (bounded waits)
  uint64_t wait_limit_ns;
};

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

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__global__ void __launch_bounds__(kGemvThreads)
ternary_gemv_kernel(const __grid_constant__ GemvLaunch L) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full[kGemvStages];
  __shared__ __align__(8) uint64_t empty[kGemvStages];
  __shared__ int red[kGemvRows * 16];  // [row][token]
  __shared__ volatile int abort_flag;
  __shared__ int is_last;

  // Which problem and tile this CTA works on.
  int pi = 0;
  for (int i = 1; i < L.count; ++i)
    if (static_cast<int>(blockIdx.x) >= L.prob[i].block_begin) pi = i;
  const GemvProblem& p = L.prob[pi];
  const int local = static_cast<int>(blockIdx.x) - p.block_begin;
  const int rbi = local % p.rb, ks = local / p.rb;
  const int n0 = rbi * kGemvRows;
  const int total_steps = (p.K + kGemvKStep - 1) / kGemvKStep;
  const int j0 = ks * p.steps;
  const int nsteps = min(p.steps, total_steps - j0);
  const int mt = L.mt;
  const int xbytes = gemv_x_bytes(mt);
  uint8_t* ws = smem;                                  // [stages][64 rows][128 B]
  uint8_t* xs = smem + kGemvStages * kGemvWBytes;      // [stages][4 atoms][mt][128 B]
  const uint64_t limit = L.wait_limit_ns;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int s = 0; s < kGemvStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvComputeWarps);
    }
    abort_flag = 0;
    fence_mbarrier_init();
  }
  for (int i = tid; i < kGemvRows * 16; i += blockDim.x) red[i] = 0;
  __syncthreads();

  if (warp == kGemvComputeWarps) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmap_w);
      tma_prefetch_desc(&p.tmap_x);
      const int pre = min(nsteps, kGemvStages);
      const bool early = L.early_weights != 0;
      if (early) {
        // The preceding grid never writes the weights (the host guarantees
        // it), so the first stages' weight copies start before waiting on it.
        for (int j = 0; j < pre; ++j) {
          mbar_expect_tx(&full[j], kGemvWBytes);
          tma_load_2d(ws + j * kGemvWBytes, &p.tmap_w, (j0 + j) * (kGemvKStep / 4), n0, &full[j]);
        }
      }
      if (L.use_pdl) pdl_wait_prior_grid();
      int issued = 0;
      for (int j = 0; j < nsteps; ++j) {
        const int s = j % kGemvStages;
        if (j >= kGemvStages &&
            !mbar_wait_bounded(&empty[s], static_cast<uint32_t>(j / kGemvStages - 1) & 1u,
                               &abort_flag, limit)) {
          abort_flag = 1;
          record_failure(L.status, DEV_TIMEOUT_GEMV);
          break;
        }
        const bool w_done = early && j < pre;
        mbar_arrive_expect_tx(&full[s], (w_done ? 0u : kGemvWBytes) + static_cast<uint32_t>(xbytes));
        if (!w_done)
          tma_load_2d(ws + s * kGemvWBytes, &p.tmap_w, (j0 + j) * (kGemvKStep / 4), n0, &full[s]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
          tma_load_2d(xs + s * xbytes + a * mt * 128, &p.tmap_x, (j0 + j) * kGemvKStep + 128 * a,
                      0, &full[s]);
        issued = j + 1;
      }
      if (abort_flag) {
        // Let the copies already in flight land before the CTA exits.
        const int first = max(0, issued - kGemvStages);
        for (int j = first; j < max(issued, early ? pre : 0); ++j)
          if (!mbar_wait_bounded(&full[j % kGemvStages], static_cast<uint32_t>(j / kGemvStages) & 1u,
                                 nullptr, limit))
            record_failure(L.status, DEV_TIMEOUT_DRAIN);
      }
    }
  } else {
    // -------------------------------------------------------------- compute
    const int g = lane >> 2, t = lane & 3;
    const int rg = warp & 3, kh = warp >> 2;
    const int ntiles = (p.M + 7) >> 3;  // 1 or 2 token tiles
    int acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[nt][j] = 0;
    // Swizzled 16-byte chunk offsets (row % 8 == g for every row and token
    // this lane touches).
    const int wchunk = 16 * ((4 * kh + t) ^ g);
    const int xatom = (2 * kh + (t >> 1)) * mt * 128;
    const int wrow_a = (16 * rg + g) * 128, wrow_b = (16 * rg + g + 8) * 128;
    for (int j = 0; j < nsteps; ++j) {
      const int s = j % kGemvStages;
      // The MMAs below are warp-collective: every lane must reach them, so
      // the wait verdict is made uniform across the warp.
      const bool got = mbar_wait_bounded(&full[s], static_cast<uint32_t>(j / kGemvStages) & 1u,
                                         &abort_flag, limit);
      if (!__all_sync(0xFFFFFFFFu, got)) {
        abort_flag = 1;
        if (lane == 0) record_failure(L.status, DEV_TIMEOUT_GEMV);
        break;
      }
      // This lane's 64-k segment: k = (j0 + j) * 512 + 256 kh + 64 t.  Lanes
      // past K (the last step) feed zero codes and zero activations; they
      // still execute every MMA.
      const bool kval = (j0 + j) * kGemvKStep + 256 * kh + 64 * t < p.K;
      const uint8_t* wst = ws + s * kGemvWBytes;
      const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
      const uint4 pa = kval ? *reinterpret_cast<const uint4*>(wst + wrow_a + wchunk) : zero4;
      const uint4 pb = kval ? *reinterpret_cast<const uint4*>(wst + wrow_b + wchunk) : zero4;
      const uint8_t* xst = xs + s * xbytes + xatom;
      uint4 bx[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          bx[nt][q] = (kval && nt < ntiles)
                          ? *reinterpret_cast<const uint4*>(
                                xst + (8 * nt + g) * 128 + 16 * ((4 * (t & 1) + q) ^ g))
                          : zero4;
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
            if (nt < ntiles) {  // uniform: depends on M only
              const uint32_t b0 = h ? bx[nt][w].z : bx[nt][w].x;
              const uint32_t b1 = h ? bx[nt][w].w : bx[nt][w].y;
              mma_m16n8k32_s8(acc[nt], a0, a1, a2, a3, b0, b1);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // Combine the two k halves (integer sums: order does not matter).
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (nt < ntiles) {
        const int r0 = 16 * rg + g, c0 = 8 * nt + 2 * t;
        atomicAdd(&red[r0 * 16 + c0], acc[nt][0]);
        atomicAdd(&red[r0 * 16 + c0 + 1], acc[nt][1]);
        atomicAdd(&red[(r0 + 8) * 16 + c0], acc[nt][2]);
        atomicAdd(&red[(r0 + 8) * 16 + c0 + 1], acc[nt][3]);
      }
    }
  }
  const int all_ok = __syncthreads_and(abort_flag == 0 ? 1 : 0);
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
