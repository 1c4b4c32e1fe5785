// gemv_tiled.cuh -- decode-path ternary matmul (M <= 16 tokens) plus fused
// dequant on weights in the tiled layout (tiled.cuh), for one problem or a
// group of independent problems in a single launch.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// sections 計算パラダイム (integer accumulation), 推論最適化とカスタムカーネル
// (weights unpacked on the fly inside the matmul), タイル化行列乗算 (tiles
// staged in fast on-chip memory so global memory is read once) and
// 量子化の仕組み (rescale by both scales).
//
// The decode matmul is bound by HBM: the packed weights are the traffic.
// On B200 a thread can start a bulk copy only every few hundred nanoseconds
// whatever its size, so the copies must be large: with the tiled layout the
// weights of consecutive tiles are contiguous and move as one copy.
//   * The problems' tiles (128 rows x 256 k, 8 KiB) are laid end to end,
//     problem by problem, row block by row block; CTA b owns the contiguous
//     tile range [tile_begin[b], tile_begin[b+1]) (cost-balanced by the
//     host).  A "segment" is the part of one row block (with group-wise
//     scales: of one group of a row block) inside that range.
//   * Eight MMA warps and three producer warps, one CTA per SM.  A ring of
//     shared-memory stages, each up to 32 KiB of weights of one segment plus
//     the activations of the same k chunks.  One lane of each producer warp
//     issues one bulk copy per stage: the first half of the stage's weights,
//     the second half, and the activations (the quantized input is stored
//     chunk-major, [K/256][M][256 bytes], so those chunks are contiguous).
//     A stage is refilled once every MMA warp has read it.  Weight copies
//     start at once; activation copies wait for the preceding
//     activation-quant grid (programmatic dependent launch).
//   * Every warp takes rows 64 (w & 1) .. +63 of tile w >> 1 of a stage
//     (64 rows x 256 k), unpacks the codes in registers (mask and shift; the
//     activations are k-interleaved so a code word pairs with a plain
//     activation word; with one token tile the codes of k = 4i+2 and 4i+3
//     are kept times 16 in a second accumulator set, which saves two shifts
//     per word) and issues
//     mma.sync m16n8k32 s8 in swap-AB form (weight rows = MMA M, tokens = N,
//     one or two n8 tiles) into register accumulators that live for the
//     whole segment.  Tokens past M read some valid token's bytes: they only
//     feed accumulator columns that are never stored.  The legacy int8 MMA
//     retires about one m16n8k32 per 8 cycles per SM on this GPU, which is
//     what bounds the kernel once two token tiles are needed; a single token
//     (M = 1) would waste seven eighths of every MMA, so its segments run on
//     dp4a instead (gt_dp4a_unit) and stay bound by the weight stream.
//   * At the end of a segment the warps add their accumulators into a
//     shared 128 x 16 table (two tables, alternating) and, after a bounded
//     barrier, finish it: y = (acc - rowsum) / (s_x * s_w) for a whole row
//     block (constants fetched while the segment streams).  A part of a row
//     block (the first and last segment of a CTA's range may be parts) goes
//     to a per-CTA workspace slot with plain stores; a second, small kernel
//     (gemv_tiled_fixup_kernel) sums the slots once the grid is done -- the
//     kernel boundary orders the stores, so no fence, counter or waiting is
//     needed in the streaming kernel.
//   * Every wait is bounded; on a timeout the kernel records the failure,
//     raises a CTA abort flag, lets the copies in flight land and exits
//     without writing results.
#pragma once

#include "common.cuh"
#include "gemv.cuh"
#include "tiled.cuh"

namespace bitnet {

constexpr int kGtMmaWarps = 8;
constexpr int kGtMmaThreads = 32 * kGtMmaWarps;
constexpr int kGtThreads = kGtMmaThreads + 96;  // + two weight producer warps + one activation producer
constexpr int kGtMaxCtas = 296;
constexpr int kGtMaxGroup = 16;
constexpr int kGtWBytes = 4 * kTileBytes;   // 32 KiB of weights per stage

// Shape of the kernel's work unit.  Plain: a unit is one 128-row tile, four
// per stage.  Pair (the fused SwiGLU): a unit is the gate tile and the up
// tile of the same rows and k chunk (pair-tiled layout, 16 KiB), two per
// stage; the table then holds 256 rows (gate rows 0-127, up rows 128-255).
// NT token tiles of 8: a stage holds the activations of up to 8 NT tokens;
// with one token tile the stages are smaller and the ring one deeper.
template <bool kPair, int NT>
struct GtCfg {
  static constexpr int UNIT_BYTES = kPair ? 2 * kTileBytes : kTileBytes;
  static constexpr int UNITS = kGtWBytes / UNIT_BYTES;         // units (= k chunks) per stage
  static constexpr int TAB_ROWS = kPair ? 2 * kTileRows : kTileRows;
  static constexpr int STAGES = NT == 1 ? 5 : 4;
  static constexpr int X_BYTES = UNITS * 8 * NT * 256;
  static constexpr int STAGE_BYTES = kGtWBytes + X_BYTES;
  static constexpr int SMEM_DYN = STAGES * STAGE_BYTES + 1024;  // + alignment slack
};

struct GtProblem {
  const uint8_t* Wt;      // tiled weights
  const uint8_t* xd;      // quantized activations, chunk-major [KC][M][256] (decode block order)
  const int32_t* rowsum;  // [M]
  const float* s_x;       // [M] (null: no dequant)
  const float* s_w;       // [1] (null: no dequant); the gate's scale for a pair
  const float* s_w2;      // [1] the up projection's scale (pair only)
  void* y;                // [M][N] fp32 or bf16, may be null
  int32_t* acc_out;       // [M][N] debug accumulators, may be null
  int32_t* part;          // partial slots, 2 per contributing CTA, [M][table rows] int32
  long long tile_base;    // first tile of this problem in the launch
  int M, N, K, KC, RB;
  int y_bf16;
  int cta_first;          // first CTA whose range holds a tile of this problem
  // Group-wise scales (group_quant.cuh): gc = k chunks per group (0: one
  // per-tensor group).  Segments then end at group boundaries, rowsum is
  // [M][G], and instead of y the kernel writes every group's integer sums
  // to gacc [G][M][N].
  int gc, G;
  int32_t* gacc;
};

struct GtLaunch {
  GtProblem prob[kGtMaxGroup];
  long long tile_begin[kGtMaxCtas + 1];  // CTA b owns [tile_begin[b], tile_begin[b+1])
  int count;
  int ctas;
  int use_pdl;
  int* status;
  uint64_t wait_limit_ns;
};

// The segment that starts at tile t of a CTA range ending at t1.
struct GtSeg {
  int p, rb, c, nt;       // problem, row block, first chunk, tiles
  long long t;            // first tile
};

__device__ __forceinline__ GtSeg gt_segment(const GtProblem* prob, int count, long long t,
                                            long long t1) {
  int p = 0;
  while (p + 1 < count && t >= prob[p + 1].tile_base) ++p;
  const GtProblem& P = prob[p];
  const long long local = t - P.tile_base;
  GtSeg s;
  s.p = p;
  s.rb = static_cast<int>(local / P.KC);
  s.c = static_cast<int>(local - static_cast<long long>(s.rb) * P.KC);
  long long end = P.tile_base + static_cast<long long>(s.rb + 1) * P.KC;
  if (P.gc > 0) {   // a segment never crosses a group boundary
    const long long gend = P.tile_base + static_cast<long long>(s.rb) * P.KC +
                           (s.c / P.gc + 1) * static_cast<long long>(P.gc);
    if (gend < end) end = gend;
  }
  s.nt = static_cast<int>((t1 < end ? t1 : end) - t);
  s.t = t;
  return s;
}

// Group of a segment (0 without groups), its first tile and its tile count:
// the unit whose sums a whole segment completes and partial ones share.
struct GtSpan {
  int grp;
  long long first;
  int len;
};

__device__ __forceinline__ GtSpan gt_span(const GtProblem& P, const GtSeg& sg) {
  GtSpan sp;
  const long long rb0 = P.tile_base + static_cast<long long>(sg.rb) * P.KC;
  if (P.gc > 0) {
    sp.grp = sg.c / P.gc;
    sp.first = rb0 + static_cast<long long>(sp.grp) * P.gc;
    sp.len = P.gc;
  } else {
    sp.grp = 0;
    sp.first = rb0;
    sp.len = P.KC;
  }
  return sp;
}

// CTA whose range holds tile t (tile_begin is increasing).
__device__ __forceinline__ int gt_cta_of(const long long* tb, int ctas, long long t) {
  int lo = 0, hi = ctas - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tb[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Per-token constants of a segment's finish: row sum, divisor s_x * s_w and
// RN(1 / divisor) (for a pair also those of the second scale).
struct GtTok {
  int rs;
  float d, rd, d2, rd2;
};

__device__ __forceinline__ void gt_write(const GtProblem& P, int64_t o, float yv) {
  if (P.y_bf16)
    reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(yv);
  else
    reinterpret_cast<float*>(P.y)[o] = yv;
}

// Output n of token m from the integer sum of codes x (t + 1):
// y = (acc - rowsum) / (s_x * s_w) with the token's constants from tk (with
// group-wise scales: the group's integer sum, for the combining kernel).
__device__ __forceinline__ void gt_store(const GtProblem& P, const GtTok& tk, int m, int n,
                                         int acc_codes, int grp) {
  const int acc = acc_codes - tk.rs;
  const int64_t o = static_cast<int64_t>(m) * P.N + n;
  if (P.gacc) {
    P.gacc[static_cast<int64_t>(grp) * P.M * P.N + o] = acc;
    return;
  }
  if (P.acc_out) P.acc_out[o] = acc;
  if (P.y) gt_write(P, o, div_rn_int(__int2float_rn(acc), tk.d, tk.rd));
}

// The fused SwiGLU output: silu(gate) * up with silu(z) = z / (1 + e^-z),
// gate and up the two BitLinear outputs (fp32, bit-identical to separate
// forwards), the activation in rounded fp32 steps (expf, then IEEE add,
// divide, multiply).
__device__ __forceinline__ void gt_store_pair(const GtProblem& P, const GtTok& tk, int m, int n,
                                              int gate_codes, int up_codes) {
  const float g = div_rn_int(__int2float_rn(gate_codes - tk.rs), tk.d, tk.rd);
  const float u = div_rn_int(__int2float_rn(up_codes - tk.rs), tk.d2, tk.rd2);
  const float sg = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
  gt_write(P, static_cast<int64_t>(m) * P.N + n, __fmul_rn(sg, u));
}

// The token constants of token m of problem P for group grp (global loads).
__device__ __forceinline__ GtTok gt_token(const GtProblem& P, int m, bool pair, int grp) {
  GtTok tk;
  tk.rs = P.gc > 0 ? P.rowsum[m * P.G + grp] : P.rowsum[m];
  tk.d = P.s_w ? __fmul_rn(P.s_x[m], P.s_w[0]) : 1.0f;
  tk.rd = recip_for_div(tk.d);
  tk.d2 = (pair && P.s_w2) ? __fmul_rn(P.s_x[m], P.s_w2[0]) : 1.0f;
  tk.rd2 = recip_for_div(tk.d2);
  return tk;
}

// Barrier among the MMA warps on an mbarrier (count = kGtMmaWarps), so that
// it can give up: lane 0 of each warp arrives, every lane waits on the
// phase.  Returns false on a timeout or abort (warp-uniform).
__device__ __forceinline__ bool gt_mma_sync(uint64_t* bar, uint32_t& phase,
                                            const volatile int* abort_flag, uint64_t limit) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = mbar_wait_bounded(bar, phase, abort_flag, limit);
  phase ^= 1u;
  return __all_sync(0xFFFFFFFFu, ok);
}

// The MMAs of one 64-row x 256-k unit for TILES token tiles, one
// accumulator set: the four code words of a packed word P are
// (P >> 2r) & 0x03030303 for r = 0..3 (k = 4i + r of its 16-k group), paired
// with the matching word of the k-interleaved activations.  Row groups
// innermost, so consecutive MMAs feed independent accumulators.
template <int NT, int TILES>
__device__ __forceinline__ void gt_mma_unit(int (&acc)[4][NT][4], const GemvBuf<NT>& b) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t a[4][4];  // [rg][a0 a1 a2 a3]
#pragma unroll
      for (int rg = 0; rg < 4; ++rg) {
        const uint32_t Pa = word_of(b.wa[rg], w) >> (4 * half);
        const uint32_t Pb = word_of(b.wb[rg], w) >> (4 * half);
        a[rg][0] = Pa & kCodeMask;
        a[rg][1] = Pb & kCodeMask;
        a[rg][2] = (Pa >> 2) & kCodeMask;
        a[rg][3] = (Pb >> 2) & kCodeMask;
      }
#pragma unroll
      for (int nt = 0; nt < TILES; ++nt)
#pragma unroll
        for (int rg = 0; rg < 4; ++rg)
          mma_m16n8k32_s8(acc[rg][nt], a[rg][0], a[rg][1], a[rg][2], a[rg][3],
                          word_of(b.x[nt][w], 2 * half), word_of(b.x[nt][w], 2 * half + 1));
    }
  }
}

// One 64-row x 256-k unit for a single token, on the integer dot-product
// units instead of the tensor cores (an mma.sync costs the same for one
// token as for eight, and its rate bounds this kernel).  Byte i of
// P & (3 << 2r) is the code of k = 4i + r times 4^r, so one dp4a of it with
// activation word r adds 4^r times that word's four products; each row keeps
// its four scales apart (row g in A[rg][0][r], row g + 8 in B[rg][kB][r])
// until gt_flush_one divides them out exactly.
template <int NT, int kB>
__device__ __forceinline__ void gt_dp4a_unit(int (&A)[4][NT][4], int (&B)[4][NT][4],
                                             const GemvBuf<NT>& b) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t x[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) x[r] = word_of(b.x[0][w], r);
#pragma unroll
    for (int rg = 0; rg < 4; ++rg) {
      const uint32_t Pa = word_of(b.wa[rg], w), Pb = word_of(b.wb[rg], w);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t m = kCodeMask << (2 * r);
        A[rg][0][r] = dp4a_us(Pa & m, x[r], A[rg][0][r]);
        B[rg][kB][r] = dp4a_us(Pb & m, x[r], B[rg][kB][r]);
      }
    }
  }
}

// Flush of gt_dp4a_unit's sums (the single token, column 0 of the table):
// the four scales of a row divided out (exact: each sum is a multiple of its
// 4^r), the four lanes t of a row added by shuffles, one shared-memory add
// per row; the accumulators cleared.
template <int NT, int kB>
__device__ __forceinline__ void gt_flush_one(int (&A)[4][NT][4], int (&B)[4][NT][4], int* red,
                                             int g, int t) {
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
    int va = A[rg][0][0] + (A[rg][0][1] >> 2) + (A[rg][0][2] >> 4) + (A[rg][0][3] >> 6);
    int vb = B[rg][kB][0] + (B[rg][kB][1] >> 2) + (B[rg][kB][2] >> 4) + (B[rg][kB][3] >> 6);
    va += __shfl_xor_sync(0xFFFFFFFFu, va, 1);
    vb += __shfl_xor_sync(0xFFFFFFFFu, vb, 1);
    va += __shfl_xor_sync(0xFFFFFFFFu, va, 2);
    vb += __shfl_xor_sync(0xFFFFFFFFu, vb, 2);
    if (t == 0) {
      atomicAdd(&red[(16 * rg + g) * 16], va);
      atomicAdd(&red[(16 * rg + g + 8) * 16], vb);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      A[rg][0][r] = 0;
      B[rg][kB][r] = 0;
    }
  }
}

// Add a warp's accumulators into the segment's shared table and clear them
// (kHi: acc16 holds the times-16 sums of gemv_mma_unit, divided exactly).
template <int NT, int TILES, bool kHi>
__device__ __forceinline__ void gt_flush(int (&acc)[4][NT][4], int (&acc16)[4][NT][4], int* red,
                                         int M, int g, int t) {
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
#pragma unroll
    for (int nt = 0; nt < TILES; ++nt) {
      const int r0 = 16 * rg + g, c0 = 8 * nt + 2 * t;
      int v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = kHi ? acc[rg][nt][e] + (acc16[rg][nt][e] >> 4) : acc[rg][nt][e];
      if (c0 < M) {
        atomicAdd(&red[r0 * 16 + c0], v[0]);
        atomicAdd(&red[(r0 + 8) * 16 + c0], v[2]);
      }
      if (c0 + 1 < M) {
        atomicAdd(&red[r0 * 16 + c0 + 1], v[1]);
        atomicAdd(&red[(r0 + 8) * 16 + c0 + 1], v[3]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[rg][nt][e] = 0;
        if (kHi) acc16[rg][nt][e] = 0;
      }
    }
  }
}

// One CTA of 352 threads (eleven warps) per SM.  The register file is split
// between the SM's four sub-partitions and three of them hold three warps,
// so the launch bound caps a thread at about 170 registers.
template <int NT, bool kPair>
__global__ void __launch_bounds__(kGtThreads, 1)
ternary_gemv_tiled_kernel(const __grid_constant__ GtLaunch L) {
  using C = GtCfg<kPair, NT>;
  // One token tile: the unpack with a second, times-16 accumulator set
  // (gemv_mma_unit, 5 ALU operations per MMA instead of 7); two token tiles
  // would not leave the registers for it.
  constexpr bool kHi = NT == 1;
  constexpr int S = C::STAGES;
  constexpr int UNITS = C::UNITS;
  constexpr int kTabRows = C::TAB_ROWS;
  extern __shared__ uint8_t gt_smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gt_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ int acc_tab[2][kTabRows * 16];        // [row][token] sums of a segment
  __shared__ GtTok tok[2][16];                     // token constants of a segment
  // full[s]: stage s has landed (three arrivals, one per producer thread,
  // plus the bytes of its copies).  empty[s]: every MMA warp has read it.
  __shared__ __align__(8) uint64_t full[S], empty[S];
  __shared__ __align__(8) uint64_t seg_bar;
  __shared__ volatile int abort_flag;

  // The dependent grid (the fixup of partial row blocks) only ever waits for
  // this grid to complete, so it may be scheduled at once.
  pdl_launch_dependents();
  // The problem table and the CTA ranges stay in kernel-parameter space:
  // every access below uses an index that is the same for all threads of a
  // warp, which that space serves as one broadcast.
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int count = L.count;
  const uint64_t limit = L.wait_limit_ns;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 3);
      mbar_init(&empty[s], kGtMmaWarps);
    }
    mbar_init(&seg_bar, kGtMmaWarps);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const long long t0 = L.tile_begin[blockIdx.x], t1 = L.tile_begin[blockIdx.x + 1];
  const GtProblem* prob = L.prob;

  if (warp >= kGtMmaWarps) {
    // ------------------------------------------------------------ producers
    // A thread starts a bulk copy only every few hundred nanoseconds, so
    // every producer thread issues one copy per stage: role 0 the first half
    // of the stage's units, role 1 the second half, role 2 the activations.
    // Weights never depend on the preceding grid; the activations do, so
    // role 2 waits for that grid (programmatic dependent launch) first.
    if (lane != 0) return;
    const int role = warp - kGtMmaWarps;
    if (role == 2 && L.use_pdl) pdl_wait_prior_grid();
    uint64_t* fb = full;
    bool failed = false;
    int j = 0;          // stage being issued
    for (long long t = t0; t < t1 && !failed;) {
      const GtSeg sg = gt_segment(prob, count, t, t1);
      const GtProblem& P = prob[sg.p];
      for (int off = 0; off < sg.nt; off += UNITS, ++j) {
        const int s = j % S;
        if (j >= S && !mbar_wait_bounded_sleep(&empty[s], static_cast<uint32_t>(j / S - 1) & 1u,
                                               &abort_flag, limit)) {
          abort_flag = 1;
          record_failure(L.status, DEV_TIMEOUT_PRODUCER);
          failed = true;
          break;
        }
        const int n = min(UNITS, sg.nt - off);
        const int n1 = (n + 1) >> 1;               // units of role 0
        uint8_t* st = ring + s * C::STAGE_BYTES;
        const long long c = sg.c + off;
        const uint8_t* wsrc = P.Wt + (static_cast<long long>(sg.rb) * P.KC + c) * C::UNIT_BYTES;
        if (role == 0) {
          const uint32_t b = static_cast<uint32_t>(n1 * C::UNIT_BYTES);
          mbar_arrive_expect_tx(&fb[s], b);
          bulk_load(st, wsrc, b, &fb[s]);
        } else if (role == 1) {
          const uint32_t b = static_cast<uint32_t>((n - n1) * C::UNIT_BYTES);
          mbar_arrive_expect_tx(&fb[s], b);
          if (b) bulk_load(st + n1 * C::UNIT_BYTES, wsrc + n1 * C::UNIT_BYTES, b, &fb[s]);
        } else {
          const uint32_t b = static_cast<uint32_t>(n * P.M * 256);
          mbar_arrive_expect_tx(&fb[s], b);
          bulk_load(st + kGtWBytes, P.xd + c * P.M * 256, b, &fb[s]);
        }
      }
      t += sg.nt;
    }
    if (abort_flag) {
      // Let this thread's copies in flight land before the CTA exits (the
      // wait gives up at the limit if another producer stopped arriving).
      for (int q = (j > S ? j - S : 0); q < j; ++q)
        if (!mbar_wait_bounded(&fb[q % S], static_cast<uint32_t>(q / S) & 1u, nullptr, limit))
          record_failure(L.status, DEV_TIMEOUT_DRAIN);
    }
    return;
  }

  // --------------------------------------------------------------- MMA warps
  for (int i = tid; i < 2 * kTabRows * 16; i += kGtMmaThreads) (&acc_tab[0][0])[i] = 0;
  // The token constants come from the quant grid.
  if (L.use_pdl) pdl_wait_prior_grid();
  const int g = lane >> 2, t = lane & 3;
  // Unit u of each stage, sub-tile sub (pair: 0 = gate, 1 = up), half h.
  const int u = kPair ? warp >> 2 : warp >> 1;
  const int sub = kPair ? (warp >> 1) & 1 : 0;
  const int h = warp & 1;
  const int tab_row0 = sub * kTileRows + 64 * h;   // this warp's first table row
  int acc[4][NT][4], acc16[4][NT][4];
#pragma unroll
  for (int rg = 0; rg < 4; ++rg)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[rg][nt][e] = 0;
        acc16[rg][nt][e] = 0;
      }
  GemvBuf<NT> buf;
  int j = 0, segi = 0;
  GtTok tk{};
  int tk_p = -1, tk_grp = -1;
  uint32_t seg_phase = 0;
  bool ok = gt_mma_sync(&seg_bar, seg_phase, &abort_flag, limit);   // tables cleared
  for (long long tt = t0; tt < t1 && ok; ++segi) {
    const GtSeg sg = gt_segment(prob, count, tt, t1);
    const GtProblem& P = prob[sg.p];
    const int M = P.M;
    const bool two = NT == 2 && M > 8;
    const bool one = M == 1;   // dp4a instead of mma.sync
    const GtSpan span = gt_span(P, sg);
    const bool whole = sg.t == span.first && sg.nt == span.len;
    // Warp 0 keeps the token constants of the current (problem, group) in
    // registers and fetches them only when that changes: a fetch stalls the
    // warp for a global-memory round trip, and every other warp would wait
    // for it at the next stage release.
    if (warp == 0 && (sg.p != tk_p || span.grp != tk_grp)) {
      if (lane < M) tk = gt_token(P, lane, kPair, span.grp);
      tk_p = sg.p;
      tk_grp = span.grp;
    }
    bool any = false;
    for (int off = 0; off < sg.nt; off += UNITS, ++j) {
      const int n = min(UNITS, sg.nt - off);
      const int s = j % S;
      const uint32_t par = static_cast<uint32_t>(j / S) & 1u;
      const bool got = mbar_wait_bounded_sleep(&full[s], par, &abort_flag, limit);
      if (!__all_sync(0xFFFFFFFFu, got)) {
        abort_flag = 1;
        if (lane == 0) record_failure(L.status, DEV_TIMEOUT_GEMV);
        ok = false;
        break;
      }
      if (u < n) {
        const uint8_t* ws =
            ring + s * C::STAGE_BYTES + u * C::UNIT_BYTES + sub * kTileBytes + h * (64 * 64);
        // Rows 64h + 16rg + g and +8 of the tile; piece t, swizzled by row.
#pragma unroll
        for (int rg = 0; rg < 4; ++rg) {
          const int r = 16 * rg + g;           // (64h + r) >> 1 has the same low bits
          const int sw = 16 * (t ^ ((r >> 1) & 3));
          buf.wa[rg] = *reinterpret_cast<const uint4*>(ws + r * 64 + sw);
          buf.wb[rg] = *reinterpret_cast<const uint4*>(ws + (r + 8) * 64 + sw);
        }
        const uint8_t* xs = ring + s * C::STAGE_BYTES + kGtWBytes + u * M * 256;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (nt == 0 || two) {
            const int m = min(8 * nt + g, M - 1);   // tokens past M: any valid bytes
#pragma unroll
            for (int q = 0; q < 4; ++q)
              buf.x[nt][q] = *reinterpret_cast<const uint4*>(
                  xs + m * 256 + 16 * x_block_pos(4 * t + q, m & 1));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (u < n) {
        any = true;
        if (one) {
          if constexpr (NT == 2)
            gt_dp4a_unit<NT, 1>(acc, acc, buf);
          else
            gt_dp4a_unit<NT, 0>(acc, acc16, buf);
        } else if (kHi) {
          gemv_mma_unit<NT, 1>(acc, acc16, buf);
        } else if (two) {
          gt_mma_unit<NT, NT>(acc, buf);
        } else {
          gt_mma_unit<NT, 1>(acc, buf);
        }
      }
    }
    if (!ok) break;
    if (whole && warp == 0 && lane < M) tok[segi & 1][lane] = tk;
    int* tab = acc_tab[segi & 1];
    if (any) {
      if (one) {
        if constexpr (NT == 2)
          gt_flush_one<NT, 1>(acc, acc, tab + tab_row0 * 16, g, t);
        else
          gt_flush_one<NT, 0>(acc, acc16, tab + tab_row0 * 16, g, t);
      } else if (two)
        gt_flush<NT, NT, kHi>(acc, acc16, tab + tab_row0 * 16, M, g, t);
      else
        gt_flush<NT, 1, kHi>(acc, acc16, tab + tab_row0 * 16, M, g, t);
    }
    if (!gt_mma_sync(&seg_bar, seg_phase, &abort_flag, limit)) {
      ok = false;
      break;
    }
    // ------------------------------------------------------- finish segment
    // Every thread clears the table entries it reads, right after reading
    // them (entries of tokens >= M are never written): the table is clean
    // for its reuse two segments later, which the next segment's barrier
    // orders after these writes.
    const int n0 = sg.rb * kTileRows;
    if (whole) {
      for (int idx = tid; idx < kTileRows * M; idx += kGtMmaThreads) {
        const int r = idx & (kTileRows - 1), m = idx >> 7;
        const int v = tab[r * 16 + m];
        tab[r * 16 + m] = 0;
        if (kPair) {
          const int v2 = tab[(kTileRows + r) * 16 + m];
          tab[(kTileRows + r) * 16 + m] = 0;
          if (n0 + r < P.N) gt_store_pair(P, tok[segi & 1][m], m, n0 + r, v, v2);
        } else if (n0 + r < P.N) {
          gt_store(P, tok[segi & 1][m], m, n0 + r, v, span.grp);
        }
      }
    } else {
      // Part of a row block (the CTA's first or last segment): its sums go
      // to this CTA's slot; gemv_tiled_fixup_kernel adds the slots up.
      const int kpart = (sg.t == t0) ? 0 : 1;
      int32_t* slot = P.part + static_cast<int64_t>(2 * (static_cast<int>(blockIdx.x) -
                                                         P.cta_first) + kpart) *
                                   kTabRows * M;
      for (int idx = tid; idx < kTabRows * M; idx += kGtMmaThreads) {
        const int r = idx % kTabRows, m = idx / kTabRows;
        slot[m * kTabRows + r] = tab[r * 16 + m];
        tab[r * 16 + m] = 0;
      }
    }
    tt += sg.nt;
  }
  if (!ok && lane == 0) record_failure(L.status, DEV_TIMEOUT_GEMV);
}

// Finish of the row blocks (with group-wise scales: row-block groups) that
// several CTAs of ternary_gemv_tiled_kernel share.  Such a span is finished
// by the CTAs of column blockIdx.x, the CTA of the streaming kernel whose
// range holds the span's first tile: that CTA's last span, when it starts
// inside the CTA's range and ends past it.  The contributors are the CTAs
// whose ranges meet the span; each left its sums in its slot 0 (its range
// starts inside the span) or slot 1 (the finishing CTA, whose range starts
// before the span).  One thread per output (row r = threadIdx.x % 128,
// token kGtFixTokens * blockIdx.y + threadIdx.x / 128), so every load of a
// thread is independent of the others and they overlap.  Launched right
// after the streaming kernel as its programmatic dependent: the wait below
// returns once that grid has completed and its stores are visible.
constexpr int kGtFixTokens = 4;
template <bool kPair>
__global__ void __launch_bounds__(kTileRows * kGtFixTokens)
gemv_tiled_fixup_kernel(const __grid_constant__ GtLaunch L) {
  constexpr int kTabRows = GtCfg<kPair, 1>::TAB_ROWS;
  pdl_wait_prior_grid();
  const long long* stb = L.tile_begin;
  const long long t0 = stb[blockIdx.x], t1 = stb[blockIdx.x + 1];
  const GtSeg sg = gt_segment(L.prob, L.count, t1 - 1, t1);
  const GtProblem& P = L.prob[sg.p];
  const GtSpan sp = gt_span(P, sg);
  if (sp.first < t0 || sp.first + sp.len <= t1) return;
  const int r = threadIdx.x % kTileRows;
  const int m = kGtFixTokens * blockIdx.y + threadIdx.x / kTileRows;
  const int n = sg.rb * kTileRows + r;
  if (m >= P.M || n >= P.N) return;
  const int c_last = gt_cta_of(stb, L.ctas, sp.first + sp.len - 1);
  const GtTok tk = gt_token(P, m, kPair, sp.grp);
  int v = 0, v2 = 0;
  for (int cb = blockIdx.x; cb <= c_last; ++cb) {
    const int sd = (stb[cb] >= sp.first) ? 0 : 1;
    const int32_t* sl =
        P.part + static_cast<int64_t>(2 * (cb - P.cta_first) + sd) * kTabRows * P.M;
    v += __ldcg(sl + m * kTabRows + r);
    if (kPair) v2 += __ldcg(sl + m * kTabRows + kTileRows + r);
  }
  if (kPair)
    gt_store_pair(P, tk, m, n, v, v2);
  else
    gt_store(P, tk, m, n, v, sp.grp);
}

}  // namespace bitnet
