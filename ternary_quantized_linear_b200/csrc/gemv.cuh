// gemv.cuh -- decode-path ternary matmul (M <= 16 tokens) plus fused dequant,
// for one problem or a group of independent problems in a single launch.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// sections 計算パラダイム (integer accumulation), 推論最適化とカスタムカーネル
// (weights unpacked on the fly inside the matmul) and 量子化の仕組み (rescale
// by both scales).
//
// The decode matmul is HBM-bound: the packed weights are the traffic, read
// once.  Design:
//   * Work is cut into units of 64 weight rows x 256 k of one problem (4 KiB
//     of packed weights); a row block is the kc = K/256 units of 64 rows.
//     The host gives each CTA a list of segments (a row block, or part of
//     one) in one of two ways: whole row blocks dealt out greedily, largest
//     first, to the least-loaded CTA (no cross-CTA reduction at all), or,
//     when that balances badly, every CTA an equal contiguous share of the
//     units laid end to end ("stream-K").  The units of a CTA's segment list
//     are split into eight equal contiguous ranges, one per compute warp.
//   * Operands move by TMA: each warp has its own ring of stages (gemv_stages)
//     and its lane 0 issues, per unit, one 2-D box of weights (64 rows x 64
//     bytes) and one of activations (the unit's 256 bytes of 8 or 16 token
//     rows), refilling a stage as soon as the warp has read it.  Eight
//     issuing lanes per SM keep enough copies in flight (one issuing thread
//     cannot: each copy costs it a few hundred nanoseconds), and rows past N,
//     tokens past M or k past K arrive as zeros.
//   * Lane (4g + t) reads 16 bytes (64 k) of rows g and g+8 of each 16-row
//     group (64-byte rows: conflict-free) and the 64 bytes of token g for the
//     same k, which the activation-quant kernel stored in the decode block
//     order (x_block_pos) so that these reads are conflict-free too.
//   * Unpack in registers with masks: byte i of a packed word holds the codes
//     t+1 of k = 4i..4i+3 of a 16-k group at bits 2r; P & 0x03030303 and
//     (P >> 2) & 0x03030303 are words of four int8 codes (r = 0, 1), and
//     P & 0x30303030, (P >> 2) & 0x30303030 the r = 2, 3 codes times 16, which
//     feed a second accumulator set.  The activations are stored
//     k-interleaved (byte 4r+i of each 16-group holds k = 4i+r), so the
//     matching activation word is a plain 4-byte slice.
//   * Warp-level int8 MMA m16n8k32 in swap-AB form: 16 weight rows are the
//     MMA's M, up to 16 tokens its N (one or two n8 tiles).  Eight
//     independent accumulator chains.  sum x*(t+1) minus the token's row sum
//     sum x gives sum x*t exactly.
//   * The weight copies start before waiting on the activation-quant grid
//     (programmatic dependent launch): only the activation copies wait.
//   * A warp adds its accumulators to its CTA's per-segment sums in shared
//     memory when it moves to another segment.  At the end, whole row blocks
//     are finished directly (y = acc / (s_x * s_w)); a part of a row block
//     (stream-K ends) adds its partials into an int32 workspace and the last
//     CTA to arrive (arrival counter, no waiting) reads them back, re-zeroes
//     them and finishes.
//   * Every wait on a copy is bounded; nothing waits on another CTA.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kGemvRows = 64;        // weight rows per unit
constexpr int kGemvUnitK = 256;      // k per unit
constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = 32 * kGemvWarps;
constexpr int kGemvMaxSegs = 6;      // row blocks one CTA's share may touch
constexpr int kGemvMaxGroup = 16;    // problems per grouped launch
constexpr uint32_t kCodeMask = 0x03030303u;
constexpr int kGemvStagesMax = 3;
constexpr int kGemvUnitBytes = kGemvRows * (kGemvUnitK / 4);  // 4 KiB of weights
// Ring stages per warp: three with one token tile, two with two, so that a
// decode CTA still fits on an SM beside an activation-quant CTA (the two
// overlap under programmatic dependent launch).
__host__ __device__ constexpr int gemv_stages(int nt) { return nt == 1 ? 3 : 2; }
// A stage: the unit's weights, then its activations (8 or 16 token rows of
// 256 bytes).
__host__ __device__ constexpr int gemv_stage_bytes(int nt) { return kGemvUnitBytes + nt * 2048; }
__host__ __device__ constexpr int gemv_smem_bytes(int nt) {
  return kGemvWarps * gemv_stages(nt) * gemv_stage_bytes(nt) + 1024;  // + alignment slack
}

// The copy engine reads these from the kernel parameters.
struct GemvMaps {
  CUtensorMap tmap_w;     // W_packed [N][K/4] bytes, box 64 x 64 rows, no swizzle
  CUtensorMap tmap_x;     // x_q [M][K] bytes (decode block order), box 256 x 8 or 16 rows
};

struct GemvProblem {
  const uint8_t* W;       // W_packed [N][K/4]
  const int8_t* xq;       // x_q k-interleaved [M][K]
  const int32_t* rowsum;  // [M]
  const float* s_x;       // [M] (null: no dequant)
  const float* s_w;       // [1] (null: no dequant)
  void* y;                // [M][N] fp32 or bf16, may be null
  int32_t* acc_out;       // [M][N] debug accumulators, may be null
  int32_t* ws_acc;        // [M][N] partials of shared row blocks, zero on entry
  unsigned* ws_cnt;       // [rb] arrival counters, zero on entry
  long long unit_begin;   // first unit of this problem in the launch
  int M, N, K;
  int y_bf16;
  int rb;                 // row blocks = ceil(N / 64)
  int kc;                 // units per row block = ceil(K / 256)
  int rb_begin;           // first row block of this problem in the launch
};

constexpr int kGemvMaxCtas = 296;    // CTAs of a launch with an explicit row-block list

struct GemvLaunch {
  GemvMaps maps[kGemvMaxGroup];
  GemvProblem prob[kGemvMaxGroup];
  long long units;        // total units of the launch
  int count;              // problems in this launch
  int use_pdl;            // wait for the preceding grid before reading activations
  int early_weights;      // start the weight copies before that wait
  int* status;            // device status word (bounded waits)
  uint64_t wait_limit_ns;
  int listed;             // 1: CTA b owns row blocks task[b][0 .. ntask[b])
                          // 0: CTA b owns units [b U / G, (b+1) U / G)
  uint8_t ntask[kGemvMaxCtas];
  uint16_t task[kGemvMaxCtas][kGemvMaxSegs];  // global row block ids
};

template <int NT>
struct GemvBuf {
  uint4 wa[4], wb[4];  // rows g and g+8 of the four row groups
  uint4 x[NT][4];      // token 8 nt + g, 64 k
};



__device__ __forceinline__ uint32_t word_of(const uint4& v, int w) {
  return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

// Unit u of the launch: its problem (p advances monotonically from a hint),
// row block and k chunk.  Used for the two ends of a stream-K share.
struct GemvUnit {
  int p, rbl, c;
};

__device__ __forceinline__ GemvUnit gemv_unit(const GemvProblem* prob, int count, long long u,
                                          int& p_hint) {
  while (p_hint + 1 < count && u >= prob[p_hint + 1].unit_begin) ++p_hint;
  const GemvProblem& P = prob[p_hint];
  const int local = static_cast<int>(u - P.unit_begin);  // < rb * kc < 2^31
  GemvUnit r;
  r.p = p_hint;
  r.rbl = local / P.kc;
  r.c = local - r.rbl * P.kc;
  return r;
}

// Activations of one unit from its stage: token 8 nt + g, this lane's 64 k
// (blocks 4t + q of the 256-byte span, stored at x_block_pos; tokens past M
// and k past K arrived as zeros).
template <int NT, int TILES>
__device__ __forceinline__ void gemv_read_stage_x(GemvBuf<NT>& b, const uint8_t* xs, int g,
                                                  int t) {
#pragma unroll
  for (int nt = 0; nt < TILES; ++nt)
#pragma unroll
    for (int q = 0; q < 4; ++q)
      b.x[nt][q] = *reinterpret_cast<const uint4*>(
          xs + (8 * nt + g) * 256 + 16 * x_block_pos(4 * t + q, g & 1));
}

// Weights of one unit from its stage: rows g and g+8 of each 16-row group,
// this lane's 16 bytes.  64-byte rows: the eight lanes of a quarter warp
// (g = 2j, 2j+1; t = 0..3) hit 32 distinct banks.
template <int NT>
__device__ __forceinline__ void gemv_read_stage(GemvBuf<NT>& b, const uint8_t* stage, int g,
                                                int t) {
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
    b.wa[rg] = *reinterpret_cast<const uint4*>(stage + (16 * rg + g) * 64 + 16 * t);
    b.wb[rg] = *reinterpret_cast<const uint4*>(stage + (16 * rg + g + 8) * 64 + 16 * t);
  }
}

// The MMAs of one unit for TILES token tiles.  Unpack: Q = P >> 2 once per
// word, then one mask per code word: P & 0x03.. and Q & 0x03.. are the codes
// of k = 4i and 4i+1 of a 16-k group; P & 0x30.. and Q & 0x30.. those of
// 4i+2 and 4i+3 times 16 (at most 32: still int8).  The times-16 words go
// to their own accumulators (acc16), divided by 16 exactly when flushed.
// Row groups innermost: consecutive MMAs feed eight independent
// accumulators, so the MMA latency overlaps.
template <int NT, int TILES>
__device__ __forceinline__ void gemv_mma_unit(int (&acc)[4][NT][4], int (&acc16)[4][NT][4],
                                              const GemvBuf<NT>& b) {
  constexpr uint32_t kHi = kCodeMask << 4;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t lo[4][4], hi[4][4];  // [rg][a0 a1 a2 a3]
#pragma unroll
    for (int rg = 0; rg < 4; ++rg) {
      const uint32_t Pa = word_of(b.wa[rg], w), Pb = word_of(b.wb[rg], w);
      const uint32_t Qa = Pa >> 2, Qb = Pb >> 2;
      lo[rg][0] = Pa & kCodeMask;
      lo[rg][1] = Pb & kCodeMask;
      lo[rg][2] = Qa & kCodeMask;
      lo[rg][3] = Qb & kCodeMask;
      hi[rg][0] = Pa & kHi;
      hi[rg][1] = Pb & kHi;
      hi[rg][2] = Qa & kHi;
      hi[rg][3] = Qb & kHi;
    }
#pragma unroll
    for (int nt = 0; nt < TILES; ++nt) {
#pragma unroll
      for (int rg = 0; rg < 4; ++rg)
        mma_m16n8k32_s8(acc[rg][nt], lo[rg][0], lo[rg][1], lo[rg][2], lo[rg][3],
                        word_of(b.x[nt][w], 0), word_of(b.x[nt][w], 1));
#pragma unroll
      for (int rg = 0; rg < 4; ++rg)
        mma_m16n8k32_s8(acc16[rg][nt], hi[rg][0], hi[rg][1], hi[rg][2], hi[rg][3],
                        word_of(b.x[nt][w], 2), word_of(b.x[nt][w], 3));
    }
  }
}

// Add a warp's accumulators into the row block's shared sums and clear them.
template <int NT, int TILES>
__device__ __forceinline__ void gemv_flush(int (&acc)[4][NT][4], int (&acc16)[4][NT][4], int* red,
                                           int M, int g, int t) {
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
#pragma unroll
    for (int nt = 0; nt < TILES; ++nt) {
      const int r0 = 16 * rg + g, c0 = 8 * nt + 2 * t;
      int v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = acc[rg][nt][j] + (acc16[rg][nt][j] >> 4);  // exact
      if (c0 < M) {
        atomicAdd(&red[r0 * 16 + c0], v[0]);
        atomicAdd(&red[(r0 + 8) * 16 + c0], v[2]);
      }
      if (c0 + 1 < M) {
        atomicAdd(&red[r0 * 16 + c0 + 1], v[1]);
        atomicAdd(&red[(r0 + 8) * 16 + c0 + 1], v[3]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[rg][nt][j] = acc16[rg][nt][j] = 0;
    }
  }
}

// rs: token m's row sum; d = RN(s_x[m] * s_w) and rd = RN(1 / d), read and
// computed once per segment into shared memory.
__device__ __forceinline__ void gemv_finish(const GemvProblem& p, float d, float rd, int rs,
                                            int m, int n, int acc_codes) {
  const int acc = acc_codes - rs;
  const int64_t o = static_cast<int64_t>(m) * p.N + n;
  if (p.acc_out) p.acc_out[o] = acc;
  if (p.y) {
    const float yv = div_rn_int(__int2float_rn(acc), d, rd);
    if (p.y_bf16)
      reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(yv);
    else
      reinterpret_cast<float*>(p.y)[o] = yv;
  }
}

// CTA whose share [b U / G, (b+1) U / G) holds unit u.
__host__ __device__ __forceinline__ long long gemv_cta_of(long long u, long long U, long long G) {
  return ((u + 1) * G - 1) / U;
}

template <int NT>
__global__ void __launch_bounds__(kGemvThreads, 1)
ternary_gemv_kernel(const __grid_constant__ GemvLaunch L) {
  extern __shared__ uint8_t gemv_smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gemv_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ int red[kGemvMaxSegs * kGemvRows * 16];  // [segment][row][token]
  __shared__ __align__(8) uint64_t full[kGemvWarps][kGemvStagesMax];
  // The problem table and this CTA's segments live in shared memory: the
  // walk indexes them by run-time numbers, which kernel-parameter space
  // serves slowly (the copy engine still reads the tensor maps from the
  // parameters).
  __shared__ GemvProblem sprob[kGemvMaxGroup];
  __shared__ int seg_p[kGemvMaxSegs], seg_rbl[kGemvMaxSegs];
  __shared__ int seg_lo[kGemvMaxSegs], seg_n[kGemvMaxSegs], seg_owned[kGemvMaxSegs];
  __shared__ int seg_count, seg_last[kGemvMaxSegs];
  __shared__ int seg_rs[kGemvMaxSegs][16];    // row sums of the segment's tokens
  __shared__ float seg_d[kGemvMaxSegs][16];   // their dequant divisors s_x * s_w
  __shared__ float seg_rd[kGemvMaxSegs][16];  // and RN(1 / divisor)
  __shared__ volatile int abort_flag;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const long long U = L.units, G = gridDim.x, b = blockIdx.x;
  const long long ub = b * U / G, ue = (b + 1) * U / G;  // stream-K share
  const int count = L.count;
  const uint64_t limit = L.wait_limit_ns;
  if (tid < count) sprob[tid] = L.prob[tid];
  if (tid < kGemvWarps * kGemvStagesMax) mbar_init(&full[0][0] + tid, 1);
  if (tid == 0) {
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const GemvProblem* prob = sprob;
  if (L.listed) {
    // One thread per listed row block: the parameter reads go out together.
    if (tid < kGemvMaxSegs) {
      const int n = L.ntask[b];
      if (tid == 0) seg_count = n;
      if (tid < n) {
        const int R = L.task[b][tid];
        int p = 0;
        while (p + 1 < count && R >= prob[p + 1].rb_begin) ++p;
        seg_p[tid] = p;
        seg_rbl[tid] = R - prob[p].rb_begin;
        seg_lo[tid] = 0;
        seg_n[tid] = prob[p].kc;
        seg_owned[tid] = 1;
      }
    }
  } else if (tid == 0) {
    int n = 0;
    if (ub < ue) {
      int p = 0;
      const GemvUnit first = gemv_unit(prob, count, ub, p);
      const GemvUnit last = gemv_unit(prob, count, ue - 1, p);
      int q = first.p, rbl = first.rbl;
      for (;;) {
        const int lo = (q == first.p && rbl == first.rbl) ? first.c : 0;
        const bool end = (q == last.p && rbl == last.rbl);
        const int hi = end ? last.c + 1 : prob[q].kc;
        seg_p[n] = q;
        seg_rbl[n] = rbl;
        seg_lo[n] = lo;
        seg_n[n] = hi - lo;
        seg_owned[n] = (lo == 0 && hi == prob[q].kc) ? 1 : 0;
        ++n;
        if (end || n == kGemvMaxSegs) break;
        if (++rbl == prob[q].rb) {
          rbl = 0;
          ++q;
        }
      }
    }
    seg_count = n;
  }
  for (int i = tid; i < kGemvMaxSegs * kGemvRows * 16; i += kGemvThreads) red[i] = 0;
  __syncthreads();
  const int nseg = seg_count;  // <= kGemvMaxSegs (host)
  if (nseg == 0) return;       // uniform over the CTA

  // Cursor over this CTA's units in segment order: (segment, offset).
  struct Cursor {
    int s, off;
  };
  auto advance = [&](Cursor& x, int step) {
    x.off += step;
    while (x.s < nseg && x.off >= seg_n[x.s]) {
      x.off -= seg_n[x.s];
      ++x.s;
    }
  };
  // Warp w takes the w-th of eight contiguous ranges of the CTA's units, of
  // equal cost: a unit of a problem with two token tiles counts 6, one with
  // one tile 5 (the host's dealing uses the same weights).
  auto unit_cost = [&](int sg) { return prob[seg_p[sg]].M > 8 ? 6 : 5; };
  int total_cost = 0;
  for (int i = 0; i < nseg; ++i) total_cost += seg_n[i] * unit_cost(i);
  // First unit (as a count of units before it) whose cost prefix reaches c.
  auto unit_at = [&](int c) {
    int u = 0;
    for (int i = 0; i < nseg; ++i) {
      const int w = unit_cost(i), segc = seg_n[i] * w;
      if (c <= segc) return u + (c + w - 1) / w;
      c -= segc;
      u += seg_n[i];
    }
    return u;
  };
  auto range_of = [&](int w, Cursor& x0) {
    const int u0 = unit_at(w * total_cost / kGemvWarps);
    const int u1 = unit_at((w + 1) * total_cost / kGemvWarps);
    x0 = Cursor{0, 0};
    advance(x0, u0);
    return u1 - u0;
  };

  // Warp w streams its range through its own ring: lane 0 issues the copies
  // (weights as soon as the CTA starts, activations once the preceding grid
  // is done), all lanes consume.
  constexpr int kStage = gemv_stage_bytes(NT);
  constexpr int kGemvStages = gemv_stages(NT);
  uint8_t* myring = ring + warp * kGemvStages * kStage;
  Cursor xA;
  const int n = range_of(warp, xA);
  Cursor xI = xA;  // next unit to issue
  int issued = 0;
  auto issue_w = [&](int j) {  // lane 0: unit j (cursor xI) weights into stage j % S
    const int st = j % kGemvStages;
    const int p = seg_p[xI.s];
    // The activation box has 8 or 16 rows: the problem's own token tiles.
    mbar_arrive_expect_tx(&full[warp][st], kGemvUnitBytes + (prob[p].M > 8 ? 4096 : 2048));
    tma_load_2d(myring + st * kStage, &L.maps[p].tmap_w, (seg_lo[xI.s] + xI.off) * (kGemvUnitK / 4),
                seg_rbl[xI.s] * kGemvRows, &full[warp][st]);
  };
  auto issue_x = [&](int j, const Cursor& x) {
    const int st = j % kGemvStages;
    tma_load_2d(myring + st * kStage + kGemvUnitBytes, &L.maps[seg_p[x.s]].tmap_x,
                (seg_lo[x.s] + x.off) * kGemvUnitK, 0, &full[warp][st]);
  };
  const int pre = min(n, kGemvStages);
  const bool early = L.early_weights != 0 || !L.use_pdl;
  if (lane == 0 && early) {
    Cursor c0 = xI;
    for (int j = 0; j < pre; ++j) {
      issue_w(j);
      if (j + 1 < pre) advance(xI, 1);
    }
    xI = c0;
  }
  if (L.use_pdl) pdl_wait_prior_grid();
  if (warp < nseg) {
    // This warp reads segment `warp`'s row sums and scales for the finish.
    const GemvProblem& P = prob[seg_p[warp]];
    if (lane < P.M) {
      seg_rs[warp][lane] = P.rowsum[lane];
      const float d = (P.y && P.s_x && P.s_w) ? __fmul_rn(P.s_x[lane], P.s_w[0]) : 1.0f;
      seg_d[warp][lane] = d;
      seg_rd[warp][lane] = recip_for_div(d);
    }
  }
  if (lane == 0) {
    for (int j = 0; j < pre; ++j) {
      if (!early) issue_w(j);
      issue_x(j, xI);
      if (j + 1 < n) advance(xI, 1);
    }
  }
  issued = pre;

  GemvBuf<NT> buf;
  int acc[4][NT][4], acc16[4][NT][4];
#pragma unroll
  for (int rg = 0; rg < 4; ++rg)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[rg][nt][j] = acc16[rg][nt][j] = 0;
  int cur_seg = -1, cur_m = 0;
  auto flush = [&]() {
    if (cur_seg < 0) return;
    int* dst = red + cur_seg * kGemvRows * 16;
    if (NT == 2 && cur_m > 8)
      gemv_flush<NT, NT>(acc, acc16, dst, cur_m, g, t);
    else
      gemv_flush<NT, 1>(acc, acc16, dst, cur_m, g, t);
  };
  int k = 0;
  for (; k < n; ++k) {
    const int st = k % kGemvStages;
    // The MMAs below are warp-collective: the wait verdict is made uniform
    // across the warp.
    const bool got = mbar_wait_bounded(&full[warp][st], static_cast<uint32_t>(k / kGemvStages) & 1u,
                                       &abort_flag, limit);
    if (!__all_sync(0xFFFFFFFFu, got)) {
      abort_flag = 1;
      if (lane == 0) record_failure(L.status, DEV_TIMEOUT_GEMV);
      break;
    }
    const uint8_t* sp = myring + st * kStage;
    const int seg = xA.s;
    if (seg != cur_seg) {
      flush();
      cur_seg = seg;
      cur_m = prob[seg_p[seg]].M;
    }
    const bool two = NT == 2 && cur_m > 8;
    gemv_read_stage(buf, sp, g, t);
    if (two)
      gemv_read_stage_x<NT, NT>(buf, sp + kGemvUnitBytes, g, t);
    else
      gemv_read_stage_x<NT, 1>(buf, sp + kGemvUnitBytes, g, t);
    // Refill this stage with unit k + S once every lane's reads are done.
    __syncwarp();
    if (lane == 0 && issued < n) {
      fence_proxy_async_smem();
      issue_w(issued);
      issue_x(issued, xI);
      if (issued + 1 < n) advance(xI, 1);
    }
    if (issued < n) ++issued;
    if (k + 1 < n) advance(xA, 1);
    if (two)
      gemv_mma_unit<NT, NT>(acc, acc16, buf);
    else
      gemv_mma_unit<NT, 1>(acc, acc16, buf);
  }
  flush();
  if (abort_flag && lane == 0) {
    // Let the copies already in flight land before the CTA exits.
    for (int j = k; j < issued; ++j)
      if (!mbar_wait_bounded(&full[warp][j % kGemvStages],
                             static_cast<uint32_t>(j / kGemvStages) & 1u, nullptr, limit))
        record_failure(L.status, DEV_TIMEOUT_DRAIN);
  }
  const int all_ok = __syncthreads_and(abort_flag == 0 ? 1 : 0);
  if (!all_ok) return;  // a timed-out copy: results would be garbage

  // Finish this CTA's segments: whole row blocks straight from the shared
  // sums; a part of a row block (stream-K ends) adds its partials to the
  // workspace and the last CTA to arrive finishes it.  The parts go through
  // one fence / counter / read-back round together.
  bool any_part = false;
  for (int s = 0; s < nseg; ++s) {
    const GemvProblem& P = prob[seg_p[s]];
    const int* rs = red + s * kGemvRows * 16;
    const int nout = kGemvRows * P.M;
    const int n0 = seg_rbl[s] * kGemvRows;
    if (seg_owned[s]) {
      for (int idx = tid; idx < nout; idx += kGemvThreads) {
        const int r = idx % kGemvRows, m = idx / kGemvRows, n = n0 + r;
        if (n < P.N) gemv_finish(P, seg_d[s][m], seg_rd[s][m], seg_rs[s][m], m, n, rs[r * 16 + m]);
      }
      continue;
    }
    any_part = true;
    for (int idx = tid; idx < nout; idx += kGemvThreads) {
      const int r = idx % kGemvRows, m = idx / kGemvRows, n = n0 + r;
      if (n < P.N) atomicAdd(P.ws_acc + static_cast<int64_t>(m) * P.N + n, rs[r * 16 + m]);
    }
  }
  if (!any_part) return;  // uniform over the CTA
  __threadfence();
  __syncthreads();
  if (tid < nseg) {
    int last = 0;
    if (!seg_owned[tid]) {
      const GemvProblem& P = prob[seg_p[tid]];
      const long long r0 = P.unit_begin + static_cast<long long>(seg_rbl[tid]) * P.kc;
      const long long r1 = r0 + P.kc;
      const long long contributors = gemv_cta_of(r1 - 1, U, G) - gemv_cta_of(r0, U, G) + 1;
      last = (atomicAdd(P.ws_cnt + seg_rbl[tid], 1u) == static_cast<unsigned>(contributors - 1))
                 ? 1
                 : 0;
    }
    seg_last[tid] = last;
  }
  __syncthreads();
  __threadfence();
  for (int s = 0; s < nseg; ++s) {
    if (!seg_last[s]) continue;
    const GemvProblem& P = prob[seg_p[s]];
    const int nout = kGemvRows * P.M;
    const int n0 = seg_rbl[s] * kGemvRows;
    for (int idx = tid; idx < nout; idx += kGemvThreads) {
      const int r = idx % kGemvRows, m = idx / kGemvRows, n = n0 + r;
      if (n < P.N) {
        const int v = atomicExch(P.ws_acc + static_cast<int64_t>(m) * P.N + n, 0);
        gemv_finish(P, seg_d[s][m], seg_rd[s][m], seg_rs[s][m], m, n, v);
      }
    }
    if (tid == 0) P.ws_cnt[seg_rbl[s]] = 0u;  // ready for the next call
  }
}

}  // namespace bitnet
