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
//     are split into eight equal contiguous ranges, one per warp.
//   * No shared-memory staging.  Lane (4g + t) loads 16 bytes (64 k) of rows
//     g and g+8 of each of the unit's four 16-row groups straight into
//     registers (eight 16-byte loads, every 32-byte sector used) and the
//     matching 64 bytes of x_q for token g (from L2: every row block reads
//     the same activations).  The next unit's loads are issued before the
//     current unit's MMAs (two register buffers).  At entry one thread asks
//     the copy engine to stream the share's whole row blocks (contiguous
//     64 x K/4 bytes each, one bulk operation per row block) into L2.
//   * Unpack in registers with masks: byte i of a packed word holds the codes
//     t+1 of k = 4i..4i+3 of a 16-k group at bits 2r; P & 0x03030303 and
//     (P >> 2) & 0x03030303 are words of four int8 codes (r = 0, 1), and
//     P & 0x30303030, (P >> 2) & 0x30303030 the r = 2, 3 codes times 16, which
//     feed a second accumulator set.  The activations are stored
//     k-interleaved (byte 4r+i of each 16-group holds k = 4i+r), so the
//     matching activation word is a plain 4-byte slice.
//   * Warp-level int8 MMA m16n8k32 in swap-AB form: 16 weight rows are the
//     MMA's M, up to 16 tokens its N (one or two n8 tiles).  The four row
//     groups are four independent accumulator chains.  sum x*(t+1) minus the
//     token's row sum sum x gives sum x*t exactly.
//   * Before waiting on the activation-quant grid (programmatic dependent
//     launch) each warp already loads its first two units' weights and the
//     L2 stream starts, so the weight traffic overlaps that grid.
//   * A warp adds its accumulators to its CTA's per-row-block sums in shared
//     memory when it moves to another row block.  At the end, a row block
//     that lies inside the CTA's share is finished directly
//     (y = acc / (s_x * s_w)); one shared with neighbouring CTAs adds its
//     partials into an int32 workspace and the last CTA to arrive (arrival
//     counter, no waiting) reads them back, re-zeroes them and finishes.
//   * Nothing in this kernel waits on a flag or barrier another CTA sets.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kGemvRows = 64;        // weight rows per unit
constexpr int kGemvUnitK = 256;      // k per unit
constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = 32 * kGemvWarps;
constexpr int kGemvMaxSegs = 8;      // row blocks one CTA's share may touch
constexpr int kGemvMaxGroup = 16;    // problems per grouped launch
constexpr uint32_t kCodeMask = 0x03030303u;
// Two register buffers per warp (next unit's loads in flight during the
// MMAs, one CTA per SM), or one buffer and two CTAs per SM.
#ifndef BITNET_GEMV_DOUBLE_BUFFER
#define BITNET_GEMV_DOUBLE_BUFFER 1
#endif
constexpr bool kGemvDoubleBuffer = BITNET_GEMV_DOUBLE_BUFFER != 0;

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

constexpr int kGemvMaxCtas = 1024;   // CTAs of a launch with an explicit row-block list
constexpr int kGemvMaxTasks = 2048;  // row blocks of such a launch

struct GemvLaunch {
  GemvProblem prob[kGemvMaxGroup];
  long long units;        // total units of the launch
  int count;              // problems in this launch
  int use_pdl;            // wait for the preceding grid before reading activations
  int early_weights;      // start the weight loads before that wait
  unsigned prefetch_bytes;  // per CTA: whole row blocks streamed into L2 at entry
  int listed;             // 1: CTA b owns row blocks task[cta_begin[b] .. cta_begin[b+1])
                          // 0: CTA b owns units [b U / G, (b+1) U / G)
  uint16_t cta_begin[kGemvMaxCtas + 1];
  uint16_t task[kGemvMaxTasks];  // global row block ids
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
// row block and k chunk.  Used once per warp; the walk then advances a
// cursor (no division per unit).
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

// Weight load of any unit.  No lane branches around its loads: rows past N
// read row N-1 (their outputs are never written) and a segment past K reads
// k = 0 (its activations are zeroed in gemv_load_x, so it adds nothing).
template <int NT>
__device__ __forceinline__ void gemv_load_w(GemvBuf<NT>& b, const GemvProblem& P, int rbl, int c,
                                            int g, int t) {
  const int kseg = c * kGemvUnitK + 64 * t;
  const int kk = kseg < P.K ? kseg : 0;  // K % 64 == 0: a segment is all in or all out
  const size_t rowb = static_cast<size_t>(P.K) / 4;
  const int r = rbl * kGemvRows + g;
  const uint8_t* base = P.W + kk / 4;
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
    const int ra = min(r + 16 * rg, P.N - 1), rb = min(r + 16 * rg + 8, P.N - 1);
    b.wa[rg] = ldg_stream_u4(base + static_cast<size_t>(ra) * rowb);
    b.wb[rg] = ldg_stream_u4(base + static_cast<size_t>(rb) * rowb);
  }
}

// Weight load of a unit inside a full row block with K % 256 == 0: no
// bounds tests.  base = row g of the row block, at this lane's 16 bytes.
template <int NT>
__device__ __forceinline__ void gemv_load_w_full(GemvBuf<NT>& b, const uint8_t* base,
                                                 size_t rowb) {
  const size_t r8 = 8 * rowb;
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
    b.wa[rg] = ldg_stream_u4(base + 2 * rg * r8);
    b.wb[rg] = ldg_stream_u4(base + (2 * rg + 1) * r8);
  }
}

// Activation load: token 8 nt + g, this lane's 64 k.  Tokens past M read
// token M-1 (their output columns are never written); a segment past K
// reads zeros.  No lane branches around the loads.
template <int NT>
__device__ __forceinline__ void gemv_load_x(GemvBuf<NT>& b, const GemvProblem& P, int c, int g,
                                            int t) {
  const int kseg = c * kGemvUnitK + 64 * t;
  const bool kval = kseg < P.K;
  const int kk = kval ? kseg : 0;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int m = min(8 * nt + g, P.M - 1);
    const int8_t* px = P.xq + static_cast<size_t>(m) * P.K + kk;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = ldg_u4_ro(px + 16 * q);
      b.x[nt][q] = kval ? v : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// Ask the copy engine to bring row block rbl of P (64 rows x K/4 bytes,
// contiguous) into L2, clipped to `limit` bytes; one bulk operation.
__device__ __forceinline__ uint32_t gemv_prefetch_rows(const GemvProblem& P, int rbl,
                                                       uint32_t limit) {
  const size_t rowb = static_cast<size_t>(P.K) / 4;
  const int rows = min(kGemvRows, P.N - rbl * kGemvRows);
  size_t bytes = static_cast<size_t>(rows) * rowb;  // multiple of 16 (K % 64 == 0)
  if (bytes > limit) bytes = limit & ~15u;
  if (bytes) prefetch_l2_bulk(P.W + static_cast<size_t>(rbl) * kGemvRows * rowb,
                              static_cast<uint32_t>(bytes));
  return static_cast<uint32_t>(bytes);
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

// CTA whose share [b U / G, (b+1) U / G) holds unit u.
__host__ __device__ __forceinline__ long long gemv_cta_of(long long u, long long U, long long G) {
  return ((u + 1) * G - 1) / U;
}

template <int NT>
__global__ void __launch_bounds__(kGemvThreads, kGemvDoubleBuffer ? 1 : 2)
ternary_gemv_kernel(const __grid_constant__ GemvLaunch L) {
  __shared__ int red[kGemvMaxSegs * kGemvRows * 16];  // [segment][row][token]
  // The problem table and this CTA's segments live in shared memory: the
  // walk indexes them by run-time numbers, which kernel-parameter space
  // serves slowly.
  __shared__ GemvProblem sprob[kGemvMaxGroup];
  __shared__ int seg_p[kGemvMaxSegs], seg_rbl[kGemvMaxSegs];
  __shared__ int seg_lo[kGemvMaxSegs], seg_n[kGemvMaxSegs], seg_owned[kGemvMaxSegs];
  __shared__ int seg_full[kGemvMaxSegs];  // 64 rows inside N and K % 256 == 0
  __shared__ int seg_count, seg_last[kGemvMaxSegs];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const long long U = L.units, G = gridDim.x, b = blockIdx.x;
  const long long ub = b * U / G, ue = (b + 1) * U / G;  // stream-K share
  const int count = L.count;
  if (tid < count) sprob[tid] = L.prob[tid];
  __syncthreads();
  const GemvProblem* prob = sprob;
  if (tid == 0) {
    int n = 0;
    if (L.listed) {
      const int t0 = L.cta_begin[b], t1 = L.cta_begin[b + 1];
      for (int i = t0; i < t1 && n < kGemvMaxSegs; ++i, ++n) {
        const int R = L.task[i];
        int p = 0;
        while (p + 1 < count && R >= prob[p + 1].rb_begin) ++p;
        seg_p[n] = p;
        seg_rbl[n] = R - prob[p].rb_begin;
        seg_lo[n] = 0;
        seg_n[n] = prob[p].kc;
        seg_owned[n] = 1;
      }
    } else if (ub < ue) {
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
    for (int i = 0; i < n; ++i) {
      const GemvProblem& P = prob[seg_p[i]];
      seg_full[i] = ((seg_rbl[i] + 1) * kGemvRows <= P.N && P.K % kGemvUnitK == 0) ? 1 : 0;
    }
  }
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
  auto load_w = [&](GemvBuf<NT>& buf, const Cursor& x) {
    const GemvProblem& P = prob[seg_p[x.s]];
    const int c = seg_lo[x.s] + x.off;
    if (seg_full[x.s]) {
      const size_t rowb = static_cast<size_t>(P.K) / 4;
      gemv_load_w_full(buf,
                       P.W + static_cast<size_t>(seg_rbl[x.s] * kGemvRows + g) * rowb +
                           c * (kGemvUnitK / 4) + 16 * t,
                       rowb);
    } else {
      gemv_load_w(buf, P, seg_rbl[x.s], c, g, t);
    }
  };
  auto load_x = [&](GemvBuf<NT>& buf, const Cursor& x) {
    gemv_load_x(buf, prob[seg_p[x.s]], seg_lo[x.s] + x.off, g, t);
  };

  // Warp w takes the w-th of eight equal contiguous ranges of the CTA's units
  // (in segment order): it touches one or two segments, and its loads walk
  // along the rows.
  int n_units = 0;
  for (int i = 0; i < nseg; ++i) n_units += seg_n[i];
  const int u_begin = warp * n_units / kGemvWarps;
  const int u_count = (warp + 1) * n_units / kGemvWarps - u_begin;

  // Before the activations exist: the weights of this warp's first two
  // units go to registers, and one thread asks the copy engine to stream the
  // CTA's whole row blocks (up to L.prefetch_bytes) into L2.
  GemvBuf<NT> bufA, bufB;
  Cursor xA{0, 0};
  advance(xA, u_begin);
  if (u_count == 0) xA.s = nseg;
  int left = u_count;  // units of this warp not yet loaded (xA counts as loaded)
  Cursor xB = xA;
  if (left > 1) advance(xB, 1);
  else xB.s = nseg;
  const bool early = L.early_weights != 0;
  if (early) {
    if (u_count > 0) load_w(bufA, xA);
    if (kGemvDoubleBuffer && u_count > 1) load_w(bufB, xB);
  }
  if (tid == 0 && L.prefetch_bytes > 0) {
    uint32_t left = L.prefetch_bytes;
    for (int s = 0; s < nseg && left > 0; ++s)
      if (seg_owned[s]) left -= gemv_prefetch_rows(prob[seg_p[s]], seg_rbl[s], left);
  }
  for (int i = tid; i < nseg * kGemvRows * 16; i += kGemvThreads) red[i] = 0;
  if (L.use_pdl) pdl_wait_prior_grid();
  __syncthreads();

  if (u_count > 0) {
    if (!early) load_w(bufA, xA);
    load_x(bufA, xA);
  }
  bool preB = early && u_count > 1;  // bufB already holds the next unit's weights
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
  auto enter = [&](int seg) {
    if (seg != cur_seg) {
      flush();
      cur_seg = seg;
      cur_m = prob[seg_p[seg]].M;
    }
  };
  // One token tile unless this problem has more than 8 tokens (uniform).
  auto mma = [&](const GemvBuf<NT>& buf) {
    if (NT == 2 && cur_m > 8)
      gemv_mma_unit<NT, NT>(acc, acc16, buf);
    else
      gemv_mma_unit<NT, 1>(acc, acc16, buf);
  };

  // left = units of this warp from xA on.
  if (!kGemvDoubleBuffer) {
    // One register buffer: load a unit, compute it; the other warps of the
    // SM (two CTAs) cover the load latency.
    bool loaded = u_count > 0;  // bufA holds xA (weights and activations)
    while (left > 0) {
      if (!loaded) {
        load_w(bufA, xA);
        load_x(bufA, xA);
      }
      loaded = false;
      enter(xA.s);
      mma(bufA);
      if (--left > 0) advance(xA, 1);
    }
    left = 0;
  }
  while (left > 0) {
    const bool hasB = left > 1;
    if (hasB) {
      if (!preB) {
        xB = xA;
        advance(xB, 1);
        load_w(bufB, xB);
      }
      load_x(bufB, xB);
    }
    preB = false;
    enter(xA.s);
    mma(bufA);
    if (!hasB) break;
    const bool hasA = left > 2;
    if (hasA) {
      xA = xB;
      advance(xA, 1);
      load_w(bufA, xA);
      load_x(bufA, xA);
    }
    enter(xB.s);
    mma(bufB);
    left -= 2;
  }
  flush();
  __syncthreads();

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
      const float sw = (P.y && P.s_w) ? __ldg(P.s_w) : 0.0f;
      for (int idx = tid; idx < nout; idx += kGemvThreads) {
        const int r = idx % kGemvRows, m = idx / kGemvRows, n = n0 + r;
        if (n < P.N) gemv_finish(P, sw, m, n, rs[r * 16 + m]);
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
    const float sw = (P.y && P.s_w) ? __ldg(P.s_w) : 0.0f;
    const int nout = kGemvRows * P.M;
    const int n0 = seg_rbl[s] * kGemvRows;
    for (int idx = tid; idx < nout; idx += kGemvThreads) {
      const int r = idx % kGemvRows, m = idx / kGemvRows, n = n0 + r;
      if (n < P.N) {
        const int v = atomicExch(P.ws_acc + static_cast<int64_t>(m) * P.N + n, 0);
        gemv_finish(P, sw, m, n, v);
      }
    }
    if (tid == 0) P.ws_cnt[seg_rbl[s]] = 0u;  // ready for the next call
  }
}

}  // namespace bitnet
