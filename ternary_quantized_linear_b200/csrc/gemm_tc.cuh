// gemm_tc.cuh -- ternary matmul on the 5th-generation tensor cores for any
// token count: tcgen05.mma kind::i8, A = unpacked weights held in TENSOR
// MEMORY, B = activations in shared memory, int32 accumulators in TMEM.
//
// Method: "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
// sections 計算パラダイム (integer matmul), 推論最適化とカスタムカーネル
// (weights unpacked on the fly inside the kernel), タイル化行列乗算 (tiles
// staged in fast on-chip memory so global memory is read once),
// 量子化の仕組み (rescale by both scales).
//
// A CTA computes a 128 (weight rows, TMEM lanes) x BN (tokens) tile of
// acc^T over a range of K, in 256-k steps:
//   warp 0      producer: per step the packed weight tile (128 rows x
//               KSTEP/4 bytes) -- a 2-D tensor copy from the row-major layout
//               or, with the tiled layout (tiled.cuh), one 1-D bulk copy of
//               the tile, which arrives already in the swizzled order the
//               unpack reads -- and the activation tile (BN rows of KSTEP
//               int8 as 128-byte swizzle atoms = the MMA's canonical K-major
//               layout) into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM; one thread issues KSTEP/32 MMAs (K = 32 each)
//               per step reading A from TMEM and B from shared memory;
//   warps 4-11  unpack: each thread expands 16 packed bytes of its weight
//               row (half a step) into 16 words of int8 codes t+1 (shift +
//               mask, no table) and stores them with tcgen05.st into one of
//               A_STAGES TMEM stages, so the unpack runs that many steps ahead
//               of the MMAs; after the last step the same warps read the
//               accumulators from TMEM (one lane = one weight row) and write
//               y = (acc - rowsum) / (s_x * s_w) coalesced along N, the
//               row sums, divisors and their reciprocals taken from a
//               per-tile shared-memory table built before the main loop.
// Keeping A in TMEM means the unpacked weights (4x the packed bytes) never
// touch shared memory; only the packed tile and the activation tile do.
// Code byte order: word r of packed word w holds k = 16w + 4i + r in byte i,
// stored to TMEM column 4w + r, i.e. k-position 16w + 4r + i -- the same
// k-interleaved order the activation kernel writes, so the MMA pairs equal k.
//
// Split-K (few row blocks): each CTA adds its int32 tile into a workspace
// with atomics; the last CTA of a row/token block (arrival counter, no
// waiting) reads back, re-zeroes and finishes the dequant.
//
// Every wait is bounded: on a timeout the thread records the failure in the
// device status word and raises a CTA abort flag; the kernel drains in-flight
// copies and MMAs, frees TMEM and exits without writing results.
#pragma once

#include "common.cuh"

namespace bitnet {

struct GemmParams {
  const uint8_t* Wt;      // tiled weights (tiled.cuh), when the kernel reads that layout
  int KC;                 // k chunks of the tiled layout
  const int32_t* rowsum;  // [M]
  const float* s_x;       // [M] (null: no dequant)
  const float* s_w;       // [1]
  int M, N, K;
  void* y;                // [M][N] or null
  int y_bf16;
  int32_t* acc_out;       // [M][N] debug or null
  int ksplit;             // CTAs along K (gridDim.z)
  int steps_per_split;    // KSTEP-k steps per CTA
  int32_t* ws_acc;        // [M][N] split-K partials, zero on entry (ksplit > 1)
  unsigned* ws_cnt;       // [row blocks * token blocks] counters, zero on entry
  int* status;            // device status word
  uint64_t wait_limit_ns;
  int use_pdl;            // wait for the preceding grid before touching its outputs
  // Group-wise scales (group_quant.cuh): the K split z is group z, rowsum
  // is [M][G], and each CTA writes its group's integer sums to gacc
  // [G][M][N] (no atomics, no dequant).  Null: per-tensor scales.
  int32_t* gacc;
  int G;
};

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;                 // weight rows per CTA (MMA M, TMEM lanes)
  static constexpr bool SMALL = BN <= 64;        // decode-sized token tile
  // 256 k per pipeline step: each TMA weight box has 64-byte rows (narrower
  // rows starve the copy engine) and each step issues 8 MMAs, amortising the
  // per-step barrier traffic.  Token tiles up to 128 run two CTAs per SM:
  // small tiles are bound by the MMA issue rate (a fixed cost per
  // instruction) and interleave two MMA streams; 128-token tiles overlap one
  // CTA's pipeline fill and epilogue with the other's main loop (the host
  // picks them for short K, where those per-tile costs dominate); 256-token
  // tiles are tensor-bound, one CTA/SM.
  static constexpr int KSTEP = 256;
  static constexpr int ATOMS = KSTEP / 128;      // 128-byte swizzle atoms per activation tile
  static constexpr int X_ATOM = BN * 128;        // bytes of one activation atom
  static constexpr int X_BYTES = BN * KSTEP;     // activation tile
  static constexpr int WP_ROW = KSTEP / 4;       // packed bytes per weight row per step
  static constexpr int WP_BYTES = BM * WP_ROW;   // packed weight tile
  static constexpr bool TWO_PER_SM = BN <= 128;
  static constexpr int STAGES = BN <= 16 ? 8 : (BN <= 32 ? 6 : (BN <= 64 ? 4 : (BN <= 128 ? 2 : 3)));
  // TMEM: A_STAGES stages of KSTEP/4 columns of unpacked weights (four int8
  // k per 32-bit column, one lane per weight row), then BN int32 accumulator
  // columns.
  static constexpr int A_COLS = KSTEP / 4;
  static constexpr int A_STAGES = SMALL ? 3 : (TWO_PER_SM ? 2 : STAGES);
  static constexpr uint32_t A_COL = 0;
  static constexpr uint32_t D_COL = A_COLS * A_STAGES;
  static constexpr uint32_t TMEM_COLS = TWO_PER_SM ? 256 : 512;
  static constexpr int MIN_BLOCKS = TWO_PER_SM ? 2 : 1;
  static constexpr int UNPACK_WARPS = 8;         // two per TMEM lane quarter
  static constexpr int THREADS = 128 + 32 * UNPACK_WARPS;
  static constexpr int PART = WP_ROW / 2;        // packed bytes per unpack thread per step
  static constexpr int OFF_X = 0;
  static constexpr int OFF_WP = OFF_X + STAGES * X_BYTES;
  static constexpr int OFF_BAR = OFF_WP + STAGES * WP_BYTES;
  static constexpr int NBAR = 3 * STAGES + A_STAGES + 1;  // fullw/fullx/done, aready, accfull
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_TAB = (OFF_MISC + 16 + 15) & ~15;  // epilogue table: one int4 per token
  static constexpr int BYTES = OFF_TAB + 16 * BN;
  static constexpr int SMEM_DYN = BYTES + 1024;  // slack for 1024-byte alignment
  static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
  static_assert(A_STAGES <= STAGES, "A stages are recycled through the stage barriers");
  static_assert(D_COL + BN <= TMEM_COLS, "tensor memory");
  static_assert(OFF_TAB % 16 == 0, "the epilogue table is read as int4");
  static_assert(X_ATOM % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");
  static_assert(PART % 16 == 0, "unpack reads 16-byte words");
  static_assert(WP_ROW == 64, "weight tile swizzle");
  static_assert(SMEM_DYN * MIN_BLOCKS <= 232448, "shared memory");
};

__device__ __forceinline__ void gemm_fail(volatile int* abort_flag, int* status, int detail) {
  *abort_flag = 1;
  record_failure(status, detail);
}

// All 32 lanes wait on `bar`; the verdict is made warp-uniform (tcgen05
// loads/stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          const volatile int* abort_flag, uint64_t limit) {
  const bool ok = mbar_wait_bounded(bar, parity, abort_flag, limit);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, int8 x int8 -> int32, one CTA.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One output: e = the tile's epilogue entry of token m, {row sum, divisor
// s_x * s_w, RN(1 / divisor)} (the last two as float bits).
// kFast: every divisor of the tile passed recip_for_div (no per-output test).
template <bool kFast = false>
__device__ __forceinline__ void gemm_store(const GemmParams& p, int4 e, int m, int n, int acc_codes) {
  const int acc = acc_codes - e.x;
  const int64_t o = static_cast<int64_t>(m) * p.N + n;
  if (p.acc_out) p.acc_out[o] = acc;
  if (p.y) {
    const float yv =
        kFast ? div_rn_int_fast(__int2float_rn(acc), __int_as_float(e.y), __int_as_float(e.z))
              : div_rn_int(__int2float_rn(acc), __int_as_float(e.y), __int_as_float(e.z));
    if (p.y_bf16)
      reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(yv);
    else
      reinterpret_cast<float*>(p.y)[o] = yv;
  }
}

template <int BN, bool kTiledW>
__global__ void __launch_bounds__(GemmCfg<BN>::THREADS, GemmCfg<BN>::MIN_BLOCKS)
ternary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_w, const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* xs = smem + C::OFF_X;
  uint8_t* wps = smem + C::OFF_WP;
  // fullw[s]: the step's weight tile landed; fullx[s]: its activation tile
  //          (both atoms) landed (TMA transaction bytes).
  // done[s]: the step's MMAs completed (one tcgen05.commit) -- which also
  //          means the unpack warps had finished reading its weight tile,
  //          since the MMAs waited for them; it frees the shared-memory stage
  //          for the producers and, A_STAGES steps later, the TMEM A stage.
  // aready[a]: the unpack warps stored TMEM A stage a.
  uint64_t* fullw = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* fullx = fullw + C::STAGES;
  uint64_t* done = fullx + C::STAGES;
  uint64_t* aready = done + C::STAGES;
  uint64_t* accfull = aready + C::A_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* is_last = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  int* all_fast = reinterpret_cast<int*>(smem + C::OFF_MISC + 12);   // every divisor in range
  int4* tab = reinterpret_cast<int4*>(smem + C::OFF_TAB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::BM;
  const int m0 = blockIdx.y * BN;
  const int total_steps = (p.K + C::KSTEP - 1) / C::KSTEP;
  const int kb0 = blockIdx.z * p.steps_per_split;
  const int kb1 = min(kb0 + p.steps_per_split, total_steps);
  const int nk = kb1 - kb0;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&fullw[s], 1);
      mbar_init(&fullx[s], 1);
      mbar_init(&done[s], 1);                     // MMA commit
    }
    for (int a = 0; a < C::A_STAGES; ++a) mbar_init(&aready[a], C::UNPACK_WARPS);
    mbar_init(accfull, 1);
    *abort_flag = 0;
    *all_fast = 1;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    if (!kTiledW) tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  // Set-up above overlaps the preceding grid; its outputs (activations, row
  // sums, scales) are read only after this point.
  if (p.use_pdl) pdl_wait_prior_grid();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // One thread issues the step's three copies (the weight tile, then the
      // two activation atoms): splitting them over three threads measured
      // slower on prefill.
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int s = j % C::STAGES;
        const uint32_t use = static_cast<uint32_t>(j / C::STAGES);
        if (j >= C::STAGES && !mbar_wait_bounded(&done[s], (use - 1u) & 1u, abort_flag, limit)) {
          gemm_fail(abort_flag, p.status, DEV_TIMEOUT_PRODUCER);
          break;
        }
        const int kb = kb0 + j;
        mbar_arrive_expect_tx(&fullw[s], C::WP_BYTES);
        if (kTiledW)
          bulk_load(wps + s * C::WP_BYTES,
                    p.Wt + (static_cast<int64_t>(blockIdx.x) * p.KC + kb) * C::WP_BYTES,
                    C::WP_BYTES, &fullw[s]);
        else
          tma_load_2d(wps + s * C::WP_BYTES, &tmap_w, kb * C::WP_ROW, n0, &fullw[s]);
        mbar_arrive_expect_tx(&fullx[s], C::X_BYTES);
#pragma unroll
        for (int at = 0; at < C::ATOMS; ++at)
          tma_load_2d(xs + s * C::X_BYTES + at * C::X_ATOM, &tmap_x, kb * C::KSTEP + 128 * at, m0,
                      &fullx[s]);
        issued = j + 1;
      }
      if (*abort_flag) {
        // Let the copies already in flight land before the CTA exits.
        const int first = issued > C::STAGES ? issued - C::STAGES : 0;
        for (int j = first; j < issued; ++j) {
          const int s = j % C::STAGES;
          const uint32_t par = static_cast<uint32_t>(j / C::STAGES) & 1u;
          if (!mbar_wait_bounded(&fullw[s], par, nullptr, limit) ||
              !mbar_wait_bounded(&fullx[s], par, nullptr, limit))
            record_failure(p.status, DEV_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t idesc = umma_idesc_i8(C::BM, BN);
      const uint32_t d_tmem = tmem_base + C::D_COL;
      for (int j = 0; j < nk; ++j) {
        const int s = j % C::STAGES, a = j % C::A_STAGES;
        // The unpacked weights (aready) and the activation tile (fullx).
        if (!mbar_wait_bounded(&aready[a], static_cast<uint32_t>(j / C::A_STAGES) & 1u,
                               abort_flag, limit) ||
            !mbar_wait_bounded(&fullx[s], static_cast<uint32_t>(j / C::STAGES) & 1u, abort_flag,
                               limit)) {
          gemm_fail(abort_flag, p.status, DEV_TIMEOUT_MMA);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_tmem = tmem_base + C::A_COL + static_cast<uint32_t>(C::A_COLS) * a;
        const uint32_t b_base = smem_u32(xs + s * C::X_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::KSTEP / 32; ++kk)
          tc_mma_i8_ts(d_tmem, a_tmem + 8u * kk,
                       umma_desc_sw128_kmajor(b_base + (kk >> 2) * C::X_ATOM + 32 * (kk & 3)),
                       idesc, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&done[s]);
      }
      // Signals the epilogue; on an abort it still marks that every MMA
      // issued so far has finished with TMEM and shared memory.
      tc_commit(accfull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- unpack
    // Warp 4+u: TMEM lane quarter q = u % 4 (rows 32q..32q+31), half h = u / 4
    // of each step's packed bytes (PART bytes -> PART TMEM columns).
    const int u = warp - 4;
    const int q = u & 3, h = u >> 2;
    const int i = 32 * q + lane;        // weight row inside the tile
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    // Epilogue table of this tile's tokens, built while the first copies are
    // in flight: row sum, divisor s_x * s_w and its correctly rounded
    // reciprocal, so each output costs a multiply and four FMAs instead of
    // a division.  Only the unpack warps read it before the final barrier.
    {
      const float swv = (p.y && p.s_w) ? *p.s_w : 0.0f;
      for (int c = threadIdx.x - 128; c < BN; c += 32 * C::UNPACK_WARPS) {
        const int m = m0 + c;
        int rs = 0;
        float d = 1.0f;
        if (m < p.M) {
          rs = p.gacc ? p.rowsum[m * p.G + blockIdx.z] : p.rowsum[m];
          if (p.y) d = __fmul_rn(p.s_x[m], swv);
        }
        const float y = recip_for_div(d);
        if (y == 0.0f) atomicAnd(all_fast, 0);
        tab[c] = make_int4(rs, __float_as_int(d), __float_as_int(y), 0);
      }
      named_barrier_sync(1, 32 * C::UNPACK_WARPS);
    }
    for (int j = 0; j < nk; ++j) {
      const int s = j % C::STAGES, a = j % C::A_STAGES;
      // A stage a was last used by step j - A_STAGES; its MMAs completed when
      // done[] of that step's shared-memory stage did.
      const int jp = j - C::A_STAGES;
      if (!warp_wait(&fullw[s], static_cast<uint32_t>(j / C::STAGES) & 1u, abort_flag, limit) ||
          (jp >= 0 && !warp_wait(&done[jp % C::STAGES],
                                 static_cast<uint32_t>(jp / C::STAGES) & 1u, abort_flag, limit))) {
        gemm_fail(abort_flag, p.status, DEV_TIMEOUT_UNPACK);
        break;
      }
      tc_fence_after_sync();
      constexpr int NV = C::PART / 16;  // 16-byte words of packed codes per thread
      uint4 pk[NV];
#pragma unroll
      for (int t = 0; t < NV; ++t) {
        // The copy engine wrote the tile swizzled (64-byte rows: chunk ^
        // (row/2)%4) so a warp's 32 rows hit distinct banks.
        const int c = (C::PART / 16) * h + t;
        const int pc = c ^ ((i >> 1) & 3);
        pk[t] = *reinterpret_cast<const uint4*>(wps + s * C::WP_BYTES + i * C::WP_ROW + 16 * pc);
      }
      const uint32_t col = tmem_base + lane_addr + C::A_COL + static_cast<uint32_t>(C::A_COLS) * a +
                           static_cast<uint32_t>(C::PART) * h;
#pragma unroll
      for (int t = 0; t < NV; ++t) {
        const uint32_t words[4] = {pk[t].x, pk[t].y, pk[t].z, pk[t].w};
        uint32_t v[16];
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int r = 0; r < 4; ++r) v[4 * w + r] = (words[w] >> (2 * r)) & 0x03030303u;
        tmem_st_32x32b_x16(col + 16u * t, v);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[a]);
    }
    // ----------------------------------------------------------- epilogue
    // Warps of half h take accumulator columns [h*BN/2, (h+1)*BN/2) (all of
    // them when BN == 16, with half 1 idle).
    const bool done = warp_wait(accfull, 0u, nullptr, limit);
    if (!done) gemm_fail(abort_flag, p.status, DEV_TIMEOUT_EPILOGUE);
    tc_fence_after_sync();
    const bool write = __all_sync(0xFFFFFFFFu, done && *abort_flag == 0);
    constexpr int kHalf = BN >= 32 ? BN / 2 : BN;
    if (write && (BN >= 32 || h == 0)) {
      const int n = n0 + i;
      const bool split = p.ksplit > 1 && !p.gacc;
      // The common case -- a plain tile whose divisors all passed -- runs a
      // loop with no per-output test.
      const bool fast = !split && !p.gacc && *all_fast != 0;
      for (int c0 = h * kHalf; c0 < (h + 1) * kHalf; c0 += 16) {
        if (m0 + c0 >= p.M) break;  // uniform across the warp
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem_base + lane_addr + C::D_COL + c0, r);
        tmem_ld_wait();
        if (n < p.N && fast) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int m = m0 + c0 + jj;
            if (m < p.M) gemm_store<true>(p, tab[c0 + jj], m, n, static_cast<int>(r[jj]));
          }
        } else if (n < p.N) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int m = m0 + c0 + jj;
            if (m < p.M) {
              if (p.gacc)
                p.gacc[(static_cast<int64_t>(blockIdx.z) * p.M + m) * p.N + n] =
                    static_cast<int>(r[jj]) - tab[c0 + jj].x;
              else if (split)
                atomicAdd(p.ws_acc + static_cast<int64_t>(m) * p.N + n, static_cast<int>(r[jj]));
              else
                gemm_store(p, tab[c0 + jj], m, n, static_cast<int>(r[jj]));
            }
          }
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }

  // Split-K: the last CTA of this output tile finishes (no waiting).
  if (p.ksplit > 1 && !p.gacc) {
    const int ok = __syncthreads_and(*abort_flag == 0 ? 1 : 0);
    if (!ok) return;
    const int tile = blockIdx.y * gridDim.x + blockIdx.x;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      *is_last = (atomicAdd(p.ws_cnt + tile, 1u) == static_cast<unsigned>(p.ksplit - 1)) ? 1 : 0;
    __syncthreads();
    if (!*is_last) return;
    __threadfence();
    const int rows = min(C::BM, p.N - n0), toks = min(BN, p.M - m0);
    for (int idx = threadIdx.x; idx < rows * toks; idx += blockDim.x) {
      const int r = idx % rows, c = idx / rows, n = n0 + r;
      const int v = atomicExch(p.ws_acc + static_cast<int64_t>(m0 + c) * p.N + n, 0);
      gemm_store(p, tab[c], m0 + c, n, v);
    }
    if (threadIdx.x == 0) p.ws_cnt[tile] = 0u;  // ready for the next call
  }
}

}  // namespace bitnet
